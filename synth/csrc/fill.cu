// Device-side bulk fill of the seeded synthetic bf16 inputs.
//
// Input generation only: no part of the retrieve-and-inject arithmetic lives
// here.  The definition (SplitMix64 output function over a counter; the
// magnitude is the bf16 code whose standard-normal rounding interval holds
// the quantile w_0 / 2^64, found in an integer threshold table; the sign is
// the top bit of w_1) is the one documented in synth/__init__.py, which also
// builds the table and hands it over.  Both implementations use integer
// arithmetic only, so they agree bit for bit.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;
constexpr int kMaxTable = 12288;   // thresholds held (the table has ~8.7k)
constexpr int kMaxDevices = 64;
constexpr int kThreads = 256;

__device__ uint64_t g_q[kMaxTable];
bool g_ready[kMaxDevices] = {};
int g_n = 0, g_first = 0;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z ^= z >> 30; z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27; z *= 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void __launch_bounds__(kThreads) fill_kernel(uint16_t* __restrict__ dst, int64_t count,
                                                        uint64_t key, int64_t base, int n, int first) {
  extern __shared__ uint64_t q[];  // [n] thresholds
  for (int i = threadIdx.x; i < n; i += blockDim.x) q[i] = g_q[i];
  __syncthreads();
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += stride) {
    const uint64_t b = key + (2ull * uint64_t(base + i)) * kGamma;
    const uint64_t w0 = mix64(b), w1 = mix64(b + kGamma);
    int lo = 0, len = n;  // number of thresholds <= w0
    while (len > 0) {
      const int half = len >> 1;
      if (q[lo + half] <= w0) {
        lo += half + 1;
        len -= half + 1;
      } else {
        len = half;
      }
    }
    dst[i] = uint16_t((first + lo) | int((w1 >> 63) << 15));
  }
}

}  // namespace

// Fill `count` bf16 values at device address `dst` with elements base ..
// base + count of a stream; `table` (host, n entries) and `first` are the
// threshold table and its first code (synth.normal_table), copied to the
// current device on its first fill.  Asynchronous on `cuda_stream`.  Returns
// a cudaError_t value (0 on success).
extern "C" int synth_fill_bf16(void* dst, int64_t count, uint64_t seed, uint64_t stream,
                               int64_t base, const uint64_t* table, int n, int first,
                               void* cuda_stream) {
  if (count <= 0) return 0;
  if (dst == nullptr || table == nullptr || n < 1 || n > kMaxTable) return int(cudaErrorInvalidValue);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return int(cudaErrorInvalidDevice);
  if (!g_ready[dev] || g_n != n || g_first != first) {
    cudaError_t e = cudaMemcpyToSymbol(g_q, table, sizeof(uint64_t) * size_t(n));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(sizeof(uint64_t) * kMaxTable));
    if (e != cudaSuccess) return int(e);
    g_ready[dev] = true;
    g_n = n;
    g_first = first;
  }
  const uint64_t key = mix64(seed * kGamma + stream);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // At least 64 elements per thread, so each CTA's copy of the table into
  // shared memory is paid for; at most two CTAs per SM.
  int64_t blocks = (count + kThreads * 64 - 1) / (kThreads * 64);
  if (blocks > int64_t(sms) * 2) blocks = int64_t(sms) * 2;
  fill_kernel<<<int(blocks), kThreads, sizeof(uint64_t) * size_t(n), static_cast<cudaStream_t>(cuda_stream)>>>(
      static_cast<uint16_t*>(dst), count, key, base, n, first);
  return int(cudaGetLastError());
}
