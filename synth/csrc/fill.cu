// Device-side bulk fill of the seeded synthetic bf16 inputs.
//
// Input generation only: no part of the retrieve-and-inject arithmetic lives
// here.  The definition (SplitMix64 output function over a counter, twelve
// 10-bit fields summed into an Irwin-Hall(12) variate, round to bf16) is the
// one documented in synth/__init__.py; both implementations use integer
// arithmetic and an exact int->float conversion, so they agree bit for bit.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z ^= z >> 30; z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27; z *= 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ inline uint16_t sample_bf16(uint64_t key, uint64_t n) {
  const uint64_t base = key + (2ull * n) * kGamma;
  int s = 0;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const uint64_t w = mix64(base + uint64_t(j) * kGamma);
#pragma unroll
    for (int i = 0; i < 6; ++i) s += int((w >> (10 * i)) & 1023ull);
  }
  const float x = float(s - 6138) * (1.0f / 1024.0f);  // exact: |s-6138| < 2^13
  uint32_t u = __float_as_uint(x);
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
  return uint16_t(u);
}

__global__ void fill_kernel(uint16_t* __restrict__ dst, int64_t count, uint64_t key, int64_t base) {
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += stride)
    dst[i] = sample_bf16(key, uint64_t(base + i));
}

}  // namespace

extern "C" int synth_fill_bf16(void* dst, int64_t count, uint64_t seed, uint64_t stream,
                               int64_t base, void* cuda_stream) {
  if (count <= 0) return 0;
  if (dst == nullptr) return int(cudaErrorInvalidValue);
  const uint64_t key = mix64(seed * kGamma + stream);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (count + 255) / 256;
  if (blocks > int64_t(sms) * 16) blocks = int64_t(sms) * 16;
  fill_kernel<<<int(blocks), 256, 0, static_cast<cudaStream_t>(cuda_stream)>>>(
      static_cast<uint16_t*>(dst), count, key, base);
  return int(cudaGetLastError());
}
