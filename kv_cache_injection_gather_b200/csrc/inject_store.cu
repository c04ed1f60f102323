// Host side of libinjectstore.so: the fact store (device or pinned-host tier,
// static or LRU hot set), the C-ABI declared in include/inject_store.h, the
// launches of the kernels in inject_kernels.cuh, and the allocation-free
// entry point at the end of the file.
#include <cuda_runtime.h>

#include <algorithm>
#include <chrono>
#include <cstdint>
#include <cstring>
#include <list>
#include <new>
#include <thread>
#include <vector>

#include "inject_store.h"
#include "inject_kernels.cuh"

namespace {

constexpr int kPlanThreads = 1024;
// Inject-kernel launch shape (compile-time knobs; the defaults are the
// measured best on B200 for the Llama-3.1-8B-shaped batch).
#ifndef IS_INJECT_THREADS
#define IS_INJECT_THREADS 256
#endif
#ifndef IS_INJECT_VECS
#define IS_INJECT_VECS 8
#endif
#ifndef IS_INJECT_MIN_BLOCKS
#define IS_INJECT_MIN_BLOCKS 2
#endif
constexpr int kInjectThreads = IS_INJECT_THREADS;
constexpr int kVecsPerThread = IS_INJECT_VECS;
constexpr int kInjectMinBlocks = IS_INJECT_MIN_BLOCKS;
// The single-kernel path for short batches has its own launch shape: its
// batches fit about one wave, so more, lighter CTAs per SM can help there.
#ifndef IS_SMALL_VECS
#define IS_SMALL_VECS IS_INJECT_VECS
#endif
#ifndef IS_SMALL_MIN_BLOCKS
#define IS_SMALL_MIN_BLOCKS IS_INJECT_MIN_BLOCKS
#endif
constexpr int kSmallVecsPerThread = IS_SMALL_VECS;
constexpr int kSmallMinBlocks = IS_SMALL_MIN_BLOCKS;
constexpr int kDefaultMaxRequests = 4096;
constexpr int kDefaultMaxFactIds = 1 << 20;
constexpr int kMaxTimedLaunches = 4096;
// single-kernel path: ids x the longest fact at most this (its sums are 32-bit)
constexpr int64_t kSmallSumLimit = (int64_t(1) << 31) - 1;

struct TimedLaunch {
  cudaEvent_t start, stop;
};

}  // namespace

struct is_store {
  is_store_config_t cfg{};
  int device = 0;
  int sm_count = 148;
  // arenas [L][H][T_cap][D] bf16
  uint16_t* k = nullptr;
  uint16_t* v = nullptr;
  bool host_arena = false;
  // host tier: device-mapped views of the pinned arenas and the HBM hot set
  uint16_t* k_view = nullptr;
  uint16_t* v_view = nullptr;
  uint16_t* k_hot = nullptr;
  uint16_t* v_hot = nullptr;
  int64_t hot_cap = 0;
  int64_t hot_used = 0;
  int32_t hot_facts = 0;
  int64_t* d_hot = nullptr;
  std::vector<int64_t> h_hot;
  // least-recently-used hot set (IS_HOT_LRU): fixed slots of slot_tokens
  int hot_policy = IS_HOT_STATIC;
  int32_t slot_tokens = 0;
  std::vector<int32_t> slot_owner;                   // fact in each slot, -1 free
  std::vector<uint64_t> slot_tick;                   // last touch that used it
  std::list<int32_t> lru;                            // slots, most recent first
  std::vector<std::list<int32_t>::iterator> lru_at;  // position of each slot
  std::vector<uint64_t> fact_tick;                   // last touch that asked for it
  uint64_t tick = 0;
  int64_t lru_hits = 0, lru_misses = 0, lru_promoted = 0, lru_promoted_tokens = 0;
  // promotion staging: pinned host list + device copy, reused after `touch_done`
  isk::Promotion* h_promo = nullptr;
  isk::Promotion* d_promo = nullptr;
  int64_t* h_pairs = nullptr;
  int64_t* d_pairs = nullptr;
  size_t promo_cap = 0;
  cudaEvent_t touch_done = nullptr;
  // promotion fused into the next batch (is_inject_batch_host): per-fact hot
  // token of a pending promotion (-1: none), and the pending lists' sizes
  int64_t* d_pend = nullptr;
  size_t pend_ne = 0, pend_np = 0;
  bool batch_pend = false;   // the batch being launched reads d_pend
  // prefetch of the next batch's cold facts (is_inject_batch_host_next):
  // copy-engine transfers on copy_stream; the next batch waits for pf_done
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t pf_done = nullptr;
  bool pf_pending = false;
  uint64_t batch_tick = 0;   // LRU tick of the last host-entry batch
  int64_t* h_pf_pairs = nullptr;
  int64_t* d_pf_pairs = nullptr;
  isk::Promotion* h_pf_promo = nullptr;
  isk::Promotion* d_pf_promo = nullptr;
  size_t pf_cap = 0;         // pairs (and promotions)
  // fact table
  int64_t* d_off = nullptr;
  int32_t* d_len = nullptr;
  std::vector<int64_t> h_off;
  std::vector<int32_t> h_len;
  int64_t used_tokens = 0;
  int32_t num_facts = 0;
  int32_t max_len = 0;        // longest fact put so far
  double* d_inv_freq = nullptr;
  // per-batch work space
  int32_t max_req = 0, max_ids = 0, max_blocks = 0;
  int32_t* ws_seg = nullptr;
  int32_t* ws_nblk = nullptr;
  int32_t* ws_blk0 = nullptr;
  long long* ws_tok0 = nullptr;
  int32_t* ws_len = nullptr;
  int32_t* ws_err = nullptr;
  isk::BlockDesc* ws_desc = nullptr;
  isk::PlanHeader* ws_hdr = nullptr;
  isk::DevStatus* d_status = nullptr;
  // staging for is_inject_batch_host
  int32_t* stage = nullptr;
  size_t stage_elems = 0;
  int32_t* host_stage = nullptr;   // pinned mirror of `stage`
  isk::DevStatus* host_status = nullptr;  // pinned, mapped
  isk::DevStatus* host_status_dev = nullptr;  // its device address
  isk::DevStatus* batch_mirror = nullptr;     // set while the host entry point runs a batch
  int64_t* stage_slots = nullptr;
  int64_t stage_slot_elems = 0;
  // timing
  bool timing = false;
  std::vector<TimedLaunch> events;
  size_t events_used = 0;
  // fact-sharded view (is_store_attach_shards): arenas of several stores and
  // a global fact table; batches take global ids while it is attached
  int32_t shard_n = 0;
  int32_t shard_facts = 0;
  const uint16_t** d_shard_k = nullptr;
  const uint16_t** d_shard_v = nullptr;
  int64_t* d_shard_plane = nullptr;  // elements between (l,h) planes
  int32_t* d_shard_of = nullptr;     // [shard_facts]
  int64_t* d_shard_off = nullptr;
  int32_t* d_shard_len = nullptr;
  int32_t shard_max_len = 0;
  // kernel configuration
  int inject_grid = 0;
  int small_grid = 0;        // resident CTAs of the single-kernel path
  unsigned int* d_small_ctr = nullptr;  // its unit counter (zero between batches)
  int32_t small_limit = isk::kSmallRequests;  // batches up to this many requests: one kernel
};

namespace {

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

template <typename T>
cudaError_t dalloc(T** p, size_t count) {
  return cudaMalloc(reinterpret_cast<void**>(p), std::max<size_t>(count, 1) * sizeof(T));
}

struct ShardView {
  const uint16_t** k = nullptr;
  const uint16_t** v = nullptr;
  int64_t* plane = nullptr;
  int32_t* of = nullptr;
  int64_t* off = nullptr;
  int32_t* len = nullptr;
  void release() {
    cudaFree(k);
    cudaFree(v);
    cudaFree(plane);
    cudaFree(of);
    cudaFree(off);
    cudaFree(len);
    *this = ShardView{};
  }
};

void free_view(is_store* s) {
  ShardView{s->d_shard_k, s->d_shard_v, s->d_shard_plane, s->d_shard_of, s->d_shard_off, s->d_shard_len}
      .release();
  s->d_shard_k = s->d_shard_v = nullptr;
  s->d_shard_plane = s->d_shard_off = nullptr;
  s->d_shard_of = s->d_shard_len = nullptr;
  s->shard_n = s->shard_facts = 0;
  s->shard_max_len = 0;
}

void free_store(is_store* s) {
  if (!s) return;
  free_view(s);
  cudaFree(s->d_off);
  cudaFree(s->d_len);
  cudaFree(s->d_inv_freq);
  cudaFree(s->ws_seg);
  cudaFree(s->ws_nblk);
  cudaFree(s->ws_blk0);
  cudaFree(s->ws_tok0);
  cudaFree(s->ws_len);
  cudaFree(s->ws_err);
  cudaFree(s->ws_desc);
  cudaFree(s->ws_hdr);
  cudaFree(s->d_status);
  cudaFree(s->d_small_ctr);
  cudaFree(s->stage);
  cudaFree(s->stage_slots);
  cudaFreeHost(s->host_stage);
  cudaFreeHost(s->host_status);
  cudaFree(s->k_hot);
  cudaFree(s->v_hot);
  cudaFree(s->d_hot);
  cudaFreeHost(s->h_promo);
  cudaFreeHost(s->h_pairs);
  cudaFree(s->d_promo);
  cudaFree(s->d_pairs);
  cudaFree(s->d_pend);
  if (s->touch_done) cudaEventDestroy(s->touch_done);
  if (s->pf_done) cudaEventDestroy(s->pf_done);
  if (s->copy_stream) cudaStreamDestroy(s->copy_stream);
  cudaFreeHost(s->h_pf_pairs);
  cudaFree(s->d_pf_pairs);
  cudaFreeHost(s->h_pf_promo);
  cudaFree(s->d_pf_promo);
  if (s->host_arena) {
    cudaFreeHost(s->k);
    cudaFreeHost(s->v);
  } else {
    cudaFree(s->k);
    cudaFree(s->v);
  }
  for (auto& e : s->events) {
    cudaEventDestroy(e.start);
    cudaEventDestroy(e.stop);
  }
  delete s;
}

bool head_dim_supported(int d) { return d == 32 || d == 64 || d == 128 || d == 256; }

template <int D, int STYLE, bool POW2, bool HOST_TIER, int HC = 0, int BC = 0, int FAST = 0>
void* inject_fn() {
  return reinterpret_cast<void*>(&isk::inject_kernel<D, STYLE, kInjectThreads, kVecsPerThread,
                                                     kInjectMinBlocks, POW2, HOST_TIER, HC, BC, FAST>);
}



template <int D, int STYLE, bool POW2, bool HOST_TIER, int HC = 0, int BC = 0, int FAST = 0>
void* small_fn() {
  return reinterpret_cast<void*>(&isk::small_inject_kernel<D, STYLE, kInjectThreads, kSmallVecsPerThread,
                                                           kSmallMinBlocks, POW2, HOST_TIER, HC, BC, FAST>);
}

template <bool POW2, bool HOST_TIER = false>
void* pick_small_t(int D, int style) {
  switch (D) {
    case 32: return style ? small_fn<32, 1, POW2, HOST_TIER>() : small_fn<32, 0, POW2, HOST_TIER>();
    case 64: return style ? small_fn<64, 1, POW2, HOST_TIER>() : small_fn<64, 0, POW2, HOST_TIER>();
    case 128: return style ? small_fn<128, 1, POW2, HOST_TIER>() : small_fn<128, 0, POW2, HOST_TIER>();
    case 256: return style ? small_fn<256, 1, POW2, HOST_TIER>() : small_fn<256, 0, POW2, HOST_TIER>();
    default: return nullptr;
  }
}

// Compile-time shapes for the common models (D = 128, block size 16, 4 or 8
// KV heads: Llama-3.1-8B, Mistral-7B, Qwen2.5-7B): the per-vector index
// arithmetic folds to constants.  Returns nullptr for other shapes.
template <bool SMALL, bool HOST_TIER, int HC, int FAST>
void* fixed_fn(int style) {
  return SMALL ? (style ? small_fn<128, 1, true, HOST_TIER, HC, 16, (FAST == 2 ? 1 : FAST)>()
                        : small_fn<128, 0, true, HOST_TIER, HC, 16, FAST>())
               : (style ? inject_fn<128, 1, true, HOST_TIER, HC, 16, (FAST == 2 ? 1 : FAST)>()
                        : inject_fn<128, 0, true, HOST_TIER, HC, 16, FAST>());
}

// loop: the copy loop of the launch -- 0 generic, 1 per-thread, 2 per-thread
// with both rotate-half halves in one thread (device tier, rotate-half only;
// other cases fall back to 1).
template <bool SMALL, bool HOST_TIER>
void* pick_fixed(int D, int style, int H, int B, int loop) {
#ifndef IS_NO_FIXED_SHAPES
  if (D != 128 || B != 16) return nullptr;
  if (loop == 2 && (HOST_TIER || style != 0)) loop = 1;
  if (H == 8)
    return loop == 2 ? fixed_fn<SMALL, HOST_TIER, 8, (HOST_TIER ? 1 : 2)>(style)
         : loop == 1 ? fixed_fn<SMALL, HOST_TIER, 8, 1>(style)
                     : fixed_fn<SMALL, HOST_TIER, 8, 0>(style);
  if (H == 4)
    return loop == 2 ? fixed_fn<SMALL, HOST_TIER, 4, (HOST_TIER ? 1 : 2)>(style)
         : loop == 1 ? fixed_fn<SMALL, HOST_TIER, 4, 1>(style)
                     : fixed_fn<SMALL, HOST_TIER, 4, 0>(style);
#else
  (void)D; (void)style; (void)H; (void)B; (void)loop;
#endif
  return nullptr;
}

template <bool POW2, bool HOST_TIER = false>
void* pick_inject_t(int D, int style) {
  switch (D) {
    case 32: return style ? inject_fn<32, 1, POW2, HOST_TIER>() : inject_fn<32, 0, POW2, HOST_TIER>();
    case 64: return style ? inject_fn<64, 1, POW2, HOST_TIER>() : inject_fn<64, 0, POW2, HOST_TIER>();
    case 128: return style ? inject_fn<128, 1, POW2, HOST_TIER>() : inject_fn<128, 0, POW2, HOST_TIER>();
    case 256: return style ? inject_fn<256, 1, POW2, HOST_TIER>() : inject_fn<256, 0, POW2, HOST_TIER>();
    default: return nullptr;
  }
}

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// The inject kernel for a head dim, RoPE style and (H, B): the shift variant
// when both are powers of two; the host-tier variant for stores in pinned
// host memory.
void* pick_inject(int D, int style, int H, int B, bool host_tier = false, int loop = 0) {
  if (void* f = host_tier ? pick_fixed<false, true>(D, style, H, B, loop) : pick_fixed<false, false>(D, style, H, B, loop))
    return f;
  const bool p2 = is_pow2(H) && is_pow2(B);
  if (host_tier) return p2 ? pick_inject_t<true, true>(D, style) : pick_inject_t<false, true>(D, style);
  return p2 ? pick_inject_t<true>(D, style) : pick_inject_t<false>(D, style);
}

// The single-kernel variant for small batches, same selection.
void* pick_small(int D, int style, int H, int B, bool host_tier, int loop) {
  if (void* f = host_tier ? pick_fixed<true, true>(D, style, H, B, loop) : pick_fixed<true, false>(D, style, H, B, loop))
    return f;
  const bool p2 = is_pow2(H) && is_pow2(B);
  if (host_tier) return p2 ? pick_small_t<true, true>(D, style) : pick_small_t<false, true>(D, style);
  return p2 ? pick_small_t<true>(D, style) : pick_small_t<false>(D, style);
}

size_t cs_smem_bytes(int D, int B) { return size_t(B) * size_t(D / 2) * sizeof(float2); }

int grow_stage(is_store* s, size_t elems, int64_t slot_elems) {
  if (elems > s->stage_elems) {
    cudaFree(s->stage);
    cudaFreeHost(s->host_stage);
    s->stage = nullptr;
    s->host_stage = nullptr;
    s->stage_elems = 0;
    if (dalloc(&s->stage, elems) != cudaSuccess) return IS_ERR_OOM;
    if (cudaHostAlloc(reinterpret_cast<void**>(&s->host_stage), elems * sizeof(int32_t),
                      cudaHostAllocDefault) != cudaSuccess)
      return IS_ERR_OOM;
    s->stage_elems = elems;
  }
  if (!s->host_status) {
    if (cudaHostAlloc(reinterpret_cast<void**>(&s->host_status), sizeof(isk::DevStatus),
                      cudaHostAllocMapped) != cudaSuccess)
      return IS_ERR_OOM;
    if (cudaHostGetDevicePointer(reinterpret_cast<void**>(&s->host_status_dev), s->host_status, 0) !=
        cudaSuccess) {
      cudaGetLastError();
      s->host_status_dev = nullptr;  // not mapped: the status is copied back instead
    }
  }
  if (slot_elems > s->stage_slot_elems) {
    cudaFree(s->stage_slots);
    s->stage_slots = nullptr;
    s->stage_slot_elems = 0;
    if (dalloc(&s->stage_slots, size_t(slot_elems)) != cudaSuccess) return IS_ERR_OOM;
    s->stage_slot_elems = slot_elems;
  }
  return IS_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of host range [p, p + bytes) when the whole range is
// page-locked host memory mapped for the current device (cudaHostAlloc,
// cudaMallocHost or a mapped registration), else nullptr.  Both ends are
// looked up and must lie in one contiguous mapping.
void* mapped_host_range(void* p, size_t bytes) {
  if (!p || bytes == 0) return nullptr;
  cudaPointerAttributes a{}, b{};
  void* last = static_cast<char*>(p) + (bytes - 1);
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess || cudaPointerGetAttributes(&b, last) != cudaSuccess) {
    cudaGetLastError();  // a failed lookup is not a CUDA error of the call
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost || b.type != cudaMemoryTypeHost || !a.devicePointer || !b.devicePointer)
    return nullptr;
  if (static_cast<char*>(b.devicePointer) != static_cast<char*>(a.devicePointer) + (bytes - 1)) return nullptr;
  return a.devicePointer;
}

// Vector order of the inject kernel for a cache layout: the row index with
// the larger cache stride runs fastest (token-major: slots; head-major:
// heads).
int vec_order_for(int64_t token_stride, int64_t head_stride) { return token_stride > head_stride ? 1 : 0; }

// Vector order of a batch launch.  The fixed-shape per-thread copy loop (D =
// 128, B = 16, H in {4, 8}) walks slot-fastest rows and serves either cache
// layout (B200: on the head-major cache it equals the (slot, head) order of
// the generic loop on the benchmark batch and lifts the small case from
// 0.952 to 0.991 of the copy peak); other shapes take the order whose
// fastest row index has the larger cache stride.
// Copy loop of a batch launch (see pick_fixed): the fixed shapes take the
// paired rotate-half loop (2) on either cache layout; pick_fixed falls back to
// the per-thread loop (1) for the interleaved pairing and for per-slot
// sources.  B200: on the head-major cache the paired loop's CTA writes two
// heads' rows at once (Llama-3.1-8B-shaped batch 0.967 -> 0.990 of the copy
// peak); on the token-major cache it is 0.15% faster on the benchmark batch
// and the Qwen2.5-7B-shaped batch and 0.15% slower on the small case.
int launch_loop(int D, int B, int H) {
#ifndef IS_NO_FIXED_SHAPES
  if (D == 128 && B == 16 && (H == 4 || H == 8)) return 2;
#else
  (void)D; (void)B; (void)H;
#endif
  return 0;
}

int launch_vec_order(int D, int B, int H, int64_t token_stride, int64_t head_stride) {
#ifndef IS_NO_FIXED_SHAPES
  if (D == 128 && B == 16 && (H == 4 || H == 8)) return 1;
#else
  (void)D; (void)B; (void)H;
#endif
  return vec_order_for(token_stride, head_stride);
}

}  // namespace

extern "C" {

const char* is_status_string(int status) {
  switch (status) {
    case IS_OK: return "ok";
    case IS_ERR_INVALID_ARG: return "invalid argument";
    case IS_ERR_BAD_FACT_ID: return "fact id outside the store";
    case IS_ERR_POSITION: return "segment runs past the request's block table";
    case IS_ERR_BAD_BLOCK: return "block-table entry outside the cache";
    case IS_ERR_CAPACITY: return "capacity exceeded";
    case IS_ERR_OOM: return "allocation failed";
    case IS_ERR_CUDA: return "CUDA runtime error";
    case IS_ERR_TIMEOUT: return "timed out";
    case IS_ERR_NOT_SUPPORTED: return "not supported";
    default: return "unknown status";
  }
}

int is_store_create(const is_store_config_t* cfg, int device, is_store_t** out) {
  if (!cfg || !out) return IS_ERR_INVALID_ARG;
  *out = nullptr;
  const is_store_config_t& c = *cfg;
  if (c.num_layers < 1 || c.num_kv_heads < 1 || c.head_dim < 2 || c.head_dim % 2) return IS_ERR_INVALID_ARG;
  if (!(c.rope_theta > 0.0) || (c.rope_style != IS_ROPE_ROTATE_HALF && c.rope_style != IS_ROPE_INTERLEAVED))
    return IS_ERR_INVALID_ARG;
  if (c.rope_scaling != IS_SCALING_NONE && c.rope_scaling != IS_SCALING_LLAMA3) return IS_ERR_INVALID_ARG;
  if (c.rope_scaling == IS_SCALING_LLAMA3 &&
      (!(c.scale_factor > 0.0) || !(c.low_freq_factor > 0.0) || !(c.high_freq_factor > c.low_freq_factor) ||
       c.original_max_position <= 0))
    return IS_ERR_INVALID_ARG;
  if (c.capacity_tokens < 1 || c.max_facts < 1 || c.max_batch_requests < 0 || c.max_batch_fact_ids < 0 ||
      c.max_batch_blocks < 0)
    return IS_ERR_INVALID_ARG;
  if (c.tier != IS_TIER_DEVICE && c.tier != IS_TIER_HOST) return IS_ERR_INVALID_ARG;
  if (!head_dim_supported(c.head_dim)) return IS_ERR_NOT_SUPPORTED;
  if (c.tier == IS_TIER_HOST && c.hot_capacity_tokens < 0) return IS_ERR_INVALID_ARG;
  if (c.capacity_tokens > (int64_t(1) << 31) - 1) return IS_ERR_NOT_SUPPORTED;

  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) return IS_ERR_CUDA;
  DeviceGuard guard(device);

  is_store* s = new (std::nothrow) is_store();
  if (!s) return IS_ERR_OOM;
  s->cfg = c;
  s->device = device;
  cudaDeviceGetAttribute(&s->sm_count, cudaDevAttrMultiProcessorCount, device);
  s->max_req = c.max_batch_requests ? c.max_batch_requests : kDefaultMaxRequests;
  s->max_ids = c.max_batch_fact_ids ? c.max_batch_fact_ids : kDefaultMaxFactIds;
  s->max_blocks = c.max_batch_blocks ? c.max_batch_blocks
                                     : int32_t(std::max<int64_t>(65536, int64_t(256) * s->max_req));

  const size_t plane_elems = size_t(c.capacity_tokens) * size_t(c.head_dim);
  const size_t arena_elems = size_t(c.num_layers) * size_t(c.num_kv_heads) * plane_elems;
  bool ok = true;
  if (c.tier == IS_TIER_HOST) {
    // Pinned, device-mapped host arenas; reads cross the host link.
    s->host_arena = true;
    const size_t bytes = arena_elems * sizeof(uint16_t);
    ok = cudaHostAlloc(reinterpret_cast<void**>(&s->k), bytes, cudaHostAllocMapped | cudaHostAllocPortable) ==
             cudaSuccess &&
         cudaHostAlloc(reinterpret_cast<void**>(&s->v), bytes, cudaHostAllocMapped | cudaHostAllocPortable) ==
             cudaSuccess &&
         cudaHostGetDevicePointer(reinterpret_cast<void**>(&s->k_view), s->k, 0) == cudaSuccess &&
         cudaHostGetDevicePointer(reinterpret_cast<void**>(&s->v_view), s->v, 0) == cudaSuccess;
    s->hot_cap = c.hot_capacity_tokens;
    const size_t hot_elems = size_t(c.num_layers) * size_t(c.num_kv_heads) * size_t(s->hot_cap) * size_t(c.head_dim);
    ok = ok && (s->hot_cap == 0 ||
                (dalloc(&s->k_hot, hot_elems) == cudaSuccess && dalloc(&s->v_hot, hot_elems) == cudaSuccess));
    ok = ok && dalloc(&s->d_hot, size_t(c.max_facts)) == cudaSuccess &&
         cudaMemset(s->d_hot, 0xFF, sizeof(int64_t) * size_t(c.max_facts)) == cudaSuccess &&
         dalloc(&s->d_pend, size_t(c.max_facts)) == cudaSuccess &&
         cudaMemset(s->d_pend, 0xFF, sizeof(int64_t) * size_t(c.max_facts)) == cudaSuccess;
    if (ok) s->h_hot.assign(size_t(c.max_facts), -1);
  } else {
    ok = dalloc(&s->k, arena_elems) == cudaSuccess && dalloc(&s->v, arena_elems) == cudaSuccess;
    s->k_view = s->k;
    s->v_view = s->v;
  }
  ok = ok && dalloc(&s->d_off, size_t(c.max_facts)) == cudaSuccess &&
            dalloc(&s->d_len, size_t(c.max_facts)) == cudaSuccess &&
            dalloc(&s->d_inv_freq, size_t(c.head_dim / 2)) == cudaSuccess &&
            dalloc(&s->ws_seg, size_t(s->max_ids)) == cudaSuccess &&
            dalloc(&s->ws_nblk, size_t(s->max_req)) == cudaSuccess &&
            dalloc(&s->ws_blk0, size_t(s->max_req) + 1) == cudaSuccess &&
            dalloc(&s->ws_tok0, size_t(s->max_req) + 1) == cudaSuccess &&
            dalloc(&s->ws_len, size_t(s->max_req)) == cudaSuccess &&
            dalloc(&s->ws_err, size_t(s->max_req)) == cudaSuccess &&
            dalloc(&s->ws_desc, size_t(s->max_blocks)) == cudaSuccess &&
            dalloc(&s->ws_hdr, 1) == cudaSuccess && dalloc(&s->d_status, 1) == cudaSuccess &&
            dalloc(&s->d_small_ctr, 1) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    free_store(s);
    return IS_ERR_OOM;
  }
  s->h_off.assign(size_t(c.max_facts), 0);
  s->h_len.assign(size_t(c.max_facts), 0);
  cudaMemset(s->d_len, 0, sizeof(int32_t) * size_t(c.max_facts));
  cudaMemset(s->d_off, 0, sizeof(int64_t) * size_t(c.max_facts));
  cudaMemset(s->d_status, 0, sizeof(isk::DevStatus));
  cudaMemset(s->ws_hdr, 0, sizeof(isk::PlanHeader));
  cudaMemset(s->d_small_ctr, 0, sizeof(unsigned int));
  const int nf = c.head_dim / 2;
  isk::inv_freq_kernel<<<(nf + 127) / 128, 128>>>(
      s->d_inv_freq, c.head_dim, c.rope_theta, c.rope_scaling, c.scale_factor, c.low_freq_factor,
      c.high_freq_factor, double(c.original_max_position));

  // Persistent inject grid: resident CTAs per SM x SMs, for the largest
  // cos/sin table (B = 128) so one grid size serves every block size.
  const size_t smem_max = cs_smem_bytes(c.head_dim, isk::kMaxBlockSize);
  void* variants[8] = {pick_inject_t<true>(c.head_dim, c.rope_style), pick_inject_t<false>(c.head_dim, c.rope_style),
                       pick_inject_t<true, true>(c.head_dim, c.rope_style),
                       pick_inject_t<false, true>(c.head_dim, c.rope_style),
                       pick_small_t<true>(c.head_dim, c.rope_style), pick_small_t<false>(c.head_dim, c.rope_style),
                       pick_small_t<true, true>(c.head_dim, c.rope_style),
                       pick_small_t<false, true>(c.head_dim, c.rope_style)};
  for (void* f : variants) cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_max));
  cudaFuncSetAttribute(reinterpret_cast<void*>(&isk::plan_kernel<kPlanThreads, true>),
                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                       int(isk::plan_smem_bytes(isk::kPlanSmemRequests, isk::kPlanSmemIds)));
  for (int h : {4, 8})
    for (int loop : {0, 1, 2})
      for (void* f : {pick_fixed<false, false>(c.head_dim, c.rope_style, h, 16, loop),
                      pick_fixed<false, true>(c.head_dim, c.rope_style, h, 16, loop),
                      pick_fixed<true, false>(c.head_dim, c.rope_style, h, 16, loop),
                      pick_fixed<true, true>(c.head_dim, c.rope_style, h, 16, loop)})
        if (f) cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_max));
  void* fn = pick_inject_t<true>(c.head_dim, c.rope_style);
  int per_sm = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kInjectThreads, cs_smem_bytes(c.head_dim, 16));
  s->inject_grid = std::max(1, per_sm) * s->sm_count;
  int per_sm_small = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm_small, pick_small_t<true>(c.head_dim, c.rope_style),
                                                kInjectThreads, cs_smem_bytes(c.head_dim, 16));
  s->small_grid = std::max(1, per_sm_small) * s->sm_count;
  if (cudaDeviceSynchronize() != cudaSuccess || cudaGetLastError() != cudaSuccess) {
    free_store(s);
    return IS_ERR_CUDA;
  }
  *out = s;
  return IS_OK;
}

void is_store_destroy(is_store_t* s) {
  if (!s) return;
  DeviceGuard guard(s->device);
  cudaDeviceSynchronize();
  free_store(s);
}

int is_store_put_fact_window(is_store_t* s, const void* k_pre, const void* v, int32_t window_len,
                             int32_t len, int32_t* fact_id_out) {
  if (!s || !k_pre || !v || len <= 0 || window_len < 0) return IS_ERR_INVALID_ARG;
  if (s->num_facts >= s->cfg.max_facts || s->used_tokens + len > s->cfg.capacity_tokens)
    return IS_ERR_CAPACITY;
  DeviceGuard guard(s->device);
  const is_store_config_t& c = s->cfg;
  const size_t row = size_t(c.head_dim) * sizeof(uint16_t);
  const size_t width = size_t(len) * row;                          // one fact run of one plane
  const size_t spitch = size_t(window_len + len) * row;            // caller's plane stride
  const size_t dpitch = size_t(c.capacity_tokens) * row;           // store's plane stride
  const size_t height = size_t(c.num_layers) * size_t(c.num_kv_heads);
  const size_t off_bytes = size_t(s->used_tokens) * row;
  const size_t skip = size_t(window_len) * row;                    // the window's rows
  char* kd = reinterpret_cast<char*>(s->k) + off_bytes;
  char* vd = reinterpret_cast<char*>(s->v) + off_bytes;
  const int32_t id = s->num_facts;
  const int64_t off = s->used_tokens;
  if (cudaMemcpy2D(kd, dpitch, static_cast<const char*>(k_pre) + skip, spitch, width, height,
                   cudaMemcpyDefault) != cudaSuccess ||
      cudaMemcpy2D(vd, dpitch, static_cast<const char*>(v) + skip, spitch, width, height,
                   cudaMemcpyDefault) != cudaSuccess ||
      cudaMemcpy(s->d_off + id, &off, sizeof(off), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(s->d_len + id, &len, sizeof(len), cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaGetLastError();
    return IS_ERR_CUDA;
  }
  s->h_off[size_t(id)] = off;
  s->h_len[size_t(id)] = len;
  s->max_len = std::max(s->max_len, len);
  s->num_facts = id + 1;
  s->used_tokens = off + len;
  if (fact_id_out) *fact_id_out = id;
  return IS_OK;
}

int is_store_put_fact(is_store_t* s, const void* k_pre, const void* v, int32_t len,
                      int32_t* fact_id_out) {
  return is_store_put_fact_window(s, k_pre, v, 0, len, fact_id_out);
}

int is_store_num_facts(const is_store_t* s, int32_t* out) {
  if (!s || !out) return IS_ERR_INVALID_ARG;
  *out = s->num_facts;
  return IS_OK;
}

int is_store_fact_info(const is_store_t* s, int32_t id, int64_t* off, int32_t* len) {
  if (!s) return IS_ERR_INVALID_ARG;
  if (id < 0 || id >= s->num_facts) return IS_ERR_BAD_FACT_ID;
  if (off) *off = s->h_off[size_t(id)];
  if (len) *len = s->h_len[size_t(id)];
  return IS_OK;
}

int is_store_read_fact(is_store_t* s, int32_t id, void* k_out, void* v_out) {
  if (!s || (!k_out && !v_out)) return IS_ERR_INVALID_ARG;
  if (id < 0 || id >= s->num_facts) return IS_ERR_BAD_FACT_ID;
  DeviceGuard guard(s->device);
  const is_store_config_t& c = s->cfg;
  const size_t row = size_t(c.head_dim) * sizeof(uint16_t);
  const size_t width = size_t(s->h_len[size_t(id)]) * row;
  const size_t spitch = size_t(c.capacity_tokens) * row;
  const size_t height = size_t(c.num_layers) * size_t(c.num_kv_heads);
  const size_t off_bytes = size_t(s->h_off[size_t(id)]) * row;
  if (k_out && cudaMemcpy2D(k_out, width, reinterpret_cast<char*>(s->k) + off_bytes, spitch, width,
                            height, cudaMemcpyDefault) != cudaSuccess)
    return IS_ERR_CUDA;
  if (v_out && cudaMemcpy2D(v_out, width, reinterpret_cast<char*>(s->v) + off_bytes, spitch, width,
                            height, cudaMemcpyDefault) != cudaSuccess)
    return IS_ERR_CUDA;
  return IS_OK;
}

int is_store_arena(const is_store_t* s, void** k, void** v, int64_t* plane_tokens) {
  if (!s) return IS_ERR_INVALID_ARG;
  if (k) *k = s->k_view;
  if (v) *v = s->v_view;
  if (plane_tokens) *plane_tokens = s->cfg.capacity_tokens;
  return IS_OK;
}

int is_store_attach_shards(is_store_t* s, int32_t n, const void* const* k_arenas, const void* const* v_arenas,
                           const int64_t* plane_tokens, int32_t nf, const int32_t* fact_shard,
                           const int64_t* fact_offset, const int32_t* fact_len) {
  if (!s || n < 1 || nf < 1 || !k_arenas || !v_arenas || !plane_tokens || !fact_shard || !fact_offset ||
      !fact_len)
    return IS_ERR_INVALID_ARG;
  if (s->host_arena) return IS_ERR_NOT_SUPPORTED;
  for (int32_t i = 0; i < n; ++i)
    if (!k_arenas[i] || !v_arenas[i] || !aligned16(k_arenas[i]) || !aligned16(v_arenas[i]) ||
        plane_tokens[i] < 1 || plane_tokens[i] > (int64_t(1) << 31) - 1)
      return IS_ERR_INVALID_ARG;
  for (int32_t g = 0; g < nf; ++g) {
    const int32_t sh = fact_shard[g];
    if (sh < 0 || sh >= n || fact_offset[g] < 0 || fact_len[g] < 1 ||
        fact_offset[g] + fact_len[g] > plane_tokens[sh])
      return IS_ERR_INVALID_ARG;
  }
  DeviceGuard guard(s->device);
  if (cudaDeviceSynchronize() != cudaSuccess) return IS_ERR_CUDA;
  const int64_t D = s->cfg.head_dim;
  std::vector<const uint16_t*> hk(static_cast<size_t>(n)), hv(static_cast<size_t>(n));
  std::vector<int64_t> hp(static_cast<size_t>(n));
  for (int32_t i = 0; i < n; ++i) {
    hk[size_t(i)] = static_cast<const uint16_t*>(k_arenas[i]);
    hv[size_t(i)] = static_cast<const uint16_t*>(v_arenas[i]);
    hp[size_t(i)] = plane_tokens[i] * D;
  }
  ShardView nv;
  if (dalloc(&nv.k, size_t(n)) != cudaSuccess || dalloc(&nv.v, size_t(n)) != cudaSuccess ||
      dalloc(&nv.plane, size_t(n)) != cudaSuccess || dalloc(&nv.of, size_t(nf)) != cudaSuccess ||
      dalloc(&nv.off, size_t(nf)) != cudaSuccess || dalloc(&nv.len, size_t(nf)) != cudaSuccess) {
    cudaGetLastError();
    nv.release();
    return IS_ERR_OOM;
  }
  if (cudaMemcpy(nv.k, hk.data(), sizeof(void*) * size_t(n), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(nv.v, hv.data(), sizeof(void*) * size_t(n), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(nv.plane, hp.data(), sizeof(int64_t) * size_t(n), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(nv.of, fact_shard, sizeof(int32_t) * size_t(nf), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(nv.off, fact_offset, sizeof(int64_t) * size_t(nf), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(nv.len, fact_len, sizeof(int32_t) * size_t(nf), cudaMemcpyHostToDevice) != cudaSuccess) {
    nv.release();
    return IS_ERR_CUDA;
  }
  free_view(s);
  s->d_shard_k = nv.k;
  s->d_shard_v = nv.v;
  s->d_shard_plane = nv.plane;
  s->d_shard_of = nv.of;
  s->d_shard_off = nv.off;
  s->d_shard_len = nv.len;
  s->shard_n = n;
  s->shard_facts = nf;
  s->shard_max_len = *std::max_element(fact_len, fact_len + nf);
  return IS_OK;
}

int is_store_detach_shards(is_store_t* s) {
  if (!s) return IS_ERR_INVALID_ARG;
  if (s->shard_n == 0) return IS_OK;
  DeviceGuard guard(s->device);
  if (cudaDeviceSynchronize() != cudaSuccess) return IS_ERR_CUDA;
  free_view(s);
  return IS_OK;
}

int is_store_shard_info(const is_store_t* s, int32_t* num_shards, int32_t* num_global_facts) {
  if (!s) return IS_ERR_INVALID_ARG;
  if (num_shards) *num_shards = s->shard_n;
  if (num_global_facts) *num_global_facts = s->shard_facts;
  return IS_OK;
}

static_assert(sizeof(cudaIpcMemHandle_t) == sizeof(is_ipc_handle_t), "IPC handle size");

int is_store_export(const is_store_t* s, is_ipc_handle_t* k_handle, is_ipc_handle_t* v_handle,
                    int64_t* plane_tokens) {
  if (!s || !k_handle || !v_handle) return IS_ERR_INVALID_ARG;
  if (s->host_arena) return IS_ERR_NOT_SUPPORTED;
  DeviceGuard guard(s->device);
  cudaIpcMemHandle_t hk, hv;
  if (cudaIpcGetMemHandle(&hk, s->k) != cudaSuccess || cudaIpcGetMemHandle(&hv, s->v) != cudaSuccess) {
    cudaGetLastError();
    return IS_ERR_CUDA;
  }
  std::memcpy(k_handle->bytes, &hk, sizeof(hk));
  std::memcpy(v_handle->bytes, &hv, sizeof(hv));
  if (plane_tokens) *plane_tokens = s->cfg.capacity_tokens;
  return IS_OK;
}

int is_ipc_open(int device, const is_ipc_handle_t* handle, void** ptr) {
  if (!handle || !ptr) return IS_ERR_INVALID_ARG;
  *ptr = nullptr;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) return IS_ERR_INVALID_ARG;
  DeviceGuard guard(device);
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle->bytes, sizeof(h));
  if (cudaIpcOpenMemHandle(ptr, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    cudaGetLastError();
    *ptr = nullptr;
    return IS_ERR_CUDA;
  }
  return IS_OK;
}

int is_ipc_close(int device, void* ptr) {
  if (!ptr) return IS_ERR_INVALID_ARG;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) return IS_ERR_INVALID_ARG;
  DeviceGuard guard(device);
  if (cudaIpcCloseMemHandle(ptr) != cudaSuccess) {
    cudaGetLastError();
    return IS_ERR_CUDA;
  }
  return IS_OK;
}

int is_store_set_hot(is_store_t* s, const int32_t* fact_ids, int32_t n) {
  if (!s || n < 0 || (n > 0 && !fact_ids)) return IS_ERR_INVALID_ARG;
  if (!s->host_arena || s->hot_policy != IS_HOT_STATIC) return IS_ERR_NOT_SUPPORTED;
  std::vector<int64_t> hot(size_t(s->cfg.max_facts), -1);
  int64_t used = 0;
  int32_t count = 0;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t f = fact_ids[i];
    if (f < 0 || f >= s->num_facts) return IS_ERR_BAD_FACT_ID;
    if (hot[size_t(f)] >= 0) continue;  // listed twice
    if (used + s->h_len[size_t(f)] > s->hot_cap) return IS_ERR_CAPACITY;
    hot[size_t(f)] = used;
    used += s->h_len[size_t(f)];
    ++count;
  }
  DeviceGuard guard(s->device);
  if (cudaDeviceSynchronize() != cudaSuccess) return IS_ERR_CUDA;  // no batch may read the old set
  const is_store_config_t& c = s->cfg;
  const size_t row = size_t(c.head_dim) * sizeof(uint16_t);
  const size_t height = size_t(c.num_layers) * size_t(c.num_kv_heads);
  for (int32_t f = 0; f < s->num_facts; ++f) {
    if (hot[size_t(f)] < 0) continue;
    const size_t width = size_t(s->h_len[size_t(f)]) * row;
    const size_t src_off = size_t(s->h_off[size_t(f)]) * row, dst_off = size_t(hot[size_t(f)]) * row;
    if (cudaMemcpy2D(reinterpret_cast<char*>(s->k_hot) + dst_off, size_t(s->hot_cap) * row,
                     reinterpret_cast<const char*>(s->k) + src_off, size_t(c.capacity_tokens) * row, width,
                     height, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy2D(reinterpret_cast<char*>(s->v_hot) + dst_off, size_t(s->hot_cap) * row,
                     reinterpret_cast<const char*>(s->v) + src_off, size_t(c.capacity_tokens) * row, width,
                     height, cudaMemcpyHostToDevice) != cudaSuccess)
      return IS_ERR_CUDA;
  }
  if (cudaMemcpy(s->d_hot, hot.data(), sizeof(int64_t) * hot.size(), cudaMemcpyHostToDevice) != cudaSuccess)
    return IS_ERR_CUDA;
  s->h_hot.swap(hot);
  s->hot_used = used;
  s->hot_facts = count;
  return IS_OK;
}

int is_store_set_hot_policy(is_store_t* s, int policy, int32_t slot_tokens) {
  if (!s || (policy != IS_HOT_STATIC && policy != IS_HOT_LRU)) return IS_ERR_INVALID_ARG;
  if (!s->host_arena) return IS_ERR_NOT_SUPPORTED;
  if (policy == IS_HOT_LRU && (slot_tokens < 1 || slot_tokens > s->hot_cap)) return IS_ERR_INVALID_ARG;
  DeviceGuard guard(s->device);
  if (cudaDeviceSynchronize() != cudaSuccess) return IS_ERR_CUDA;  // no batch may read the old set
  // every fact cold
  if (cudaMemset(s->d_hot, 0xFF, sizeof(int64_t) * size_t(s->cfg.max_facts)) != cudaSuccess ||
      cudaMemset(s->d_pend, 0xFF, sizeof(int64_t) * size_t(s->cfg.max_facts)) != cudaSuccess)
    return IS_ERR_CUDA;
  std::fill(s->h_hot.begin(), s->h_hot.end(), int64_t(-1));
  s->hot_used = 0;
  s->hot_facts = 0;
  s->hot_policy = policy;
  s->slot_tokens = policy == IS_HOT_LRU ? slot_tokens : 0;
  const size_t nslots = policy == IS_HOT_LRU ? size_t(s->hot_cap / slot_tokens) : 0;
  s->slot_owner.assign(nslots, -1);
  s->slot_tick.assign(nslots, 0);
  s->lru.clear();
  s->lru_at.assign(nslots, s->lru.end());
  for (size_t i = 0; i < nslots; ++i) s->lru_at[i] = s->lru.insert(s->lru.end(), int32_t(i));
  s->fact_tick.assign(size_t(s->cfg.max_facts), 0);
  s->tick = 0;
  s->batch_tick = 0;
  s->pf_pending = false;  // the device is idle: any prefetch has landed
  s->lru_hits = s->lru_misses = s->lru_promoted = s->lru_promoted_tokens = 0;
  if (!s->touch_done && cudaEventCreateWithFlags(&s->touch_done, cudaEventDisableTiming) != cudaSuccess)
    return IS_ERR_CUDA;
  return IS_OK;
}

// LRU promotion of the listed facts: hits move to the front; misses that fit
// a slot take the least recently used slot not used by this call.
//   fused == false: the data moves on `stream` now (promote_kernel reads the
//     mapped host arenas), then the hot table is patched; later work on the
//     stream sees the new set.
//   fused == true (a batch of these ids follows on `stream`): evicted facts
//     leave the hot table now and the promoted ones are marked pending, so
//     the batch reads them from host memory and, as it goes, also writes
//     their rows into their HBM slots -- each row crosses the host link once
//     and no copy runs ahead of the batch; lru_finish then enters them in
//     the hot table.
// The LRU decisions for one list of ids (host only): hits move to the front
// of the list; misses that fit a slot take the least recently used slot,
// unless that slot was used at or after tick `protect` (this call, and a
// batch that may still be running).  Fills the evicted facts, the
// (fact, hot token) promotions and their copy descriptors.
static void lru_plan(is_store* s, const int32_t* fact_ids, int32_t n, uint64_t tick, uint64_t protect,
                     bool count_use, std::vector<int64_t>& evict, std::vector<int64_t>& prom,
                     std::vector<isk::Promotion>& promo) {
  for (int32_t i = 0; i < n; ++i) {
    const int32_t f = fact_ids[i];
    if (f < 0 || f >= s->num_facts) continue;  // the batch itself reports it
    if (s->fact_tick[size_t(f)] == tick) continue;  // listed twice in this call
    s->fact_tick[size_t(f)] = tick;
    const int64_t ho = s->h_hot[size_t(f)];
    if (ho >= 0) {
      const int32_t slot = int32_t(ho / s->slot_tokens);
      s->lru.splice(s->lru.begin(), s->lru, s->lru_at[size_t(slot)]);
      s->slot_tick[size_t(slot)] = tick;
      if (count_use) ++s->lru_hits;
      continue;
    }
    if (count_use) ++s->lru_misses;
    if (s->lru.empty() || s->h_len[size_t(f)] > s->slot_tokens) continue;  // served from host
    const int32_t slot = s->lru.back();
    if (s->slot_tick[size_t(slot)] >= protect) continue;  // every slot is in use
    const int32_t old = s->slot_owner[size_t(slot)];
    if (old >= 0) {
      s->h_hot[size_t(old)] = -1;
      evict.push_back(old);
    } else {
      ++s->hot_facts;
    }
    const int64_t dst = int64_t(slot) * s->slot_tokens;
    s->slot_owner[size_t(slot)] = f;
    s->slot_tick[size_t(slot)] = tick;
    s->h_hot[size_t(f)] = dst;
    s->lru.splice(s->lru.begin(), s->lru, s->lru_at[size_t(slot)]);
    prom.push_back(f);
    prom.push_back(dst);
    promo.push_back(isk::Promotion{s->h_off[size_t(f)], dst, s->h_len[size_t(f)], 0});
    s->lru_promoted_tokens += s->h_len[size_t(f)];
  }
  s->lru_promoted += int64_t(promo.size());
  s->hot_used = int64_t(s->hot_facts) * s->slot_tokens;
}

static int lru_touch(is_store* s, const int32_t* fact_ids, int32_t n, cudaStream_t st, bool fused,
                     int32_t* promoted_out) {
  // The staging of the previous touch must have been consumed, and a
  // prefetch's transfers must have landed before its slots are reconsidered.
  if (cudaEventSynchronize(s->touch_done) != cudaSuccess) return IS_ERR_CUDA;
  if (s->pf_pending && cudaEventSynchronize(s->pf_done) != cudaSuccess) return IS_ERR_CUDA;
  const uint64_t tick = ++s->tick;
  std::vector<isk::Promotion> promo;
  std::vector<int64_t> evict, prom;  // evicted facts; (fact, hot token) promoted
  lru_plan(s, fact_ids, n, tick, tick, true, evict, prom, promo);
  if (promoted_out) *promoted_out = int32_t(promo.size());
  s->pend_ne = s->pend_np = 0;
  if (promo.empty()) return IS_OK;
  // Pair lists (fact, value) for the table kernel: evictions (fact, -1),
  // then the promotions as (fact, hot token); fused adds the promotions
  // again (for the hot table after the batch) and as (fact, -1) (to clear
  // their pending mark).
  const size_t ne = evict.size(), np = promo.size();
  std::vector<int64_t> pairs;
  for (int64_t f : evict) { pairs.push_back(f); pairs.push_back(-1); }
  pairs.insert(pairs.end(), prom.begin(), prom.end());
  if (fused) {
    pairs.insert(pairs.end(), prom.begin(), prom.end());
    for (size_t i = 0; i < np; ++i) { pairs.push_back(prom[2 * i]); pairs.push_back(-1); }
  }
  const size_t nq = pairs.size() / 2;
  if (np > s->promo_cap || nq > 2 * s->promo_cap) {
    const size_t cap = std::max(np, nq) * 2;
    cudaFreeHost(s->h_promo);
    cudaFreeHost(s->h_pairs);
    cudaFree(s->d_promo);
    cudaFree(s->d_pairs);
    s->h_promo = nullptr;
    s->h_pairs = nullptr;
    s->d_promo = nullptr;
    s->d_pairs = nullptr;
    s->promo_cap = 0;
    if (cudaHostAlloc(reinterpret_cast<void**>(&s->h_promo), cap * sizeof(isk::Promotion), 0) != cudaSuccess ||
        cudaHostAlloc(reinterpret_cast<void**>(&s->h_pairs), cap * 4 * sizeof(int64_t), 0) != cudaSuccess ||
        dalloc(&s->d_promo, cap) != cudaSuccess || dalloc(&s->d_pairs, cap * 4) != cudaSuccess)
      return IS_ERR_OOM;
    s->promo_cap = cap;
  }
  std::memcpy(s->h_promo, promo.data(), np * sizeof(isk::Promotion));
  std::memcpy(s->h_pairs, pairs.data(), pairs.size() * sizeof(int64_t));
  if (cudaMemcpyAsync(s->d_promo, s->h_promo, np * sizeof(isk::Promotion), cudaMemcpyHostToDevice, st) !=
          cudaSuccess ||
      cudaMemcpyAsync(s->d_pairs, s->h_pairs, pairs.size() * sizeof(int64_t), cudaMemcpyHostToDevice, st) !=
          cudaSuccess)
    return IS_ERR_CUDA;
  if (fused) {
    isk::hot_table_kernel<<<unsigned((ne + np + 255) / 256), 256, 0, st>>>(s->d_hot, s->d_pend, s->d_pairs,
                                                                          int32_t(ne), int32_t(np));
    s->pend_ne = ne;
    s->pend_np = np;
    return cudaGetLastError() == cudaSuccess ? IS_OK : IS_ERR_CUDA;
  }
  const is_store_config_t& c = s->cfg;
  const int vpr = c.head_dim / 8;
  dim3 grid(unsigned(std::max(1, s->sm_count / 2)), unsigned(std::min<size_t>(np, 65535)));
  isk::promote_kernel<<<grid, 256, 0, st>>>(s->d_promo, int32_t(np), c.num_layers * c.num_kv_heads, vpr,
                                             s->k_view, s->v_view, int64_t(c.capacity_tokens) * c.head_dim,
                                             s->k_hot, s->v_hot, s->hot_cap * c.head_dim);
  isk::hot_table_kernel<<<unsigned((nq + 255) / 256), 256, 0, st>>>(s->d_hot, s->d_hot, s->d_pairs,
                                                                    int32_t(nq), 0);
  if (cudaEventRecord(s->touch_done, st) != cudaSuccess || cudaGetLastError() != cudaSuccess) return IS_ERR_CUDA;
  return IS_OK;
}

// After the batch of a fused touch: the pending promotions enter the hot
// table.  A batch that did not run clean (an error skipped requests or
// blocks, so some rows may not have been written to the slots) first copies
// the promoted facts whole, as an unfused touch does.
static int lru_finish(is_store* s, cudaStream_t st, bool batch_ok) {
  if (s->pend_np == 0) return IS_OK;
  const size_t ne = s->pend_ne, np = s->pend_np;
  s->pend_ne = s->pend_np = 0;
  const is_store_config_t& c = s->cfg;
  if (!batch_ok) {
    dim3 grid(unsigned(std::max(1, s->sm_count / 2)), unsigned(std::min<size_t>(np, 65535)));
    isk::promote_kernel<<<grid, 256, 0, st>>>(s->d_promo, int32_t(np), c.num_layers * c.num_kv_heads,
                                               c.head_dim / 8, s->k_view, s->v_view,
                                               int64_t(c.capacity_tokens) * c.head_dim, s->k_hot, s->v_hot,
                                               s->hot_cap * c.head_dim);
  }
  isk::hot_table_kernel<<<unsigned((2 * np + 255) / 256), 256, 0, st>>>(
      s->d_hot, s->d_pend, s->d_pairs + 2 * (ne + np), int32_t(np), int32_t(np));
  if (cudaEventRecord(s->touch_done, st) != cudaSuccess || cudaGetLastError() != cudaSuccess) return IS_ERR_CUDA;
  return IS_OK;
}

// Prefetch for the next batch (LRU): its cold facts take slots not used by
// the batch just launched (tick s->batch_tick or later) and are copied into
// HBM on the store's copy stream while that batch runs, by promote_kernel
// (the SMs' reads of the mapped host arenas: on B200 they keep ~0.91 of a
// large copy-engine transfer's host-link rate, where one copy-engine transfer
// per fact, ~1 MB each, keeps ~0.78); then the hot table learns them.  The
// next batch on the store waits for pf_done.
static int lru_prefetch(is_store* s, const int32_t* fact_ids, int32_t n) {
  if (!s->copy_stream &&
      cudaStreamCreateWithFlags(&s->copy_stream, cudaStreamNonBlocking) != cudaSuccess)
    return IS_ERR_CUDA;
  if (!s->pf_done && cudaEventCreateWithFlags(&s->pf_done, cudaEventDisableTiming) != cudaSuccess)
    return IS_ERR_CUDA;
  // the previous prefetch's lists must have been consumed
  if (s->pf_pending && cudaEventSynchronize(s->pf_done) != cudaSuccess) return IS_ERR_CUDA;
  const uint64_t tick = ++s->tick;
  std::vector<isk::Promotion> promo;
  std::vector<int64_t> evict, prom;
  lru_plan(s, fact_ids, n, tick, s->batch_tick, false, evict, prom, promo);
  if (promo.empty()) return IS_OK;
  std::vector<int64_t> pairs;
  for (int64_t f : evict) { pairs.push_back(f); pairs.push_back(-1); }
  pairs.insert(pairs.end(), prom.begin(), prom.end());
  const size_t nq = pairs.size() / 2, np = promo.size();
  if (nq > s->pf_cap) {
    cudaFreeHost(s->h_pf_pairs);
    cudaFree(s->d_pf_pairs);
    cudaFreeHost(s->h_pf_promo);
    cudaFree(s->d_pf_promo);
    s->h_pf_pairs = nullptr;
    s->d_pf_pairs = nullptr;
    s->h_pf_promo = nullptr;
    s->d_pf_promo = nullptr;
    s->pf_cap = 0;
    const size_t cap = nq * 2;
    if (cudaHostAlloc(reinterpret_cast<void**>(&s->h_pf_pairs), cap * 2 * sizeof(int64_t), 0) != cudaSuccess ||
        dalloc(&s->d_pf_pairs, cap * 2) != cudaSuccess ||
        cudaHostAlloc(reinterpret_cast<void**>(&s->h_pf_promo), cap * sizeof(isk::Promotion), 0) != cudaSuccess ||
        dalloc(&s->d_pf_promo, cap) != cudaSuccess)
      return IS_ERR_OOM;
    s->pf_cap = cap;
  }
  std::memcpy(s->h_pf_pairs, pairs.data(), pairs.size() * sizeof(int64_t));
  std::memcpy(s->h_pf_promo, promo.data(), np * sizeof(isk::Promotion));
  const is_store_config_t& c = s->cfg;
  cudaStream_t cs = s->copy_stream;
  if (cudaMemcpyAsync(s->d_pf_promo, s->h_pf_promo, np * sizeof(isk::Promotion), cudaMemcpyHostToDevice, cs) !=
          cudaSuccess ||
      cudaMemcpyAsync(s->d_pf_pairs, s->h_pf_pairs, pairs.size() * sizeof(int64_t), cudaMemcpyHostToDevice, cs) !=
          cudaSuccess)
    return IS_ERR_CUDA;
  dim3 grid(unsigned(std::max(1, s->sm_count / 2)), unsigned(std::min<size_t>(np, 65535)));
  isk::promote_kernel<<<grid, 256, 0, cs>>>(s->d_pf_promo, int32_t(np), c.num_layers * c.num_kv_heads,
                                             c.head_dim / 8, s->k_view, s->v_view,
                                             int64_t(c.capacity_tokens) * c.head_dim, s->k_hot, s->v_hot,
                                             s->hot_cap * c.head_dim);
  isk::hot_table_kernel<<<unsigned((nq + 255) / 256), 256, 0, cs>>>(s->d_hot, s->d_hot, s->d_pf_pairs,
                                                                   int32_t(nq), 0);
  if (cudaEventRecord(s->pf_done, cs) != cudaSuccess || cudaGetLastError() != cudaSuccess) return IS_ERR_CUDA;
  s->pf_pending = true;
  return IS_OK;
}

int is_store_touch(is_store_t* s, const int32_t* fact_ids, int32_t n, void* stream, int32_t* promoted_out) {
  if (!s || n < 0 || (n > 0 && !fact_ids)) return IS_ERR_INVALID_ARG;
  if (!s->host_arena || s->hot_policy != IS_HOT_LRU) return IS_ERR_NOT_SUPPORTED;
  DeviceGuard guard(s->device);
  return lru_touch(s, fact_ids, n, static_cast<cudaStream_t>(stream), false, promoted_out);
}

int is_store_lru_stats(const is_store_t* s, int64_t* hits, int64_t* misses, int64_t* promoted,
                       int64_t* promoted_tokens) {
  if (!s) return IS_ERR_INVALID_ARG;
  if (hits) *hits = s->lru_hits;
  if (misses) *misses = s->lru_misses;
  if (promoted) *promoted = s->lru_promoted;
  if (promoted_tokens) *promoted_tokens = s->lru_promoted_tokens;
  return IS_OK;
}

int is_store_tier_info(const is_store_t* s, int32_t* tier, int64_t* hot_capacity, int64_t* hot_used,
                       int32_t* hot_facts) {
  if (!s) return IS_ERR_INVALID_ARG;
  if (tier) *tier = s->host_arena ? IS_TIER_HOST : IS_TIER_DEVICE;
  if (hot_capacity) *hot_capacity = s->hot_cap;
  if (hot_used) *hot_used = s->hot_used;
  if (hot_facts) *hot_facts = s->hot_facts;
  return IS_OK;
}

int is_inject_batch(is_store_t* s, int32_t R, const int32_t* req_off, const int32_t* fact_ids,
                    int32_t num_ids, const int32_t* start_pos, const int32_t* block_tables,
                    int32_t max_blocks_per_req, const is_cache_t* cache, int64_t* slot_out,
                    int64_t slot_cap, void* stream) {
  if (!s || !cache || R < 0 || num_ids < 0 || max_blocks_per_req < 1) return IS_ERR_INVALID_ARG;
  if (R > 0 && (!req_off || !start_pos || !block_tables)) return IS_ERR_INVALID_ARG;
  if (num_ids > 0 && !fact_ids) return IS_ERR_INVALID_ARG;
  if (R == 0 && !req_off) return IS_ERR_INVALID_ARG;
  if (R > s->max_req || num_ids > s->max_ids) return IS_ERR_CAPACITY;
  const is_cache_t& c = *cache;
  if (!c.k_cache || !c.v_cache || c.num_blocks < 1 || c.block_size < 1 ||
      c.block_size > isk::kMaxBlockSize)
    return IS_ERR_INVALID_ARG;
  if (!aligned16(c.k_cache) || !aligned16(c.v_cache) || c.layer_stride % 8 || c.block_stride % 8 ||
      c.token_stride % 8 || c.head_stride % 8 || c.layer_stride < 0 || c.block_stride < 0 ||
      c.token_stride < 0 || c.head_stride < 0)
    return IS_ERR_INVALID_ARG;
  if (slot_out && slot_cap < 0) return IS_ERR_INVALID_ARG;
  if (int64_t(max_blocks_per_req) * c.block_size > (int64_t(1) << 31) - 1) return IS_ERR_NOT_SUPPORTED;
  DeviceGuard guard(s->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const is_store_config_t& cf = s->cfg;
  // a prefetch's transfers and hot-table changes land before this batch reads
  if (s->pf_pending && cudaStreamWaitEvent(st, s->pf_done, 0) != cudaSuccess) return IS_ERR_CUDA;

  isk::PlanArgs pa;
  pa.R = R;
  pa.req_off = req_off;
  pa.fact_ids = fact_ids;
  pa.num_ids = num_ids;
  pa.start_pos = start_pos;
  pa.block_tables = block_tables;
  pa.max_blocks = max_blocks_per_req;
  pa.num_blocks = c.num_blocks;
  pa.B = c.block_size;
  pa.L = cf.num_layers;
  pa.H = cf.num_kv_heads;
  pa.chk_off = nullptr;  // the library's own fact table
  pa.chk_plane = 0;
  // With a sharded view attached, ids are global: the view's fact table.
  const bool view = s->shard_n > 0;
  const int32_t nfacts = view ? s->shard_facts : s->num_facts;
  pa.fact_len = view ? s->d_shard_len : s->d_len;
  pa.num_facts = nfacts;
  pa.slot_out = slot_out;
  pa.slot_cap = slot_cap;
  pa.grid_ctas = s->inject_grid;
  // The per-thread copy loops of the common shapes take any (layer, head)
  // row range as a unit; the generic loop takes whole layers.
  const int loop = launch_loop(cf.head_dim, c.block_size, cf.num_kv_heads);
  pa.row_units = loop != 0;
  pa.max_batch_blocks = s->max_blocks;
  pa.seg = s->ws_seg;
  pa.req_nblk = s->ws_nblk;
  pa.req_blk0 = s->ws_blk0;
  pa.req_tok0 = s->ws_tok0;
  pa.req_len = s->ws_len;
  pa.req_err = s->ws_err;
  pa.desc = s->ws_desc;
  pa.hdr = s->ws_hdr;
  pa.st = s->d_status;
  pa.st_mirror = s->batch_mirror;
  // The single kernel saves the plan launch (and the inject kernel's reads
  // of the plan); its units come from a counter like the inject kernel's.
  // It takes batches of up to small_limit requests and kSmallIds ids whose
  // 32-bit sums cannot wrap (ids x the longest fact below 2^31).
  const int64_t longest = view ? s->shard_max_len : s->max_len;
  const bool small = R <= s->small_limit && num_ids <= isk::kSmallIds &&
                     int64_t(num_ids) * longest <= kSmallSumLimit;
  if (!small) {
    if (R <= isk::kPlanSmemRequests && num_ids <= isk::kPlanSmemIds)
      isk::plan_kernel<kPlanThreads, true><<<1, kPlanThreads, isk::plan_smem_bytes(R, num_ids), st>>>(pa);
    else
      isk::plan_kernel<kPlanThreads, false><<<1, kPlanThreads, 0, st>>>(pa);
  }

  isk::InjectArgs ia{};
  ia.k_store = s->k_view;
  ia.v_store = s->v_view;
  ia.k_hot = s->k_hot;
  ia.v_hot = s->v_hot;
  ia.hot_plane = s->hot_cap * cf.head_dim;
  ia.hot_off = s->d_hot;
  ia.pend = s->batch_pend ? s->d_pend : nullptr;
  ia.k_prom = s->k_hot;
  ia.v_prom = s->v_hot;
  ia.plane = int64_t(cf.capacity_tokens) * cf.head_dim;
  ia.fact_off = view ? s->d_shard_off : s->d_off;
  ia.fact_len = view ? s->d_shard_len : s->d_len;
  ia.shard_k = view ? s->d_shard_k : nullptr;
  ia.shard_v = view ? s->d_shard_v : nullptr;
  ia.shard_plane = s->d_shard_plane;
  ia.fact_shard = s->d_shard_of;
  ia.inv_freq = s->d_inv_freq;
  ia.L = cf.num_layers;
  ia.H = cf.num_kv_heads;
  ia.req_off = req_off;
  ia.fact_ids = fact_ids;
  ia.start_pos = start_pos;
  ia.block_tables = block_tables;
  ia.max_blocks = max_blocks_per_req;
  ia.k_cache = static_cast<uint16_t*>(c.k_cache);
  ia.v_cache = static_cast<uint16_t*>(c.v_cache);
  ia.ls = c.layer_stride;
  ia.bs = c.block_stride;
  ia.ts = c.token_stride;
  ia.hs = c.head_stride;
  ia.num_blocks = c.num_blocks;
  ia.B = c.block_size;
  ia.vec_order = launch_vec_order(cf.head_dim, c.block_size, cf.num_kv_heads, c.token_stride, c.head_stride);
  ia.slot_out = slot_out;
  ia.seg = s->ws_seg;
  ia.req_tok0 = s->ws_tok0;
  ia.desc = s->ws_desc;
  ia.hdr = s->ws_hdr;
  ia.st = s->d_status;
  ia.st_mirror = s->batch_mirror;
  ia.fact_len_count = nfacts;
  // Per-slot sources: the host tier, or the arenas of a sharded view.
  const bool per_slot = s->host_arena || view;
  void* fn = small ? pick_small(cf.head_dim, cf.rope_style, cf.num_kv_heads, c.block_size, per_slot, loop)
                   : pick_inject(cf.head_dim, cf.rope_style, cf.num_kv_heads, c.block_size, per_slot, loop);
  int32_t small_R = R, small_ids = num_ids, small_grid = s->small_grid, small_blocks = s->max_blocks;
  int64_t small_cap = slot_cap;
  unsigned int* small_ctr = s->d_small_ctr;
  void* small_args[] = {&ia, &small_R, &small_ids, &small_cap, &small_grid, &small_blocks, &small_ctr};
  void* args[] = {&ia};
  TimedLaunch* ev = nullptr;
  if (s->timing && s->events_used < size_t(kMaxTimedLaunches)) {
    if (s->events_used == s->events.size()) {
      TimedLaunch e{};
      if (cudaEventCreate(&e.start) == cudaSuccess && cudaEventCreate(&e.stop) == cudaSuccess)
        s->events.push_back(e);
    }
    if (s->events_used < s->events.size()) ev = &s->events[s->events_used++];
  }
  cudaError_t e;
  const size_t smem = cs_smem_bytes(cf.head_dim, c.block_size);
  if (ev) cudaEventRecord(ev->start, st);
  if (small) {
    // One kernel composes and injects the whole small batch.
    e = cudaLaunchKernel(fn, dim3(unsigned(s->small_grid)), dim3(kInjectThreads), small_args, smem, st);
  } else if (ev) {
    // Timed: events bracket the inject kernel alone (no early launch).
    e = cudaLaunchKernel(fn, dim3(unsigned(s->inject_grid)), dim3(kInjectThreads), args, smem, st);
  } else {
    // Programmatic dependent launch: the inject grid becomes resident while
    // the plan kernel runs and starts work when the plan's results are ready.
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(unsigned(s->inject_grid));
    lc.blockDim = dim3(kInjectThreads);
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    e = cudaLaunchKernelExC(&lc, fn, args);
  }
  if (ev) cudaEventRecord(ev->stop, st);
  if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) return IS_ERR_CUDA;
  return IS_OK;
}

static int host_batch(is_store_t* s, int32_t R, const int32_t* req_off, const int32_t* fact_ids,
                      int32_t num_ids, const int32_t* start_pos, const int32_t* block_tables,
                      int32_t max_blocks_per_req, const is_cache_t* cache, int64_t* slot_out,
                      int64_t slot_cap, const int32_t* next_ids, int32_t num_next, void* stream) {
  if (!s || !cache || R < 0 || num_ids < 0 || max_blocks_per_req < 1 || !req_off) return IS_ERR_INVALID_ARG;
  if ((R > 0 && (!start_pos || !block_tables)) || (num_ids > 0 && !fact_ids)) return IS_ERR_INVALID_ARG;
  if (num_next < 0 || (num_next > 0 && !next_ids)) return IS_ERR_INVALID_ARG;
  if (R > s->max_req || num_ids > s->max_ids) return IS_ERR_CAPACITY;
  if (slot_out && slot_cap < 0) return IS_ERR_INVALID_ARG;
  DeviceGuard guard(s->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n_off = size_t(R) + 1, n_ids = size_t(num_ids), n_sp = size_t(R);
  const size_t n_bt = size_t(R) * size_t(max_blocks_per_req);
  // A slot mapping in page-locked host memory is written in place by the
  // kernels (its bytes cross the host link while the batch runs, no copy
  // follows); any other host buffer gets a device buffer and a copy back.
  // So does every buffer of a host-tier store, whose batches keep the host
  // link busy with their cold rows: measured on B200 (LRU hot set with
  // prefetch, Qwen shapes, 1.26 MB of slots), the writes in place cost
  // 0.44 ms a batch there, the copy after the batch much less.
  int64_t* direct_slots = (slot_out && slot_cap > 0 && !s->host_arena)
      ? static_cast<int64_t*>(mapped_host_range(slot_out, size_t(slot_cap) * 8)) : nullptr;
  const int64_t n_slots = (slot_out && !direct_slots) ? slot_cap : 0;
  int rc = grow_stage(s, n_off + n_ids + n_sp + n_bt + 4, n_slots);
  if (rc != IS_OK) return rc;
  const bool lru = s->hot_policy == IS_HOT_LRU;
  if (lru) {  // this batch's cold facts: promotions fused into the batch
    rc = lru_touch(s, fact_ids, num_ids, st, true, nullptr);
    if (rc != IS_OK) return rc;
    s->batch_tick = s->tick;
  }
  // Pack the four index arrays into one pinned buffer: one host-to-device copy.
  int32_t* h = s->host_stage;
  std::memcpy(h, req_off, n_off * 4);
  if (n_ids) std::memcpy(h + n_off, fact_ids, n_ids * 4);
  if (n_sp) std::memcpy(h + n_off + n_ids, start_pos, n_sp * 4);
  if (n_bt) std::memcpy(h + n_off + n_ids + n_sp, block_tables, n_bt * 4);
  int32_t* d_off = s->stage;
  int32_t* d_ids = d_off + n_off;
  int32_t* d_sp = d_ids + n_ids;
  int32_t* d_bt = d_sp + n_sp;
  if (cudaMemcpyAsync(d_off, h, (n_off + n_ids + n_sp + n_bt) * 4, cudaMemcpyHostToDevice, st) != cudaSuccess) {
    lru_finish(s, st, false);
    return IS_ERR_CUDA;
  }
  s->batch_pend = s->pend_np > 0;
  // The kernel that records the batch's errors also writes the status into
  // the mapped pinned copy: no copy back after the batch.  (A value it did
  // not write is seen as the marker, and the status is then copied.)
  constexpr int32_t kUnwritten = INT32_MIN;
  s->host_status->code = kUnwritten;
  s->batch_mirror = s->host_status_dev;
  rc = is_inject_batch(s, R, d_off, d_ids, num_ids, d_sp, d_bt, max_blocks_per_req, cache,
                       direct_slots ? direct_slots : slot_out ? s->stage_slots : nullptr, slot_cap, stream);
  s->batch_mirror = nullptr;
  s->batch_pend = false;
  if (rc != IS_OK) {
    lru_finish(s, st, false);  // nothing ran: copy the promoted facts instead
    return rc;
  }
  // The next batch's cold facts move over the host link while this one runs.
  // (A failure here is reported after this batch has been completed: its
  // pending promotions must still enter the hot table.)
  const int rc_pf = (lru && num_next > 0) ? lru_prefetch(s, next_ids, num_next) : IS_OK;
  bool copied = !(slot_out && slot_cap > 0) || direct_slots ||
                cudaMemcpyAsync(slot_out, s->stage_slots, size_t(slot_cap) * 8, cudaMemcpyDeviceToHost,
                                st) == cudaSuccess;
  // One wait; the status is already on its way to the pinned copy.
  const bool mirrored = s->host_status_dev != nullptr;
  if (!mirrored)
    copied = copied && cudaMemcpyAsync(s->host_status, s->d_status, sizeof(isk::DevStatus),
                                       cudaMemcpyDeviceToHost, st) == cudaSuccess;
  bool waited = cudaStreamSynchronize(st) == cudaSuccess;
  if (copied && waited && s->host_status->code == kUnwritten)
    waited = cudaMemcpy(s->host_status, s->d_status, sizeof(isk::DevStatus), cudaMemcpyDeviceToHost) ==
             cudaSuccess;
  const int code = (copied && waited) ? s->host_status->code : IS_ERR_CUDA;
  if (s->pend_np > 0 && (lru_finish(s, st, code == 0) != IS_OK || cudaStreamSynchronize(st) != cudaSuccess))
    return IS_ERR_CUDA;
  if (!copied || !waited) return IS_ERR_CUDA;
  if (code != 0 && cudaMemset(s->d_status, 0, sizeof(isk::DevStatus)) != cudaSuccess) return IS_ERR_CUDA;
  return code != IS_OK ? code : rc_pf;
}

int is_inject_batch_host(is_store_t* s, int32_t R, const int32_t* req_off, const int32_t* fact_ids,
                         int32_t num_ids, const int32_t* start_pos, const int32_t* block_tables,
                         int32_t max_blocks_per_req, const is_cache_t* cache, int64_t* slot_out,
                         int64_t slot_cap, void* stream) {
  return host_batch(s, R, req_off, fact_ids, num_ids, start_pos, block_tables, max_blocks_per_req, cache,
                    slot_out, slot_cap, nullptr, 0, stream);
}

int is_inject_batch_host_next(is_store_t* s, int32_t R, const int32_t* req_off, const int32_t* fact_ids,
                              int32_t num_ids, const int32_t* start_pos, const int32_t* block_tables,
                              int32_t max_blocks_per_req, const is_cache_t* cache, int64_t* slot_out,
                              int64_t slot_cap, const int32_t* next_fact_ids, int32_t num_next_ids,
                              void* stream) {
  return host_batch(s, R, req_off, fact_ids, num_ids, start_pos, block_tables, max_blocks_per_req, cache,
                    slot_out, slot_cap, next_fact_ids, num_next_ids, stream);
}

int is_last_error(is_store_t* s, void* stream, int64_t* detail) {
  if (!s) return IS_ERR_INVALID_ARG;
  DeviceGuard guard(s->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  isk::DevStatus h{};
  if (cudaStreamSynchronize(st) != cudaSuccess) return IS_ERR_CUDA;
  if (cudaMemcpy(&h, s->d_status, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return IS_ERR_CUDA;
  if (h.code != 0 && cudaMemset(s->d_status, 0, sizeof(h)) != cudaSuccess) return IS_ERR_CUDA;
  if (detail) *detail = h.detail;
  return h.code;
}

int is_last_error_timeout(is_store_t* s, void* stream, int32_t timeout_ms, int64_t* detail) {
  if (!s || timeout_ms < 0) return IS_ERR_INVALID_ARG;
  DeviceGuard guard(s->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto deadline = std::chrono::steady_clock::now() + std::chrono::milliseconds(timeout_ms);
  for (;;) {
    const cudaError_t q = cudaStreamQuery(st);
    if (q == cudaSuccess) break;
    if (q != cudaErrorNotReady) return IS_ERR_CUDA;
    if (std::chrono::steady_clock::now() >= deadline) return IS_ERR_TIMEOUT;
    std::this_thread::sleep_for(std::chrono::microseconds(200));
  }
  return is_last_error(s, stream, detail);
}

int is_store_set_small_batch_limit(is_store_t* s, int32_t max_requests) {
  if (!s || max_requests < 0 || max_requests > isk::kSmallRequests) return IS_ERR_INVALID_ARG;
  s->small_limit = max_requests;
  return IS_OK;
}

int is_store_set_timing(is_store_t* s, int enable) {
  if (!s) return IS_ERR_INVALID_ARG;
  s->timing = enable != 0;
  return IS_OK;
}

int is_store_kernel_time(is_store_t* s, double* total_ms, int64_t* launches) {
  if (!s) return IS_ERR_INVALID_ARG;
  DeviceGuard guard(s->device);
  double sum = 0.0;
  for (size_t i = 0; i < s->events_used; ++i) {
    if (cudaEventSynchronize(s->events[i].stop) != cudaSuccess) return IS_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, s->events[i].start, s->events[i].stop) != cudaSuccess) return IS_ERR_CUDA;
    sum += ms;
  }
  if (total_ms) *total_ms = sum;
  if (launches) *launches = int64_t(s->events_used);
  s->events_used = 0;
  return IS_OK;
}

}  // extern "C"

// ===================================================================
// Allocation-free entry point (is_inject_batch_noalloc).
//
// For callers that must not allocate device memory (an engine whose pool
// owns the GPU, a plugin host that forbids hidden allocations).  The per-batch work space is one fixed
// device array in this module; the same plan and inject kernels as
// is_inject_batch run on it.
// ===================================================================

#include <mutex>

namespace {

constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Work-space layout, byte offsets into g_noalloc_scratch.
constexpr size_t kNaStatus = 0;
constexpr size_t kNaHeader = align256(kNaStatus + sizeof(isk::DevStatus));
constexpr size_t kNaInvFreq = align256(kNaHeader + sizeof(isk::PlanHeader));
constexpr size_t kNaSeg = align256(kNaInvFreq + sizeof(double) * (IS_NOALLOC_MAX_HEAD_DIM / 2));
constexpr size_t kNaNblk = align256(kNaSeg + sizeof(int32_t) * IS_NOALLOC_MAX_FACT_IDS);
constexpr size_t kNaBlk0 = align256(kNaNblk + sizeof(int32_t) * IS_NOALLOC_MAX_REQUESTS);
constexpr size_t kNaTok0 = align256(kNaBlk0 + sizeof(int32_t) * (IS_NOALLOC_MAX_REQUESTS + 1));
constexpr size_t kNaLen = align256(kNaTok0 + sizeof(long long) * (IS_NOALLOC_MAX_REQUESTS + 1));
constexpr size_t kNaErr = align256(kNaLen + sizeof(int32_t) * IS_NOALLOC_MAX_REQUESTS);
constexpr size_t kNaDesc = align256(kNaErr + sizeof(int32_t) * IS_NOALLOC_MAX_REQUESTS);
constexpr size_t kNaBytes = align256(kNaDesc + sizeof(isk::BlockDesc) * IS_NOALLOC_MAX_BLOCKS);

constexpr int kNaMaxDevices = 64;

// Per-device launch settings, filled by the first call on the device.
struct NoAllocDevice {
  bool ready = false;
  unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch
  int grid[4][2] = {};               // inject grid per head-dim slot and RoPE style
};

NoAllocDevice g_na_devices[kNaMaxDevices];
std::mutex g_na_mutex;

int head_dim_slot(int d) { return d == 32 ? 0 : d == 64 ? 1 : d == 128 ? 2 : 3; }

}  // namespace

// The work space: one array per GPU that loads this library, kept until exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNaBytes];

namespace {

// Once per device, with that device current: the work space's device
// address (host code cannot use the symbol itself as an address) and the
// kernels' shared-memory limits and resident-CTA grid sizes.
int noalloc_setup(int dev, NoAllocDevice** out) {
  std::lock_guard<std::mutex> lock(g_na_mutex);
  NoAllocDevice& d = g_na_devices[dev];
  if (!d.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return IS_ERR_CUDA;
    }
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return IS_ERR_CUDA;
    const int dims[4] = {32, 64, 128, 256};
    for (int di = 0; di < 4; ++di)
      for (int style = 0; style < 2; ++style) {
        const int D = dims[di];
        const size_t smem_max = cs_smem_bytes(D, isk::kMaxBlockSize);
        void* f_pow2 = pick_inject_t<true>(D, style);
        void* f_gen = pick_inject_t<false>(D, style);
        if (cudaFuncSetAttribute(f_pow2, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_max)) !=
                cudaSuccess ||
            cudaFuncSetAttribute(f_gen, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_max)) !=
                cudaSuccess)
          return IS_ERR_CUDA;
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, f_pow2, kInjectThreads,
                                                          cs_smem_bytes(D, 16)) != cudaSuccess)
          return IS_ERR_CUDA;
        d.grid[di][style] = std::max(1, per_sm) * sms;
      }
    d.scratch = static_cast<unsigned char*>(p);
    d.ready = true;
  }
  *out = &d;
  return IS_OK;
}

}  // namespace

extern "C" int is_inject_batch_noalloc(const is_store_config_t* cfg, const void* k_store,
                                       const void* v_store, int64_t plane_tokens,
                                       const int64_t* fact_offsets, const int32_t* fact_lens,
                                       int32_t num_facts, int32_t R, const int32_t* req_off,
                                       const int32_t* fact_ids, int32_t num_ids,
                                       const int32_t* start_pos, const int32_t* block_tables,
                                       int32_t max_blocks_per_req, const is_cache_t* cache,
                                       int64_t* slot_out, int64_t slot_cap, void* status_out,
                                       void* stream) {
  if (!cfg || !cache || !k_store || !v_store || plane_tokens < 1 || num_facts < 0 || R < 0 ||
      num_ids < 0 || max_blocks_per_req < 1 || !req_off)
    return IS_ERR_INVALID_ARG;
  if (num_facts > 0 && (!fact_offsets || !fact_lens)) return IS_ERR_INVALID_ARG;
  if ((R > 0 && (!start_pos || !block_tables)) || (num_ids > 0 && !fact_ids)) return IS_ERR_INVALID_ARG;
  const is_store_config_t& c = *cfg;
  if (c.num_layers < 1 || c.num_kv_heads < 1 || !(c.rope_theta > 0.0) ||
      (c.rope_style != IS_ROPE_ROTATE_HALF && c.rope_style != IS_ROPE_INTERLEAVED) ||
      (c.rope_scaling != IS_SCALING_NONE && c.rope_scaling != IS_SCALING_LLAMA3))
    return IS_ERR_INVALID_ARG;
  if (c.rope_scaling == IS_SCALING_LLAMA3 &&
      (!(c.scale_factor > 0.0) || !(c.low_freq_factor > 0.0) || !(c.high_freq_factor > c.low_freq_factor) ||
       c.original_max_position <= 0))
    return IS_ERR_INVALID_ARG;
  if (!head_dim_supported(c.head_dim) || c.head_dim > IS_NOALLOC_MAX_HEAD_DIM) return IS_ERR_NOT_SUPPORTED;
  if (R > IS_NOALLOC_MAX_REQUESTS || num_ids > IS_NOALLOC_MAX_FACT_IDS) return IS_ERR_CAPACITY;
  const is_cache_t& k = *cache;
  if (!k.k_cache || !k.v_cache || k.num_blocks < 1 || k.block_size < 1 || k.block_size > isk::kMaxBlockSize)
    return IS_ERR_INVALID_ARG;
  if (!aligned16(k.k_cache) || !aligned16(k.v_cache) || !aligned16(k_store) || !aligned16(v_store) ||
      k.layer_stride % 8 || k.block_stride % 8 || k.token_stride % 8 || k.head_stride % 8 ||
      k.layer_stride < 0 || k.block_stride < 0 || k.token_stride < 0 || k.head_stride < 0)
    return IS_ERR_INVALID_ARG;
  if (slot_out && slot_cap < 0) return IS_ERR_INVALID_ARG;
  if (int64_t(max_blocks_per_req) * k.block_size > (int64_t(1) << 31) - 1) return IS_ERR_NOT_SUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNaMaxDevices) return IS_ERR_CUDA;
  NoAllocDevice* nd = nullptr;
  int rc = noalloc_setup(dev, &nd);
  if (rc != IS_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned char* ws = nd->scratch;
  auto* status = reinterpret_cast<isk::DevStatus*>(ws + kNaStatus);
  auto* hdr = reinterpret_cast<isk::PlanHeader*>(ws + kNaHeader);
  auto* inv_freq = reinterpret_cast<double*>(ws + kNaInvFreq);

  // The status word is the only field read before it is written: clear it.
  if (cudaMemsetAsync(status, 0, sizeof(isk::DevStatus), st) != cudaSuccess) return IS_ERR_CUDA;
  const int nf = c.head_dim / 2;
  isk::inv_freq_kernel<<<(nf + 127) / 128, 128, 0, st>>>(
      inv_freq, c.head_dim, c.rope_theta, c.rope_scaling, c.scale_factor, c.low_freq_factor,
      c.high_freq_factor, double(c.original_max_position));

  const int grid = nd->grid[head_dim_slot(c.head_dim)][c.rope_style];
  isk::PlanArgs pa;
  pa.R = R;
  pa.req_off = req_off;
  pa.fact_ids = fact_ids;
  pa.num_ids = num_ids;
  pa.start_pos = start_pos;
  pa.block_tables = block_tables;
  pa.max_blocks = max_blocks_per_req;
  pa.num_blocks = k.num_blocks;
  pa.B = k.block_size;
  pa.L = c.num_layers;
  pa.H = c.num_kv_heads;
  pa.fact_len = fact_lens;
  pa.num_facts = num_facts;
  // The caller's fact table: ids whose entry leaves the arenas are refused.
  pa.chk_off = fact_offsets;
  pa.chk_plane = plane_tokens;
  pa.slot_out = slot_out;
  pa.slot_cap = slot_cap;
  pa.grid_ctas = grid;
  const int loop = launch_loop(c.head_dim, k.block_size, c.num_kv_heads);
  pa.row_units = loop != 0;
  pa.max_batch_blocks = IS_NOALLOC_MAX_BLOCKS;
  pa.seg = reinterpret_cast<int32_t*>(ws + kNaSeg);
  pa.req_nblk = reinterpret_cast<int32_t*>(ws + kNaNblk);
  pa.req_blk0 = reinterpret_cast<int32_t*>(ws + kNaBlk0);
  pa.req_tok0 = reinterpret_cast<long long*>(ws + kNaTok0);
  pa.req_len = reinterpret_cast<int32_t*>(ws + kNaLen);
  pa.req_err = reinterpret_cast<int32_t*>(ws + kNaErr);
  pa.desc = reinterpret_cast<isk::BlockDesc*>(ws + kNaDesc);
  pa.hdr = hdr;
  pa.st = status;
  pa.st_mirror = nullptr;
  isk::plan_kernel<kPlanThreads, false><<<1, kPlanThreads, 0, st>>>(pa);

  isk::InjectArgs ia{};
  ia.k_store = static_cast<const uint16_t*>(k_store);
  ia.v_store = static_cast<const uint16_t*>(v_store);
  ia.plane = plane_tokens * c.head_dim;
  ia.fact_off = fact_offsets;
  ia.fact_len = fact_lens;
  ia.inv_freq = inv_freq;
  ia.L = c.num_layers;
  ia.H = c.num_kv_heads;
  ia.req_off = req_off;
  ia.fact_ids = fact_ids;
  ia.start_pos = start_pos;
  ia.block_tables = block_tables;
  ia.max_blocks = max_blocks_per_req;
  ia.k_cache = static_cast<uint16_t*>(k.k_cache);
  ia.v_cache = static_cast<uint16_t*>(k.v_cache);
  ia.ls = k.layer_stride;
  ia.bs = k.block_stride;
  ia.ts = k.token_stride;
  ia.hs = k.head_stride;
  ia.num_blocks = k.num_blocks;
  ia.B = k.block_size;
  ia.vec_order = launch_vec_order(c.head_dim, k.block_size, c.num_kv_heads, k.token_stride, k.head_stride);
  ia.slot_out = slot_out;
  ia.seg = pa.seg;
  ia.req_tok0 = pa.req_tok0;
  ia.desc = pa.desc;
  ia.hdr = hdr;
  ia.st = status;
  // The kernel variant is_inject_batch launches for the same shape and layout.
  void* fn = pick_inject(c.head_dim, c.rope_style, c.num_kv_heads, k.block_size, false, loop);
  void* args[] = {&ia};
  if (cudaLaunchKernel(fn, dim3(unsigned(grid)), dim3(kInjectThreads), args,
                       cs_smem_bytes(c.head_dim, k.block_size), st) != cudaSuccess)
    return IS_ERR_CUDA;
  if (status_out && cudaMemcpyAsync(status_out, status, sizeof(isk::DevStatus),
                                    cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return IS_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? IS_OK : IS_ERR_CUDA;
}
