// Device code of the retrieve-and-inject path for sm_100a.
//
// What a batch computes (technical summary of "InferScale: GPU-Native KV
// Injection for Personalized LLM Serving", section "Methodology -- 2. Online
// phase: Chunked RoPE and KV injection"): each request's retrieved facts are
// laid out as one contiguous segment at new serving positions ("Dynamic
// rotation"), every stored pre-RoPE key is rotated to its token's position
// (RoPE; fp64 angles, fp32 rotation, bf16 round-to-nearest-even), and K and
// the raw V are scatter-copied into the paged KV cache ("Injection").
//
// Kernels:
//   plan_kernel          one CTA: composes the segments, validates the batch,
//                        writes one descriptor per touched cache block.
//   inject_kernel        persistent grid, launched as a programmatic
//                        dependent of the plan: per work unit (one cache
//                        block of one request x a range of layers) gathers
//                        the block's K/V rows, rotates K, writes the cache.
//   small_inject_kernel  small batches: every CTA composes the batch itself
//                        in shared memory, then runs the same per-unit work.
//   promote_kernel,      host-tier store, LRU hot set: copy promoted facts
//   hot_table_kernel     into HBM slots, patch the hot table.
//   inv_freq_kernel      RoPE frequencies (fp64, Llama-3.1 rule optional).
//
// The path is a copy with a small rotation: bandwidth-bound on HBM.  Every
// global access is a 16-byte vector; stored rows are read in runs along
// their token planes and each block's layer of the cache is one contiguous
// run written by the whole CTA.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#ifndef IS_UNITS_PER_CTA
#define IS_UNITS_PER_CTA 256
#endif
// Smallest (layer, head) row count of a work unit of a large batch, and the
// larger count used when it still leaves IS_UNITS_PER_CTA_MIN units per CTA.
#ifndef IS_UNIT_MIN_ROWS
#define IS_UNIT_MIN_ROWS 16
#endif
#ifndef IS_UNIT_ROWS_LARGE
#define IS_UNIT_ROWS_LARGE 32
#endif
#ifndef IS_UNITS_PER_CTA_MIN
#define IS_UNITS_PER_CTA_MIN 32
#endif
// 1: the copy loop keeps two half-chunks in flight (software pipeline).
#ifndef IS_PIPELINE
#define IS_PIPELINE 1
#endif


namespace isk {

// Status codes, same values as inject_store.h.
enum : int32_t {
  kOk = 0,
  kErrInvalidArg = -1,
  kErrBadFactId = -2,
  kErrPosition = -3,
  kErrBadBlock = -4,
  kErrCapacity = -5,
};

struct DevStatus {
  int32_t code;
  int32_t pad;
  long long detail;
};

// Written by plan_kernel, read by inject_kernel.
struct PlanHeader {
  int32_t total_blocks;      // touched cache blocks over all valid requests
  int32_t rows_per_unit;     // (layer, head) rows one work unit covers
  int32_t units_per_block;   // ceil(L * H / rows_per_unit)
  int32_t total_units;       // total_blocks * units_per_block (0: write nothing)
  unsigned int next_unit;    // dynamic work counter, reset by plan_kernel
  int32_t pad;
  long long total_tokens;    // segment tokens over all requests
};

// One touched cache block of one request.
struct __align__(16) BlockDesc {
  int32_t r;     // request
  int32_t b;     // logical block index in the request's table
  int32_t j;     // CSR index of the first fact with a token in the block
  int32_t pad;
};

__device__ __forceinline__ void record_error(DevStatus* st, int32_t code, long long detail) {
  if (atomicCAS(&st->code, 0, code) == 0) st->detail = detail;
}

// The status once the batch's errors are recorded (by the thread that
// records them), copied to m when set: pinned host memory mapped for the
// device, which the host entry point reads after its wait instead of
// copying the status back.
__device__ __forceinline__ void mirror_status(const DevStatus* st, DevStatus* m) {
  if (m == nullptr) return;
  m->detail = __ldcg(&st->detail);
  m->code = __ldcg(&st->code);
}

// ---------------------------------------------------------------- plan kernel

// Work-unit size: rows per unit rpu and units per block upb, where a row is
// one (layer, head) pair of a cache block, numbered w = layer * H + head, and
// unit g of a block covers rows [g * rpu, min(L * H, (g + 1) * rpu)).  A batch
// whose one-layer units fit in about two waves of the grid is split into at
// most one wave of units (latency: everything is in flight at once and no
// CTA runs a second unit after the first -- one more unit than the grid
// holds doubles the time of a single request), as many as fit: with
// row_units (the per-thread copy loops, which take any row range) into
// equal row ranges, otherwise into equal layer ranges.  Larger batches aim at ~IS_UNITS_PER_CTA units
// per CTA, so the dynamic schedule's tail (at most one unit) stays short,
// in whole layers with at least IS_UNIT_MIN_ROWS rows (and at least two
// layers) per unit so a unit's set-up (slot walk, cos/sin table, barriers)
// is shared by enough copies, and IS_UNIT_ROWS_LARGE rows when the batch
// still has IS_UNITS_PER_CTA_MIN units per CTA with them.  Measured on B200
// over the Mistral/Qwen sweep grid: with H = 4, two-layer units ran at 0.87
// of the copy peak, 16-row units at 0.93-0.96, 32-row units up to 0.97 on
// large batches but slower where they leave few units per CTA.
__device__ __forceinline__ void unit_size(int32_t total_blocks, int32_t L, int32_t H, int32_t grid_ctas,
                                          bool row_units, int32_t& rpu, int32_t& upb) {
  const long long grid = grid_ctas;
  const int32_t LH = L * H;
  upb = 1;
  if (total_blocks > 0 && (long long)total_blocks * L <= 2 * grid) {
    // units per block such that every unit has a CTA of its own (ceil-ing
    // the range lengths below only lowers the count)
    const int32_t fit = max(1, grid_ctas / total_blocks);
    if (row_units) {
      upb = min(LH, fit);
      rpu = (LH + upb - 1) / upb;
      upb = (LH + rpu - 1) / rpu;
      return;
    }
    upb = min(L, fit);
  } else if (total_blocks > 0) {
    const int32_t h = max(H, 1);
    const int32_t lmin = min(L, max(2, (IS_UNIT_MIN_ROWS + h - 1) / h));
    const int32_t lbig = min(L, max(2, (IS_UNIT_ROWS_LARGE + h - 1) / h));
    const long long cap_big = max(1, L / lbig);
    const long long cap = (long long)total_blocks * cap_big >= IS_UNITS_PER_CTA_MIN * grid
                              ? cap_big : (long long)max(1, L / lmin);
    const long long want = (grid * IS_UNITS_PER_CTA + total_blocks - 1) / total_blocks;
    upb = int32_t(max(1LL, min(want, cap)));
  }
  const int32_t lpu = (L + upb - 1) / upb;
  upb = (L + lpu - 1) / lpu;
  rpu = lpu * H;
}

struct PlanArgs {
  int32_t R;
  const int32_t* req_off;    // [R+1]
  const int32_t* fact_ids;   // [num_ids]
  int32_t num_ids;
  const int32_t* start_pos;  // [R]
  const int32_t* block_tables;  // [R][max_blocks]
  int32_t max_blocks;
  int32_t num_blocks;        // cache blocks (table entries outside: BAD_BLOCK)
  int32_t B;
  int32_t L;
  int32_t H;
  const int32_t* fact_len;   // store: [num_facts]
  int32_t num_facts;
  // A fact table the library did not build (the allocation-free entry
  // point): when chk_off is set, an id whose entry does not lie inside the
  // arenas -- offset < 0, length < 1 or offset + length > chk_plane tokens
  // -- counts as an id outside the store.
  const int64_t* chk_off;
  int64_t chk_plane;
  int64_t* slot_out;         // optional
  int64_t slot_cap;
  int32_t grid_ctas;         // size of the inject grid (for unit sizing)
  int32_t row_units;         // the inject kernel's copy loop takes any row range
  int32_t max_batch_blocks;  // capacity of desc
  // work space
  int32_t* seg;              // [num_ids]   segment offset of each CSR entry (-1: bad id)
  int32_t* req_nblk;         // [R]         touched blocks (0 when invalid)
  int32_t* req_blk0;         // [R+1]       exclusive prefix of req_nblk
  long long* req_tok0;       // [R+1]       exclusive prefix of segment lengths
  int32_t* req_len;          // [R]         segment length (valid facts)
  int32_t* req_err;          // [R]         0, or the request's IS_ERR code
  BlockDesc* desc;           // [max_batch_blocks]
  PlanHeader* hdr;
  DevStatus* st;
  DevStatus* st_mirror;      // optional: see mirror_status
};

// Shared-memory plan: batches of at most kPlanSmemRequests requests and
// kPlanSmemIds fact ids keep the CSR, the start positions, the lengths /
// segment offsets and the per-request sums in shared memory, so the
// per-request phases chain shared-memory rather than L2 latencies; only seg,
// req_tok0 and the descriptors (what the inject kernel reads) go to global
// memory.  Larger batches run the same phases on the global work space.
constexpr int kPlanSmemRequests = 1024;
constexpr int kPlanSmemIds = 16384;

__host__ __device__ constexpr size_t plan_smem_bytes(int R, int num_ids) {
  return sizeof(long long) * size_t(R + 1) + sizeof(int32_t) * (size_t(R + 1) * 2 + size_t(R) * 4 + size_t(num_ids));
}

template <int NT, bool SMEM>
__global__ void __launch_bounds__(NT) plan_kernel(PlanArgs a) {
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ int s_bad;
  __shared__ int s_len_over;  // a request's facts total more than 2^31 - 1 tokens
  __shared__ long long s_wsum_blk[NW];
  __shared__ long long s_wsum_tok[NW];
  __shared__ long long s_total_blk;
  // First error in request order: (request << 32) | logical block, the
  // block part used for a block-table entry outside the cache.
  __shared__ unsigned long long s_err_key;
  extern __shared__ __align__(16) unsigned char plan_dyn[];

  // The inject grid may be scheduled now; it waits for this grid's results
  // (griddepcontrol.wait) before reading any of them.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int32_t* req_off = a.req_off;
  const int32_t* start_pos = a.start_pos;
  int32_t* seg = a.seg;
  int32_t* req_nblk = a.req_nblk;
  int32_t* req_blk0 = a.req_blk0;
  long long* req_tok0 = a.req_tok0;
  int32_t* req_len = a.req_len;
  int32_t* req_err = a.req_err;
  if constexpr (SMEM) {
    long long* s_tok0 = reinterpret_cast<long long*>(plan_dyn);  // [R+1]
    int32_t* s_off = reinterpret_cast<int32_t*>(s_tok0 + (a.R + 1));
    int32_t* s_blk0 = s_off + (a.R + 1);     // [R+1]
    int32_t* s_start = s_blk0 + (a.R + 1);   // [R]
    int32_t* s_nblk = s_start + a.R;         // [R]
    int32_t* s_len = s_nblk + a.R;           // [R]
    int32_t* s_err = s_len + a.R;            // [R]
    int32_t* s_seg = s_err + a.R;            // [num_ids]
    for (int i = tid; i <= a.R; i += NT) s_off[i] = a.req_off[i];
    for (int i = tid; i < a.R; i += NT) s_start[i] = a.start_pos[i];
    __syncthreads();
    req_off = s_off;
    start_pos = s_start;
    seg = s_seg;
    req_nblk = s_nblk;
    req_blk0 = s_blk0;
    req_tok0 = s_tok0;
    req_len = s_len;
    req_err = s_err;
  }

  // The CSR must start at 0, end at num_ids and never decrease; otherwise
  // the whole batch is rejected and nothing is written.
  if (tid == 0) {
    s_bad = a.R < 0 || req_off[0] != 0 || req_off[a.R] != a.num_ids;
    s_len_over = 0;
    s_err_key = ~0ull;
  }
  __syncthreads();
  for (int r = tid; r < a.R; r += NT)
    if (req_off[r + 1] < req_off[r]) s_bad = 1;
  __syncthreads();
  if (tid == 0 && s_bad) {
    record_error(a.st, kErrInvalidArg, -1);
    mirror_status(a.st, a.st_mirror);
    a.hdr->total_blocks = 0;
    a.hdr->total_units = 0;
    a.hdr->units_per_block = 1;
    a.hdr->rows_per_unit = a.L * a.H;
    a.hdr->next_unit = 0;
    a.hdr->total_tokens = 0;
  }
  if (s_bad) return;

  // Phase 0, all threads: the length of every listed fact (-1 for an id
  // outside the store), fetched in parallel into seg[], which phase 1 then
  // overwrites with segment offsets.
  constexpr int P0 = 8;  // loads in flight per thread
  for (int32_t base = 0; base < a.num_ids; base += NT * P0) {
    int32_t f[P0];
#pragma unroll
    for (int q = 0; q < P0; ++q) {
      const int32_t j = base + q * NT + tid;
      f[q] = j < a.num_ids ? a.fact_ids[j] : -1;
    }
    if (a.chk_off == nullptr) {
#pragma unroll
      for (int q = 0; q < P0; ++q) {
        const int32_t j = base + q * NT + tid;
        if (j < a.num_ids) seg[j] = (f[q] >= 0 && f[q] < a.num_facts) ? a.fact_len[f[q]] : -1;
      }
    } else {
#pragma unroll
      for (int q = 0; q < P0; ++q) {
        const int32_t j = base + q * NT + tid;
        if (j >= a.num_ids) continue;
        int32_t lf = -1;
        if (f[q] >= 0 && f[q] < a.num_facts) {
          const int32_t n = a.fact_len[f[q]];
          const int64_t o = a.chk_off[f[q]];
          if (n >= 1 && o >= 0 && o <= a.chk_plane - n) lf = n;
        }
        seg[j] = lf;
      }
    }
  }
  __syncthreads();

  // Phase 1, one warp per request: segment offsets of its facts (exclusive
  // prefix of their lengths, in retrieval order), length, validity, blocks.
  for (int r = warp; r < a.R; r += NW) {
    const int32_t j0 = req_off[r], j1 = req_off[r + 1];
    int32_t err = kOk;
    long long S = 0;
    if (j0 < 0 || j1 < j0 || j1 > a.num_ids) {
      err = kErrInvalidArg;  // malformed range: no tokens
    } else {
      for (int32_t base = j0; base < j1; base += 32) {
        const int32_t j = base + lane;
        const int32_t lj = j < j1 ? seg[j] : 0;
        const bool ok = lj >= 0;
        const long long len = ok ? lj : 0;
        long long x = len;  // inclusive warp scan, 64-bit: lengths may be large
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const long long y = __shfl_up_sync(0xffffffffu, x, d);
          if (lane >= d) x += y;
        }
        // (offsets of a request longer than 2^31 - 1 tokens wrap here, but
        // such a request fails the batch below and its offsets are not read)
        if (j < j1) seg[j] = ok ? int32_t(S + x - len) : -1;
        const unsigned badm = __ballot_sync(0xffffffffu, j < j1 && !ok);
        if (badm && err == kOk) err = kErrBadFactId;
        S += __shfl_sync(0xffffffffu, x, 31);
      }
    }
    const int32_t start = start_pos[r];
    if (err == kOk && start < 0) err = kErrInvalidArg;
    if (err == kOk && (long long)start + S > (long long)a.max_blocks * a.B) err = kErrPosition;
    if (lane == 0) {
      int32_t nblk = 0;
      if (err == kOk && S > 0) nblk = int32_t((start + S - 1) / a.B - start / a.B + 1);
      req_nblk[r] = nblk;
      if (S > 0x7fffffffLL) s_len_over = 1;
      req_len[r] = int32_t(min(S, 0x7fffffffLL));
      req_err[r] = err;
      if (err != kOk) atomicMin(&s_err_key, (unsigned long long)r << 32);
    }
  }
  __syncthreads();

  // Phase 2: exclusive prefixes over requests (blocks and tokens).  Thread t
  // owns a contiguous run of requests.
  const int per = (a.R + NT - 1) / NT;
  const int r0 = min(a.R, tid * per), r1 = min(a.R, r0 + per);
  long long my_blk = 0;
  long long my_tok = 0;
  for (int r = r0; r < r1; ++r) { my_blk += req_nblk[r]; my_tok += req_len[r]; }
  long long xb = my_blk;
  long long xt = my_tok;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const long long yb = __shfl_up_sync(0xffffffffu, xb, d);
    const long long yt = __shfl_up_sync(0xffffffffu, xt, d);
    if (lane >= d) { xb += yb; xt += yt; }
  }
  if (lane == 31) { s_wsum_blk[warp] = xb; s_wsum_tok[warp] = xt; }
  __syncthreads();
  // Exclusive prefix of the warp sums: a shuffle scan over lanes = warps.
  long long wb = lane < NW ? s_wsum_blk[lane] : 0;
  long long wt = lane < NW ? s_wsum_tok[lane] : 0;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const long long yb = __shfl_up_sync(0xffffffffu, wb, d);
    const long long yt = __shfl_up_sync(0xffffffffu, wt, d);
    if (lane >= d) { wb += yb; wt += yt; }
  }
  wb = warp > 0 ? __shfl_sync(0xffffffffu, wb, warp - 1) : 0;
  wt = warp > 0 ? __shfl_sync(0xffffffffu, wt, warp - 1) : 0;
  // Block prefixes are stored in 32 bits: a batch whose total would not
  // fit is over every block capacity and fails below before they are read.
  long long eb = wb + xb - my_blk;
  long long et = wt + xt - my_tok;
  for (int r = r0; r < r1; ++r) {
    req_blk0[r] = int32_t(min(eb, 0x7fffffffLL));
    req_tok0[r] = et;
    eb += req_nblk[r];
    et += req_len[r];
  }
  if (tid == NT - 1) {
    req_blk0[a.R] = int32_t(min(eb, 0x7fffffffLL));
    req_tok0[a.R] = et;
    s_total_blk = eb;
  }
  __syncthreads();
  if constexpr (SMEM) {
    // What the inject kernel reads: segment offsets and token prefixes.
    for (int32_t j = tid; j < a.num_ids; j += NT) a.seg[j] = seg[j];
    for (int r = tid; r <= a.R; r += NT) a.req_tok0[r] = req_tok0[r];
  }
  const int32_t total_blocks = req_blk0[a.R];
  const long long total_tokens = req_tok0[a.R];
  const bool over_slots = (a.slot_out != nullptr && total_tokens > a.slot_cap) || s_len_over;
  const bool over_blocks = s_total_blk > a.max_batch_blocks;

  // Work units are counted in 32 bits: a batch needing more is over capacity.
  __shared__ int s_over_units;
  if (tid == 0) {
    int32_t rpu, upb;
    unit_size(total_blocks, a.L, a.H, a.grid_ctas, a.row_units != 0, rpu, upb);
    s_over_units = (long long)total_blocks * upb > 0x7fffffffLL;
    const bool over = over_slots || over_blocks || s_over_units;
    a.hdr->rows_per_unit = rpu;
    a.hdr->units_per_block = upb;
    a.hdr->total_blocks = total_blocks;
    a.hdr->total_tokens = total_tokens;
    a.hdr->next_unit = 0;
    a.hdr->total_units = over ? 0 : total_blocks * upb;
    // A batch over capacity writes nothing and reports only that.
    if (over) {
      record_error(a.st, kErrCapacity, total_tokens);
      mirror_status(a.st, a.st_mirror);
    }
  }
  __syncthreads();
  if (over_slots || over_blocks || s_over_units) return;

  // Phase 3, one warp per request: block descriptors (lanes over blocks, so
  // a warp writes consecutive descriptors), the check of every touched
  // block-table entry, and -1 slots for the tokens of invalid requests.
  auto check_entry = [&](int r, int32_t b, int32_t phys) {
    if (phys < 0 || phys >= a.num_blocks) atomicMin(&s_err_key, ((unsigned long long)r << 32) | unsigned(b));
  };
  for (int r = warp; r < a.R; r += NW) {
    const int32_t j0 = req_off[r], j1 = req_off[r + 1];
    const long long t0 = req_tok0[r];
    if (req_err[r] != kOk) {
      if (a.slot_out)
        for (int32_t i = lane; i < req_len[r]; i += 32) a.slot_out[t0 + i] = -1;
      continue;
    }
    const int32_t nblk = req_nblk[r];
    if (nblk == 0) continue;
    const int32_t start = start_pos[r];
    const int32_t fb = start / a.B;            // first logical block
    const int32_t g0 = req_blk0[r];
    // Block bi >= 1 starts at segment index (fb + bi) * B - start, block 0
    // at 0; in a valid request every fact has a length >= 1, so seg[] rises
    // strictly over [j0, j1).
    if constexpr (SMEM) {
      // Lanes over blocks: the block's first fact is the last j with seg[j]
      // <= its first index (binary search in shared memory); a warp writes
      // consecutive descriptors.
      // Four blocks per lane per round; their table entries are loaded first,
      // so the loads are in flight together and overlap the searches.
      constexpr int PB = 4;
      for (int32_t base = lane; base < nblk; base += 32 * PB) {
        int32_t phys[PB];
#pragma unroll
        for (int q = 0; q < PB; ++q) {
          const int32_t bi = base + 32 * q;
          phys[q] = bi < nblk ? a.block_tables[(long long)r * a.max_blocks + fb + bi] : 0;
        }
#pragma unroll
        for (int q = 0; q < PB; ++q) {
          const int32_t bi = base + 32 * q;
          if (bi >= nblk) break;
          const int32_t i0 = bi == 0 ? 0 : (fb + bi) * a.B - start;
          int32_t lo = j0, hi = j1 - 1;  // seg[j0] = 0 <= i0
          while (lo < hi) {
            const int32_t mid = (lo + hi + 1) >> 1;
            if (seg[mid] <= i0) lo = mid; else hi = mid - 1;
          }
          BlockDesc d;
          d.r = r;
          d.b = fb + bi;
          d.j = lo;
          d.pad = 0;
          a.desc[g0 + bi] = d;
          check_entry(r, fb + bi, phys[q]);
        }
      }
    } else {
      // Lanes over facts (no dependent L2 reads): fact j [s, e) owns the
      // blocks whose first segment index lies in [s, e).
      const int32_t S = req_len[r];
      for (int32_t base = j0; base < j1; base += 32) {
        const int32_t j = base + lane;
        if (j >= j1) continue;
        const int32_t s = seg[j];
        const int32_t e = j + 1 < j1 ? seg[j + 1] : S;  // exclusive end
        if (e == s) continue;
        int32_t bi_lo = (s + start + a.B - 1) / a.B - fb;
        const int32_t bi_hi = (e + start + a.B - 1) / a.B - fb;  // exclusive
        if (s == 0) bi_lo = 0;
        for (int32_t bi = max(bi_lo, 0); bi < bi_hi && bi < nblk; ++bi) {
          BlockDesc d;
          d.r = r;
          d.b = fb + bi;
          d.j = j;
          d.pad = 0;
          a.desc[g0 + bi] = d;
          check_entry(r, fb + bi, a.block_tables[(long long)r * a.max_blocks + fb + bi]);
        }
      }
    }
  }
  // The batch's first error in request order: a request's own error, or,
  // in a valid request, its first block-table entry outside the cache (the
  // inject kernel skips such blocks).
  __syncthreads();
  if (tid == 0 && s_err_key != ~0ull) {
    const int r = int(s_err_key >> 32);
    const int32_t b = int32_t(s_err_key & 0xffffffffull);
    if (req_err[r] != kOk) record_error(a.st, req_err[r], r);
    else record_error(a.st, kErrBadBlock, (long long)r * a.max_blocks + b);
  }
  if (tid == 0) mirror_status(a.st, a.st_mirror);
}

// -------------------------------------------------------------- inject kernel

struct InjectArgs {
  const uint16_t* k_store;   // [L][H][T_cap][D]
  const uint16_t* v_store;
  int64_t plane;             // T_cap * D  (elements between (l,h) planes)
  const int64_t* fact_off;   // store token offset of each fact
  const int32_t* fact_len;
  const double* inv_freq;    // [D/2]
  int32_t L, H;
  const int32_t* req_off;
  const int32_t* fact_ids;
  const int32_t* start_pos;
  const int32_t* block_tables;
  int32_t max_blocks;
  uint16_t* k_cache;
  uint16_t* v_cache;
  int64_t ls, bs, ts, hs;    // cache strides (elements)
  int32_t num_blocks, B;
  int32_t vec_order;         // 0: (slot, head) rows, 1: (head, slot) rows
  int32_t fact_len_count;    // number of facts (small-batch kernel's id check)
  int64_t* slot_out;
  const int32_t* seg;
  const long long* req_tok0;
  const BlockDesc* desc;
  PlanHeader* hdr;
  DevStatus* st;
  DevStatus* st_mirror;      // optional: see mirror_status
  // host tier only: the arenas above are device-mapped pinned host memory,
  // and facts with hot_off[f] >= 0 are also held in these HBM arenas
  const uint16_t* k_hot;     // [L][H][hot_cap][D]
  const uint16_t* v_hot;
  int64_t hot_plane;         // hot_cap * D
  const int64_t* hot_off;    // [num_facts], -1 when the fact is not in HBM
  // least-recently-used hot set, promotion fused into the batch: facts with
  // pend[f] >= 0 are read from host memory as cold ones and their rows are
  // also written to hot tokens [pend[f], pend[f] + len) of these (the hot)
  // arenas; pend == nullptr: no promotion in this batch
  const int64_t* pend;
  uint16_t* k_prom;
  uint16_t* v_prom;
  // fact-sharded view (per-slot source variant; shard_k == nullptr: none):
  // fact f's rows sit in arena fact_shard[f] ([L][H][plane][D], this GPU's
  // or a peer's memory) at token fact_off[f]
  const uint16_t* const* shard_k;  // [num_shards]
  const uint16_t* const* shard_v;
  const int64_t* shard_plane;      // elements between (l,h) planes of each arena
  const int32_t* fact_shard;       // [num_facts]
};

// Streaming 16-byte accesses: every store row is read once per batch and
// every cache row written once, so neither is kept in L1; stores are marked
// evict-first.  (IS_LOAD_HINT / IS_STORE_HINT select other forms when tuning.)
#ifndef IS_LOAD_HINT
#define IS_LOAD_HINT 0
#endif
#ifndef IS_STORE_HINT
#define IS_STORE_HINT 0
#endif
__device__ __forceinline__ uint4 ld_stream(const uint16_t* p) {
  uint4 v;
#if IS_LOAD_HINT == 2
  asm volatile("ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
#else
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
#endif
  return v;
}

__device__ __forceinline__ void st_stream(uint16_t* p, const uint4& v) {
#if IS_STORE_HINT == 1
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
#else
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
#endif
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Index (in float2 units) of the cos/sin entry of frequency i for in-block
// token o, laid out so that the lanes of one row read consecutive 16-byte
// words (no shared-memory bank conflicts):
//   rotate-half: vector c' = i / 8 of a half row, element e = i % 8
//                float4 index (o * 4 + e / 2) * (D / 16) + c', half e % 2
//   interleaved: vector c = i / 4, pair m = i % 4
//                float4 index (o * 2 + m / 2) * (D / 8) + c, half m % 2
template <int D, int STYLE>
__device__ __forceinline__ int cs_index(int o, int i) {
  if (STYLE == 0) {
    const int cp = i >> 3, e = i & 7;
    return (((o * 4 + (e >> 1)) * (D / 16) + cp) << 1) + (e & 1);
  } else {
    const int c = i >> 2, m = i & 3;
    return (((o * 2 + (m >> 1)) * (D / 8) + c) << 1) + (m & 1);
  }
}

// The cos/sin words one lane needs to rotate its vector c of a key row (the
// table of its token, float4 words as laid out above): rotate-half uses
// t[0..3] (elements 2q, 2q+1 of the half row), interleaved t[0..1].
template <int D, int STYLE>
__device__ __forceinline__ void load_cs(const float4* cs_tok, int c, float4 (&t)[4]) {
  if (STYLE == 0) {
    constexpr int VH = D / 16;
    const int cp = c < VH ? c : c - VH;
#pragma unroll
    for (int q = 0; q < 4; ++q) t[q] = cs_tok[q * VH + cp];
  } else {
    t[0] = cs_tok[c];
    t[1] = cs_tok[D / 8 + c];
    t[2] = t[3] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// Rotate one 16-byte vector (8 bf16) of a key row with its cos/sin words.
//   own: this lane's vector; c: its index in the row (0 .. D/8-1)
template <int D, int STYLE>
__device__ __forceinline__ uint4 rotate_regs(const uint4 own, int c, const float4 (&t)[4]) {
  const uint32_t w[4] = {own.x, own.y, own.z, own.w};
  float x[8];
#pragma unroll
  for (int q = 0; q < 4; ++q) { x[2 * q] = bf_lo(w[q]); x[2 * q + 1] = bf_hi(w[q]); }
  float y[8];
  if (STYLE == 0) {
    // Pair (i, i + D/2): the partner vector sits D/16 lanes away.
    constexpr int VH = D / 16;
    uint32_t pw[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) pw[q] = __shfl_xor_sync(0xffffffffu, w[q], VH);
    float p[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) { p[2 * q] = bf_lo(pw[q]); p[2 * q + 1] = bf_hi(pw[q]); }
    const bool first = c < VH;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float s0 = first ? -t[q].y : t[q].y, s1 = first ? -t[q].w : t[q].w;
      // first half:  x cos - partner sin;  second half: x cos + partner sin
      y[2 * q] = fmaf(x[2 * q], t[q].x, p[2 * q] * s0);
      y[2 * q + 1] = fmaf(x[2 * q + 1], t[q].z, p[2 * q + 1] * s1);
    }
  } else {
    // Pairs (2m, 2m+1) inside the vector.
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int a0 = 4 * h, a1 = 4 * h + 2;
      y[a0] = fmaf(x[a0], t[h].x, -(x[a0 + 1] * t[h].y));
      y[a0 + 1] = fmaf(x[a0 + 1], t[h].x, x[a0] * t[h].y);
      y[a1] = fmaf(x[a1], t[h].z, -(x[a1 + 1] * t[h].w));
      y[a1 + 1] = fmaf(x[a1 + 1], t[h].z, x[a1] * t[h].w);
    }
  }
  uint4 out;
  out.x = pack_bf16(y[0], y[1]);
  out.y = pack_bf16(y[2], y[3]);
  out.z = pack_bf16(y[4], y[5]);
  out.w = pack_bf16(y[6], y[7]);
  return out;
}

// Packed fp32 pairs: sm_100's two-lane fp32 multiply and fused multiply-add
// (one instruction for two lanes; each lane rounds as its scalar form).
typedef unsigned long long f32x2_t;

__device__ __forceinline__ f32x2_t f2_pack(float lo, float hi) {
  return (f32x2_t)__float_as_uint(lo) | ((f32x2_t)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ f32x2_t f2_from_bf16x2(uint32_t w) { return f2_pack(bf_lo(w), bf_hi(w)); }
__device__ __forceinline__ uint32_t f2_to_bf16x2(f32x2_t v) {
  return pack_bf16(__uint_as_float(uint32_t(v)), __uint_as_float(uint32_t(v >> 32)));
}
__device__ __forceinline__ f32x2_t f2_mul(f32x2_t a, f32x2_t b) {
  f32x2_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2_t f2_fma(f32x2_t a, f32x2_t b, f32x2_t c) {
  f32x2_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// cos and sin of 8 consecutive frequencies as packed pairs.
struct CsPairs {
  f32x2_t c[4], s[4];
};

// The rotate-half cos/sin words of frequencies 8c .. 8c+7 (table of one
// token, as load_cs reads them for vector c < D/16), packed in pairs.
template <int D>
__device__ __forceinline__ void load_cs_pairs(const float4* cs_tok, int c, CsPairs& p) {
  float4 t[4];
  load_cs<D, 0>(cs_tok, c, t);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    p.c[q] = f2_pack(t[q].x, t[q].z);
    p.s[q] = f2_pack(t[q].y, t[q].w);
  }
}

// Rotate-half, both halves in one thread: a holds elements 8c .. 8c+7 of a
// key row and b elements D/2 + 8c .. D/2 + 8c+7, which pair with them and
// share their frequencies:  a' = a cos - b sin,  b' = b cos + a sin.  The
// cross product is rounded before the fused multiply-add, as in rotate_regs,
// so both give the same bits (-b is b with its bf16 sign bits flipped, and
// (-b) sin rounds to exactly -(b sin)).
__device__ __forceinline__ void rotate_half_pair(uint4& a, uint4& b, const CsPairs& p) {
  uint32_t wa[4] = {a.x, a.y, a.z, a.w};
  uint32_t wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const f32x2_t x = f2_from_bf16x2(wa[q]);
    const f32x2_t y = f2_from_bf16x2(wb[q]);
    const f32x2_t ny = f2_from_bf16x2(wb[q] ^ 0x80008000u);
    wa[q] = f2_to_bf16x2(f2_fma(x, p.c[q], f2_mul(ny, p.s[q])));
    wb[q] = f2_to_bf16x2(f2_fma(y, p.c[q], f2_mul(x, p.s[q])));
  }
  a = make_uint4(wa[0], wa[1], wa[2], wa[3]);
  b = make_uint4(wb[0], wb[1], wb[2], wb[3]);
}

template <int D, int STYLE>
__device__ __forceinline__ uint4 rotate_vec(const uint4 own, int c, const float4* cs_tok) {
  float4 t[4];
  load_cs<D, STYLE>(cs_tok, c, t);
  return rotate_regs<D, STYLE>(own, c, t);
}

// cos and sin of an fp64 RoPE angle, each the fp32 rounding of the fp64
// value (to within ~1e-15), so small ones are as accurate relatively as large
// ones: a key element near 0 rotates to its partner times the sine exactly as
// the oracle rounds it.  The angle is reduced to r in [-pi/4, pi/4] and a
// quadrant q, ang = q * pi/2 + r, by Cody and Waite's additive reduction in
// fp64 (pi/2 split into the nearest double and its remainder; each product is
// exact inside its fused multiply-add; exact to < 1e-15 rad for positions
// below 2^31).  sin r and cos r are their Taylor series through r^13 and r^14
// (the first neglected terms are below 3e-14 on [-pi/4, pi/4]) by Horner's
// rule in fp64, then the quadrant swaps and negates: sin(q pi/2 + r) = sin r,
// cos r, -sin r, -cos r for q = 0..3, cos alike shifted by one.
__device__ __forceinline__ void rope_cos_sin(double ang, float& c, float& s) {
  constexpr double kTwoOverPi = 0.63661977236758134307553505349005745;
  constexpr double kPiOver2Hi = 1.5707963267948965579989817342720925;   // nearest double to pi/2
  constexpr double kPiOver2Lo = 6.1232339957367660359e-17;               // pi/2 - kPiOver2Hi
  const double k = rint(ang * kTwoOverPi);
  const double r = fma(-k, kPiOver2Lo, fma(-k, kPiOver2Hi, ang));
  const double z = r * r;
  // sin r = r (1 - z/3! + z^2/5! - ... + z^6/13!)
  double ps = 1.0 / 6227020800.0;
  ps = fma(ps, z, -1.0 / 39916800.0);
  ps = fma(ps, z, 1.0 / 362880.0);
  ps = fma(ps, z, -1.0 / 5040.0);
  ps = fma(ps, z, 1.0 / 120.0);
  ps = fma(ps, z, -1.0 / 6.0);
  ps = fma(ps, z, 1.0);
  // cos r = 1 - z/2! + z^2/4! - ... - z^7/14!
  double pc = -1.0 / 87178291200.0;
  pc = fma(pc, z, 1.0 / 479001600.0);
  pc = fma(pc, z, -1.0 / 3628800.0);
  pc = fma(pc, z, 1.0 / 40320.0);
  pc = fma(pc, z, -1.0 / 720.0);
  pc = fma(pc, z, 1.0 / 24.0);
  pc = fma(pc, z, -0.5);
  pc = fma(pc, z, 1.0);
  const float sr = float(r * ps), cr = float(pc);
  const int q = int((long long)k & 3);
  s = (q == 0) ? sr : (q == 1) ? cr : (q == 2) ? -sr : -cr;
  c = (q == 0) ? cr : (q == 1) ? -sr : (q == 2) ? -cr : sr;
}

constexpr int kMaxBlockSize = 128;

// x / d and x % d for a divisor fixed per launch: shifts when d is a power
// of two (POW2), plain division otherwise.
template <bool POW2>
struct Divisor {
  int d, sh;
  __device__ __forceinline__ int div(int x) const { return POW2 ? (x >> sh) : x / d; }
  __device__ __forceinline__ int mod(int x) const { return POW2 ? (x & (d - 1)) : x % d; }
};

__device__ __forceinline__ int ilog2(int x) { return 31 - __clz(x); }
__host__ __device__ constexpr int clog2(int x) { return x <= 1 ? 0 : 1 + clog2(x / 2); }

// Vector order inside one layer of a block (rem = the vector's index in the
// layer; a head row is D/8 consecutive vectors, so rotate-half partners stay
// in one warp).  Sets the slot o and hv = head * D/8 + word.
//   order 0: rows in (slot, head) order, head fastest;
//   order 1: rows in (head, slot) order, slot fastest.
// The launch picks the order whose fastest row index has the larger cache
// stride, so the rows a wave of threads writes are spread over the block's
// run of the cache while each head plane of the store is still read in
// runs of consecutive rows (measured on B200: 97.6% vs 96.0% of the copy
// peak on the token-major cache, 98.7% vs 96.2% on the head-major cache).
template <bool POW2>
__device__ __forceinline__ void split_vec(int rem, int order, const Divisor<POW2>& by_row,
                                          const Divisor<POW2>& by_hrow, int vpr, int log_vpr,
                                          int& o, int& hv) {
  if (order == 0) {
    o = by_row.div(rem);
    hv = by_row.mod(rem);
  } else {
    const int h = by_hrow.div(rem), r2 = by_hrow.mod(rem);
    o = r2 >> log_vpr;
    hv = (h << log_vpr) + (r2 & (vpr - 1));
  }
}

constexpr int kMaxHalfDim = 128;  // D / 2 for the largest head_dim (256)

// Shared-memory state of a CTA of the inject kernels, reused unit after unit.
template <bool HOST_TIER>
struct UnitShared {
  double inv_freq[kMaxHalfDim];  // the store's RoPE frequencies, loaded once per CTA
  long long src[kMaxBlockSize];  // store token of each in-block slot (-1: none)
  // per-slot sources (host tier, sharded view): K/V row bases (token offset
  // applied) and plane stride
  const uint16_t* kb[HOST_TIER ? kMaxBlockSize : 1];
  const uint16_t* vb[HOST_TIER ? kMaxBlockSize : 1];
  long long pl[HOST_TIER ? kMaxBlockSize : 1];
  // host tier, fused promotion: hot-arena row bases that also receive the
  // slot's stored K and V rows (nullptr: none); plane stride a.hot_plane
  uint16_t* pk[HOST_TIER ? kMaxBlockSize : 1];
  uint16_t* pv[HOST_TIER ? kMaxBlockSize : 1];
};

// One work unit: cache block b (logical, of request r) x (layer, head) rows
// [w0, w1), row w = layer * H + head (the copy loop FAST == 0 takes whole
// layers only: w0 and w1 multiples of H).
// j is the CSR index of the first fact with a token in the block, seg[] the
// facts' segment offsets (global or shared memory), j1 the end of the
// request's CSR range, len_r its segment length, tok0 its first slot-mapping
// index.  The slot mapping is written when write_slots.  jfid / joff, when
// given (shared memory), hold each CSR entry's fact id and store offset, so
// the slot walk reads no global memory.  Vector order inside
// a layer: split_vec.  Every thread of the CTA calls this with the same
// arguments; the caller puts a barrier between units.
template <int D, int STYLE, int NT, int VPT, bool POW2, bool HOST_TIER, int HC, int BC, int FAST>
__device__ __forceinline__ void run_unit(const InjectArgs& a, UnitShared<HOST_TIER>& sm,
                                         float4* s_cs4, int r, int b, int j_first,
                                         const int32_t* seg, int j1, int start, int len_r,
                                         long long tok0, int w0, int w1, bool write_slots,
                                         const int32_t* jfid = nullptr, const long long* joff = nullptr) {
  constexpr int VPR = D / 8;  // 16-byte vectors per head row
  constexpr int LOG_VPR = (VPR == 4) ? 2 : (VPR == 8) ? 3 : (VPR == 16) ? 4 : 5;
  const int tid = threadIdx.x;
  // HC / BC > 0: the KV head count / block size are compile-time constants
  // (the common model shapes), which folds the per-vector index arithmetic.
  const int B = BC > 0 ? BC : a.B;
  const int H = HC > 0 ? HC : a.H;
  const int row_vecs = H * VPR;         // vectors per token (all heads)
  const int vecs_layer = B * row_vecs;  // vectors per block and layer
  const Divisor<POW2> by_layer{vecs_layer, POW2 ? (BC > 0 && HC > 0 ? clog2(BC * HC * VPR) : ilog2(vecs_layer)) : 0};
  const Divisor<POW2> by_row{row_vecs, POW2 ? (HC > 0 ? clog2(HC * VPR) : ilog2(row_vecs)) : 0};
  const Divisor<POW2> by_hrow{B * VPR, POW2 ? (BC > 0 ? clog2(BC * VPR) : ilog2(B * VPR)) : 0};
  const int order = a.vec_order;
  long long* s_src = sm.src;
  const uint16_t** s_kb = sm.kb;
  const uint16_t** s_vb = sm.vb;
  long long* s_pl = sm.pl;
  uint16_t** s_pk = sm.pk;
  uint16_t** s_pv = sm.pv;

  const int blk_pos = b * B;                         // position of in-block slot 0
  const int o_lo = max(start - blk_pos, 0);
  const int o_hi = min(start + len_r - blk_pos, B);  // exclusive
  const int phys = a.block_tables[(long long)r * a.max_blocks + b];
  const bool phys_ok = phys >= 0 && phys < a.num_blocks;

  // Store token of each in-block slot: walk forward from the block's first
  // fact (facts cover consecutive segment ranges).
  if (tid < B) {
    const int o = tid;
    long long src = -1;
    if (HOST_TIER) s_pk[o] = s_pv[o] = nullptr;
    if (o >= o_lo && o < o_hi) {
      const int i = blk_pos + o - start;  // segment index
      int j = j_first;
      while (j + 1 < j1 && seg[j + 1] <= i) ++j;
      const int f = jfid ? jfid[j] : a.fact_ids[j];
      const int t = i - seg[j];
      src = (joff ? joff[j] : a.fact_off[f]) + t;
      if (HOST_TIER && a.shard_k) {
        const int sh = a.fact_shard[f];
        s_kb[o] = a.shard_k[sh] + src * D;
        s_vb[o] = a.shard_v[sh] + src * D;
        s_pl[o] = a.shard_plane[sh];
      } else if (HOST_TIER) {
        const long long ho = a.hot_off[f];
        if (ho >= 0) {
          s_kb[o] = a.k_hot + (ho + t) * D;
          s_vb[o] = a.v_hot + (ho + t) * D;
          s_pl[o] = a.hot_plane;
        } else {
          s_kb[o] = a.k_store + src * D;
          s_vb[o] = a.v_store + src * D;
          s_pl[o] = a.plane;
          const long long pd = a.pend ? a.pend[f] : -1;
          if (pd >= 0) {
            s_pk[o] = a.k_prom + (pd + t) * D;
            s_pv[o] = a.v_prom + (pd + t) * D;
          }
        }
      }
      if (write_slots && a.slot_out) a.slot_out[tok0 + i] = phys_ok ? (long long)phys * B + o : -1;
    }
    s_src[o] = src;
  }
  // cos/sin of every (slot, frequency) of the block: fp64 angle, fp32 values.
  auto fill_cs = [&]() {
    for (int e = tid; e < B * (D / 2); e += NT) {
      const int o = e / (D / 2), i = e % (D / 2);
      float cn, sn;
      rope_cos_sin(double(blk_pos + o) * sm.inv_freq[i], cn, sn);
      reinterpret_cast<float2*>(s_cs4)[cs_index<D, STYLE>(o, i)] = make_float2(cn, sn);
    }
  };
  // A block-table entry outside the cache: nothing is stored (uniform; the
  // caller's barrier follows).  The plan reports it.
  auto bad_block = [&]() {};
  if constexpr (FAST == 0) {
    fill_cs();  // before the block-table entry is checked, so its load overlaps
    if (!phys_ok) return bad_block();
    __syncthreads();
  } else {
    // The per-thread loops issue their first loads (which need only the
    // slots' sources), then fill the table while those loads are in flight.
    __syncthreads();
  }

  // FAST: compile-time H and B with one head's block row of vectors (B * D/8)
  // equal to the CTA, slot-fastest rows (token-major cache; the launch picks
  // FAST only for vector order 1).  Each thread then owns one (slot o, word
  // c) for every head and layer of the unit: its source row and plane stride
  // (the store's, or the slot's own with per-slot sources), cache address
  // and cos/sin words are set up once per unit, and each vector costs one
  // plane step.
  if constexpr (FAST == 2) {
    // FAST == 2 (rotate-half, device tier): the CTA is (row parity) x (slot
    // o) x (half-row word c); each thread owns words c and c + D/16 of its
    // slot -- the two halves that rotate together -- for every other (layer,
    // head) row of the unit: no partner exchange, packed fp32 pair
    // arithmetic, 14% fewer instructions.  A warp instruction still covers
    // whole 128-byte half rows, and the CTA writes two heads' rows at once.
    // (Per-slot sources keep the loop below: their extra per-slot state
    // does not fit the registers.)
    static_assert(STYLE == 0 && !HOST_TIER, "paired loop: rotate-half, device tier");
    static_assert(HC > 0 && BC > 0 && BC * VPR == NT, "fast path shape");
    constexpr int VH = VPR / 2;   // 16-byte words per half row
    constexpr int HALF = D / 2;   // elements per half row
    const int rp = tid / (NT / 2);
    const int o = (tid % (NT / 2)) / VH, c = tid % VH;
    const long long src = s_src[o];
    const bool act = src >= 0;
    CsPairs cp;  // loaded once the table is filled
    const long long pl = a.plane;
    const uint16_t* kp = a.k_store + (act ? src : 0) * D + c * 8 + (long long)(w0 + rp) * pl;
    const uint16_t* vp = a.v_store + (act ? src : 0) * D + c * 8 + (long long)(w0 + rp) * pl;
    uint16_t* kd = a.k_cache + (long long)phys * a.bs + (long long)o * a.ts + c * 8;
    uint16_t* vd = a.v_cache + (long long)phys * a.bs + (long long)o * a.ts + c * 8;
    const int nr = (w1 - w0 - rp + 1) / 2;  // rows w0 + 2i + rp, i < nr
    constexpr int HR = IS_PIPELINE ? VPT / 4 : VPT / 2;  // rows per stage, 4 vectors each
    auto load_r = [&](uint4 (&ka)[HR], uint4 (&kb)[HR], uint4 (&va)[HR], uint4 (&vb)[HR], int i0) {
#pragma unroll
      for (int q = 0; q < HR; ++q) {
        const int i = i0 + q;
        ka[q] = kb[q] = va[q] = vb[q] = make_uint4(0, 0, 0, 0);
        if (act && i < nr) {
          const long long so = (long long)(2 * i) * pl;
          ka[q] = ld_stream(kp + so);
          kb[q] = ld_stream(kp + so + HALF);
          va[q] = ld_stream(vp + so);
          vb[q] = ld_stream(vp + so + HALF);
        }
      }
    };
    auto store_r = [&](uint4 (&ka)[HR], uint4 (&kb)[HR], const uint4 (&va)[HR], const uint4 (&vb)[HR],
                       int i0) {
#pragma unroll
      for (int q = 0; q < HR; ++q) {
        const int i = i0 + q;
        rotate_half_pair(ka[q], kb[q], cp);
        if (act && i < nr) {
          const int w = w0 + 2 * i + rp;
          const int l = w / HC, h = w % HC;
          const long long off = (long long)l * a.ls + (long long)h * a.hs;
          st_stream(kd + off, ka[q]);
          st_stream(kd + off + HALF, kb[q]);
          st_stream(vd + off, va[q]);
          st_stream(vd + off + HALF, vb[q]);
        }
      }
    };
#if IS_PIPELINE
    uint4 k0[HR], k1[HR], v0[HR], v1[HR], k2[HR], k3[HR], v2[HR], v3[HR];
    if (nr > 0) load_r(k0, k1, v0, v1, 0);
    fill_cs();
    __syncthreads();
    if (!phys_ok) return bad_block();
    load_cs_pairs<D>(s_cs4 + o * (D / 4), c, cp);
    for (int i0 = 0; i0 < nr; i0 += 2 * HR) {
      if (i0 + HR < nr) load_r(k2, k3, v2, v3, i0 + HR);
      store_r(k0, k1, v0, v1, i0);
      if (i0 + HR >= nr) break;
      if (i0 + 2 * HR < nr) load_r(k0, k1, v0, v1, i0 + 2 * HR);
      store_r(k2, k3, v2, v3, i0 + HR);
    }
#else
    fill_cs();
    __syncthreads();
    if (!phys_ok) return bad_block();
    load_cs_pairs<D>(s_cs4 + o * (D / 4), c, cp);
    for (int i0 = 0; i0 < nr; i0 += HR) {
      uint4 k0[HR], k1[HR], v0[HR], v1[HR];
      load_r(k0, k1, v0, v1, i0);
      store_r(k0, k1, v0, v1, i0);
    }
#endif
  } else if constexpr (FAST == 1) {
    static_assert(HC > 0 && BC > 0 && BC * VPR == NT, "fast path shape");
    {
      const int o = tid / VPR, c = tid % VPR;
      const long long src = s_src[o];
      const bool act = src >= 0;
      float4 cs[4];  // loaded once the table is filled
      const uint16_t* krow;
      const uint16_t* vrow;
      long long pl;
      uint16_t* pkp = nullptr;  // fused promotion: this slot's hot rows
      uint16_t* pvp = nullptr;
      if constexpr (HOST_TIER) {
        krow = act ? s_kb[o] : a.k_store;
        vrow = act ? s_vb[o] : a.v_store;
        pl = act ? s_pl[o] : 0;
        if (act && s_pk[o] != nullptr) {
          pkp = s_pk[o] + c * 8 + (long long)w0 * a.hot_plane;
          pvp = s_pv[o] + c * 8 + (long long)w0 * a.hot_plane;
        }
      } else {
        krow = a.k_store + (act ? src : 0) * D;
        vrow = a.v_store + (act ? src : 0) * D;
        pl = a.plane;
      }
      const uint16_t* kp = krow + c * 8 + (long long)w0 * pl;
      const uint16_t* vp = vrow + c * 8 + (long long)w0 * pl;
      uint16_t* kd = a.k_cache + (long long)phys * a.bs + (long long)o * a.ts + c * 8;
      uint16_t* vd = a.v_cache + (long long)phys * a.bs + (long long)o * a.ts + c * 8;
      const int nw = w1 - w0;  // (layer, head) rows of this thread, in plane order
      constexpr int HW = IS_PIPELINE ? VPT / 2 : VPT;
      // (stage rows s0 + q of the unit; w0 is the unit's first row)
      auto load_w = [&](uint4 (&kv)[HW], uint4 (&vv)[HW], int s0) {
#pragma unroll
        for (int q = 0; q < HW; ++q) {
          const int w = s0 + q;
          kv[q] = make_uint4(0, 0, 0, 0);
          vv[q] = kv[q];
          if (act && w < nw) {
            kv[q] = ld_stream(kp + (long long)w * pl);
            vv[q] = ld_stream(vp + (long long)w * pl);
          }
        }
      };
      auto store_w = [&](const uint4 (&kv)[HW], const uint4 (&vv)[HW], int s0) {
#pragma unroll
        for (int q = 0; q < HW; ++q) {
          const int w = s0 + q;
          const uint4 kr = rotate_regs<D, STYLE>(kv[q], c, cs);
          if (act && w < nw) {
            const int l = (w0 + w) / HC, h = (w0 + w) % HC;
            const long long off = (long long)l * a.ls + (long long)h * a.hs;
            st_stream(kd + off, kr);
            st_stream(vd + off, vv[q]);
            if (HOST_TIER && pkp != nullptr) {  // the stored rows, unrotated
              st_stream(pkp + (long long)w * a.hot_plane, kv[q]);
              st_stream(pvp + (long long)w * a.hot_plane, vv[q]);
            }
          }
        }
      };
#if IS_PIPELINE
      uint4 ka[HW], va[HW], kb[HW], vb[HW];
      if (nw > 0) load_w(ka, va, 0);
      fill_cs();
      __syncthreads();
      if (!phys_ok) return bad_block();
      load_cs<D, STYLE>(s_cs4 + o * (D / 4), c, cs);
      for (int s0 = 0; s0 < nw; s0 += 2 * HW) {
        if (s0 + HW < nw) load_w(kb, vb, s0 + HW);
        store_w(ka, va, s0);
        if (s0 + HW >= nw) break;
        if (s0 + 2 * HW < nw) load_w(ka, va, s0 + 2 * HW);
        store_w(kb, vb, s0 + HW);
      }
#else
      fill_cs();
      __syncthreads();
      if (!phys_ok) return bad_block();
      load_cs<D, STYLE>(s_cs4 + o * (D / 4), c, cs);
      for (int s0 = 0; s0 < nw; s0 += HW) {
        uint4 kv[HW], vv[HW];
        load_w(kv, vv, s0);
        store_w(kv, vv, s0);
      }
#endif
    }
  } else {
    const int l0 = w0 / H, l1 = w1 / H;  // whole layers
    const int total = (l1 - l0) * vecs_layer;
    const uint16_t* kst = a.k_store;
    const uint16_t* vst = a.v_store;
    constexpr int HV = IS_PIPELINE ? VPT / 2 : VPT;  // vectors per thread per stage

    // One stage: vectors base + q*NT + tid, q < HV, of the unit's flat range.
    auto load_stage = [&](uint4 (&kv)[HV], uint4 (&vv)[HV], int base) {
#pragma unroll
      for (int q = 0; q < HV; ++q) {
        const int v = base + q * NT + tid;
        const int l = l0 + by_layer.div(v);
        const int rem = by_layer.mod(v);
        int o, hv;
        split_vec<POW2>(rem, order, by_row, by_hrow, VPR, LOG_VPR, o, hv);
        const long long src = v < total ? s_src[o] : -1;
        kv[q] = make_uint4(0, 0, 0, 0);
        vv[q] = kv[q];
        if (src >= 0) {
          if (HOST_TIER) {
            const long long so = (long long)(l * H + (hv >> LOG_VPR)) * s_pl[o] + (hv & (VPR - 1)) * 8;
            kv[q] = ld_stream(s_kb[o] + so);
            vv[q] = ld_stream(s_vb[o] + so);
          } else {
            const long long so = (long long)(l * H + (hv >> LOG_VPR)) * a.plane + src * D +
                                 (hv & (VPR - 1)) * 8;
            kv[q] = ld_stream(kst + so);
            vv[q] = ld_stream(vst + so);
          }
        }
      }
    };
    auto store_stage = [&](const uint4 (&kv)[HV], const uint4 (&vv)[HV], int base) {
#pragma unroll
      for (int q = 0; q < HV; ++q) {
        const int v = base + q * NT + tid;
        const int l = l0 + by_layer.div(v);
        const int rem = by_layer.mod(v);
        int o, hv;
        split_vec<POW2>(rem, order, by_row, by_hrow, VPR, LOG_VPR, o, hv);
        if (v >= total) o = 0;
        const int c = hv & (VPR - 1);
        const uint4 kr = rotate_vec<D, STYLE>(kv[q], c, s_cs4 + o * (D / 4));
        if (v < total && s_src[o] >= 0) {
          const long long dst = (long long)l * a.ls + (long long)phys * a.bs + (long long)o * a.ts +
                                (long long)(hv >> LOG_VPR) * a.hs + c * 8;
          st_stream(a.k_cache + dst, kr);
          st_stream(a.v_cache + dst, vv[q]);
          if (HOST_TIER && s_pk[o] != nullptr) {  // fused promotion: the stored rows
            const long long hso = (long long)(l * H + (hv >> LOG_VPR)) * a.hot_plane + c * 8;
            st_stream(s_pk[o] + hso, kv[q]);
            st_stream(s_pv[o] + hso, vv[q]);
          }
        }
      }
    };

#if IS_PIPELINE
    // Two stages in flight: the next stage's loads are issued before the
    // current stage is rotated and stored (stage control is uniform).
    const int step = NT * HV;
    uint4 ka[HV], va[HV], kb[HV], vb[HV];
    if (total > 0) load_stage(ka, va, 0);
    for (int base = 0; base < total; base += 2 * step) {
      if (base + step < total) load_stage(kb, vb, base + step);
      store_stage(ka, va, base);
      if (base + step >= total) break;
      if (base + 2 * step < total) load_stage(ka, va, base + 2 * step);
      store_stage(kb, vb, base + step);
    }
#else
    for (int base = 0; base < total; base += NT * HV) {
      uint4 kv[HV], vv[HV];
      load_stage(kv, vv, base);
      store_stage(kv, vv, base);
    }
#endif
  }
}

// Persistent gather-rotate-scatter kernel.  Work unit u covers global block
// gb = u % total_blocks and rows [lg * rpu, min(L * H, (lg + 1) * rpu)),
// lg = u / total_blocks, so CTAs running side by side read neighbouring
// tokens of the same layers.  Units are taken from an atomic counter; the
// next unit is fetched while the current one is copied.  POW2: H and B are
// powers of two (all index splits are shifts).  HOST_TIER: the source of
// every slot is chosen per fact — the store lives in pinned host memory read
// over the host link, except the facts that also sit in the HBM hot arenas;
// or, with a sharded view, facts live in several stores' arenas (peer GPUs'
// memory read over NVLink, or this GPU's).
template <int D, int STYLE, int NT, int VPT, int MINB, bool POW2, bool HOST_TIER, int HC = 0, int BC = 0,
          int FAST = 0>
__global__ void __launch_bounds__(NT, MINB) inject_kernel(InjectArgs a) {
  extern __shared__ float4 s_cs4[];  // [B * D/4] cos/sin of the block
  __shared__ UnitShared<HOST_TIER> sm;
  __shared__ int s_unit;

  const int tid = threadIdx.x;
  for (int i = tid; i < D / 2; i += NT) sm.inv_freq[i] = a.inv_freq[i];  // store data, not the plan's
  // When launched as a programmatic dependent of the plan kernel, wait here
  // for its results; without such a launch this returns at once.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int total_units = a.hdr->total_units;
  const int total_blocks = a.hdr->total_blocks;
  const int rpu = a.hdr->rows_per_unit;

  // Unit blockIdx.x first (no CTA waits on the counter to start), then
  // gridDim.x + the counter's answer, fetched one unit ahead.
  int next = blockIdx.x;
  unsigned int fetched = ~0u;
  for (;;) {
    __syncthreads();  // the previous unit's tables are no longer read
    if (tid == 0) {
      if (fetched != ~0u) {
        next = fetched < unsigned(total_units) - gridDim.x ? int(gridDim.x + fetched) : total_units;
        fetched = ~0u;
      }
      s_unit = next;
      if (next < total_units) fetched = atomicAdd(&a.hdr->next_unit, 1u);
    }
    __syncthreads();
    const int u = s_unit;
    if (u >= total_units) break;
    const int gb = u % total_blocks;
    const int lg = u / total_blocks;
    const BlockDesc d = a.desc[gb];
    const int r = d.r;
    const long long tok0 = a.req_tok0[r];
    const int w0 = lg * rpu;
    run_unit<D, STYLE, NT, VPT, POW2, HOST_TIER, HC, BC, FAST>(a, sm, s_cs4, r, d.b, d.j, a.seg, a.req_off[r + 1],
                                                 a.start_pos[r], int(a.req_tok0[r + 1] - tok0), tok0,
                                                 w0, min(a.L * a.H, w0 + rpu), lg == 0);
  }
}

// Small batches (at most kSmallRequests requests and kSmallIds fact ids):
// one kernel.  Every CTA of the persistent grid composes the batch itself in
// shared memory -- the same definitions as plan_kernel (CSR check, lengths,
// segment offsets, validity, token and block prefixes, work-unit size) --
// and takes unit blockIdx.x, then, when the batch has more than two waves
// of units, units gridDim.x, gridDim.x + 1, ... from the store's counter
// (dynamic, as the inject kernel; up to two waves, blockIdx.x + gridDim.x).
// The counter is zero when a launch starts and is fetched exactly once per
// unit (each unit a CTA takes makes it fetch the next; the fetch after a
// CTA's last unit returns one past the end), so the fetch that returns
// total_units - 1 is the launch's last and its CTA sets the counter back to
// zero (batches on one store run one at a time).  The last CTA (the one a small batch leaves without units) alone
// records the batch's errors and writes the -1 slots of invalid requests.
// No work space, no second launch.
constexpr int kSmallRequests = 32;  // one lane of a warp per request
constexpr int kSmallIds = 256;      // one thread per fact id

struct SmallPlan {
  long long off[kSmallIds];    // store token offset per CSR entry (valid ids)
  int32_t fid[kSmallIds];      // fact id per CSR entry
  int32_t len[kSmallIds];      // fact length per CSR entry, -1 for an id outside the store
  int32_t seg[kSmallIds];      // segment offset of each entry inside its request
  int32_t pref[kSmallIds + 1]; // exclusive prefix of valid lengths over the whole batch
  int32_t roff[kSmallRequests + 1];
  int32_t start[kSmallRequests];
  int32_t err[kSmallRequests];
  int32_t nblk[kSmallRequests];
  int32_t blk0[kSmallRequests + 1];
  int32_t total_units, total_blocks, rpu;
  int32_t over;  // over a capacity: the batch writes nothing
};

template <int D, int STYLE, int NT, int VPT, int MINB, bool POW2, bool HOST_TIER, int HC = 0, int BC = 0,
          int FAST = 0>
__global__ void __launch_bounds__(NT, MINB) small_inject_kernel(InjectArgs a, int32_t R, int32_t num_ids,
                                                                int64_t slot_cap, int32_t grid_ctas,
                                                                int32_t max_batch_blocks,
                                                                unsigned int* ctr) {
  static_assert(NT == kSmallIds, "one thread per fact id");
  extern __shared__ float4 s_cs4[];
  __shared__ UnitShared<HOST_TIER> sm;
  __shared__ SmallPlan p;
  __shared__ int32_t s_wsum[NT / 32];
  __shared__ unsigned long long s_err_key;
  __shared__ unsigned int s_bad_ids;  // bit r: request r lists an id outside the store
  __shared__ int s_unit;
  static_assert(kSmallRequests <= 32, "request bit mask and warp-0 lanes");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool reporter = blockIdx.x == gridDim.x - 1;

  // Everything the plan reads from the caller is loaded at once: the CSR,
  // the starts, the ids and right behind them their lengths and store
  // offsets (which need nothing but the id), and the frequencies.
  const int32_t fid = tid < num_ids ? a.fact_ids[tid] : -1;
  if (tid <= R) p.roff[tid] = a.req_off[tid];
  if (tid < R) p.start[tid] = a.start_pos[tid];
  for (int i = tid; i < D / 2; i += NT) sm.inv_freq[i] = a.inv_freq[i];
  const bool id_ok = fid >= 0 && fid < a.fact_len_count;  // false past num_ids
  int32_t len = 0;  // length of this thread's id (0 for an id outside the store)
  if (tid < num_ids) {
    const int32_t lf = id_ok ? a.fact_len[fid] : -1;
    p.off[tid] = id_ok ? a.fact_off[fid] : -1;
    p.fid[tid] = fid;
    p.len[tid] = lf;
    len = id_ok ? lf : 0;
  }
  if (tid == 0) s_bad_ids = 0u;
  // Block size: a shift when it is a power of two.  The plan's sums fit 32
  // bits: the host launches this kernel only when ids x the store's longest
  // fact is below 2^31, and start + segment <= max_blocks * B < 2^31 once
  // checked.
  const int lb = POW2 ? ilog2(a.B) : 0;
  auto div_b = [&](int32_t x) { return POW2 ? (x >> lb) : x / a.B; };
  __syncthreads();
  // The CSR must start at 0, end at num_ids and never decrease (checked
  // with the scan's barrier below; until then nothing leaves shared memory
  // but L2 prefetches of table rows inside the table).
  const bool csr_bad = (tid < R && p.roff[tid + 1] < p.roff[tid]) ||
                       (tid == 0 && (p.roff[0] != 0 || p.roff[R] != num_ids));
  // Warm L2 with the block-table lines of each request's first blocks (up to
  // 128 entries), read later by every unit's slot set-up.
  if (tid < R * 4) {
    const int r = tid >> 2, st0 = p.start[r];
    const int b = (st0 >= 0 ? div_b(st0) : a.max_blocks) + 32 * (tid & 3);
    if (b < a.max_blocks)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(a.block_tables + (long long)r * a.max_blocks + b));
  }
  // Request of the entry at CSR index x (of the block at batch index x):
  // the last request whose first entry (block) is at or before x.
  auto request_of = [&](const int32_t* first, int x) {
    int lo = 0, hi = max(R - 1, 0);
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (first[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  // This id's request; requests holding an id outside the store.
  const int myr = request_of(p.roff, tid);
  if (tid < num_ids && !id_ok) atomicOr(&s_bad_ids, 1u << myr);
  // Exclusive prefix of the lengths over the batch: warp scans, then the
  // warps' totals.
  int32_t x = len;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, x, d);
    if (lane >= d) x += y;
  }
  if (lane == 31) s_wsum[warp] = x;
  if (__syncthreads_or(csr_bad)) {
    if (reporter && tid == 0) {
      record_error(a.st, kErrInvalidArg, -1);
      mirror_status(a.st, a.st_mirror);
    }
    return;
  }
  int32_t ws = lane < NT / 32 ? s_wsum[lane] : 0;
#pragma unroll
  for (int d = 1; d < NT / 32; d <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, ws, d);
    if (lane >= d) ws += y;
  }
  const int32_t wbase = warp > 0 ? __shfl_sync(0xffffffffu, ws, warp - 1) : 0;
  p.pref[tid] = wbase + x - len;
  if (tid == NT - 1) p.pref[NT] = wbase + x;  // so p.pref[num_ids] is the batch total
  __syncthreads();
  // Warp 0, lane r per request: validity, touched blocks and their prefix;
  // lane 0 then sizes the work units.
  if (warp == 0) {
    const int r = lane;
    int32_t err = kOk, nblk = 0;
    if (r < R) {
      const int32_t st0 = p.start[r];
      const int32_t S = p.pref[p.roff[r + 1]] - p.pref[p.roff[r]];
      err = (s_bad_ids >> r) & 1u ? kErrBadFactId : kOk;
      if (err == kOk && st0 < 0) err = kErrInvalidArg;
      if (err == kOk && (long long)st0 + S > (long long)a.max_blocks * a.B) err = kErrPosition;
      if (err == kOk && S > 0) nblk = div_b(st0 + S - 1) - div_b(st0) + 1;
      p.err[r] = err;
      p.nblk[r] = nblk;
    }
    int32_t acc = nblk;  // inclusive prefix over requests
#pragma unroll
    for (int d = 1; d < kSmallRequests; d <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, acc, d);
      if (lane >= d) acc += y;
    }
    if (r < R) p.blk0[r] = acc - nblk;
    const int32_t total = __shfl_sync(0xffffffffu, acc, kSmallRequests - 1);
    if (lane == 0) {
      p.blk0[R] = total;
      const int32_t total_tokens = p.pref[num_ids];
      // the same limits as the two-kernel path, so results never depend on
      // which path a batch takes
      int32_t rpu, upb;
      unit_size(total, a.L, a.H, grid_ctas, FAST != 0, rpu, upb);
      // (work units are counted in 32 bits: a batch needing more is over
      // capacity, as in the two-kernel path)
      const bool over = (a.slot_out != nullptr && total_tokens > slot_cap) || total > max_batch_blocks ||
                        (long long)total * upb > 0x7fffffffLL;
      p.rpu = rpu;
      p.total_blocks = total;
      p.total_units = over ? 0 : total * upb;
      p.over = over;
      // A batch over capacity writes nothing and reports only that.
      if (reporter && over) record_error(a.st, kErrCapacity, total_tokens);
      s_err_key = ~0ull;
    }
  }
  // Segment offsets inside each request.
  if (tid < num_ids) p.seg[tid] = p.pref[tid] - p.pref[p.roff[myr]];
  __syncthreads();
  // -1 slots for the tokens of invalid requests (nothing at all on capacity).
  const bool over_cap = p.over != 0;
  if (reporter && a.slot_out && !over_cap) {
    for (int r = 0; r < R; ++r) {
      if (p.err[r] == kOk) continue;
      const int32_t S = p.pref[p.roff[r + 1]] - p.pref[p.roff[r]];
      for (int32_t i = tid; i < S; i += NT) a.slot_out[p.pref[p.roff[r]] + i] = -1;
    }
  }
  // The batch's first error in request order: a request's own error, or, in
  // a valid request, its first block-table entry outside the cache (units
  // skip such blocks).
  if (reporter && !over_cap) {
    if (tid < R && p.err[tid] != kOk) atomicMin(&s_err_key, (unsigned long long)tid << 32);
    for (int gb = tid; gb < p.total_blocks; gb += NT) {
      const int r = request_of(p.blk0, gb);
      const int b = div_b(p.start[r]) + (gb - p.blk0[r]);
      const int32_t phys = a.block_tables[(long long)r * a.max_blocks + b];
      if (phys < 0 || phys >= a.num_blocks) atomicMin(&s_err_key, ((unsigned long long)r << 32) | unsigned(b));
    }
    __syncthreads();
    if (tid == 0 && s_err_key != ~0ull) {
      const int r = int(s_err_key >> 32);
      const int b = int(s_err_key & 0xffffffffull);
      if (p.err[r] != kOk) record_error(a.st, p.err[r], r);
      else record_error(a.st, kErrBadBlock, (long long)r * a.max_blocks + b);
    }
  }
  if (reporter && tid == 0) mirror_status(a.st, a.st_mirror);  // the batch's errors are in

  const int total_units = p.total_units, total_blocks = p.total_blocks, rpu = p.rpu;
  // Up to two waves the units are strided (u, u + gridDim.x: as balanced as
  // the counter, without 296 CTAs' atomics on one word); beyond, counted.
  const bool counted = total_units > 2 * int(gridDim.x);
  int next = blockIdx.x;  // the first wave is static
  unsigned int fetched = ~0u;  // the counter's answer for the next unit, read one unit later
  for (;;) {
    __syncthreads();  // the previous unit's tables (and s_unit) are no longer read
    if (tid == 0) {
      if (fetched != ~0u) {
        if (fetched == unsigned(total_units) - 1u) atomicExch(ctr, 0u);  // the launch's last fetch
        next = fetched < unsigned(total_units) - gridDim.x ? int(gridDim.x + fetched) : total_units;
        fetched = ~0u;
      }
      s_unit = next;
      if (next < total_units) {
        if (counted) fetched = atomicAdd(ctr, 1u);
        else next += gridDim.x;
      }
    }
    __syncthreads();
    const int u = s_unit;
    if (u >= total_units) break;
    const int gb = u % total_blocks, lg = u / total_blocks;
    const int r = request_of(p.blk0, gb);
    const int start = p.start[r];
    const int b = div_b(start) + (gb - p.blk0[r]);
    const int j0 = p.roff[r], j1 = p.roff[r + 1];
    const int i_first = max(0, b * a.B - start);
    int lo = j0, hi = j1 - 1;  // last fact with seg <= i_first
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.seg[mid] <= i_first) lo = mid; else hi = mid - 1;
    }
    const int w0 = lg * rpu;
    run_unit<D, STYLE, NT, VPT, POW2, HOST_TIER, HC, BC, FAST>(a, sm, s_cs4, r, b, lo, p.seg, j1, start,
                                                 p.pref[j1] - p.pref[j0], p.pref[j0], w0,
                                                 min(a.L * a.H, w0 + rpu), lg == 0, p.fid, p.off);
  }
}

// Host tier, least-recently-used hot set: copy newly promoted facts from the
// pinned (device-mapped) host arenas into their HBM slots.  Promotion i moves
// fact rows [src_tok, src_tok + len) of every (layer, head) plane to rows
// [dst_tok, dst_tok + len) of the hot planes; 16 bytes per thread-step.
struct Promotion {
  long long src_tok;  // token offset in the host planes
  long long dst_tok;  // token offset in the hot planes
  int32_t len;
  int32_t pad;
};

__global__ void promote_kernel(const Promotion* __restrict__ list, int32_t n, int32_t planes,
                               int32_t vec_per_row, const uint16_t* __restrict__ k_host,
                               const uint16_t* __restrict__ v_host, long long host_plane,
                               uint16_t* __restrict__ k_hot, uint16_t* __restrict__ v_hot,
                               long long hot_plane) {
  for (int32_t i = blockIdx.y; i < n; i += gridDim.y) {
    const Promotion pr = list[i];
    const long long per_plane = (long long)pr.len * vec_per_row;
    const long long total = per_plane * planes;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
      const long long p = e / per_plane, r = e % per_plane;
      const long long so = p * host_plane + pr.src_tok * vec_per_row * 8 + r * 8;
      const long long dso = p * hot_plane + pr.dst_tok * vec_per_row * 8 + r * 8;
      *reinterpret_cast<uint4*>(k_hot + dso) = ld_stream(k_host + so);
      *reinterpret_cast<uint4*>(v_hot + dso) = ld_stream(v_host + so);
    }
  }
}

// Hot-table changes: entry pairs (fact, token offset in the hot planes or -1)
// applied to table t0 (n0 pairs) and table t1 (n1 pairs after them).
__global__ void hot_table_kernel(int64_t* __restrict__ t0, int64_t* __restrict__ t1,
                                 const int64_t* __restrict__ pairs, int32_t n0, int32_t n1) {
  const int32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n0) t0[pairs[2 * i]] = pairs[2 * i + 1];
  else if (i < n0 + n1) t1[pairs[2 * i]] = pairs[2 * i + 1];
}

// RoPE frequencies, fp64: inv_freq_i = theta^(-2i/D), optionally with the
// Llama-3.1 wavelength-band rule (wavelength 2 pi / f below orig/high: kept;
// above orig/low: divided by factor; between: blended with weight
// (orig / wavelength - low) / (high - low) on the unscaled frequency).
__global__ void inv_freq_kernel(double* out, int D, double theta, int scaling, double factor,
                                double low, double high, double orig) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= D / 2) return;
  double f = pow(theta, -2.0 * double(i) / double(D));
  if (scaling == 1) {
    const double wl = 2.0 * 3.14159265358979323846 / f;
    if (wl > orig / low) {
      f = f / factor;
    } else if (wl >= orig / high) {
      const double w = (orig / wl - low) / (high - low);
      f = (1.0 - w) * (f / factor) + w * f;
    }
  }
  out[i] = f;
}

}  // namespace isk
