/*
 * inject_store.h -- C-ABI of the B200 retrieve-and-inject library
 * (libinjectstore.so).
 *
 * What it computes follows the online phase of InferScale ("InferScale:
 * GPU-Native KV Injection for Personalized LLM Serving", summaries at
 * gist.science/{ja,nl,it}/paper/2607.27090, technical summary, section
 * "Methodology -- 2. Online phase: Chunked RoPE and KV injection"):
 *
 *   Pre-RoPE storage   keys are captured before RoPE and kept, with the raw
 *                      values, in a fact store on the GPU;
 *   Dynamic rotation   the retrieved facts are composed into one contiguous
 *                      segment and each stored key gets the RoPE rotation of
 *                      its new serving position (Theorem 6: exact);
 *   Injection          the composed K/V are scatter-copied into the paged KV
 *                      cache, so the model prefills only the query tokens.
 *
 * Conventions for every call:
 *   - All functions return IS_OK (0) or a negative IS_ERR_* status and never
 *     abort the process.  Device-side problems found while a batch runs are
 *     recorded on the device and returned by is_last_error().
 *   - Tensors are bf16 (IEEE binary32 upper halves) passed as void*; integer
 *     arrays are int32 or int64 as declared.  "device" pointers must be
 *     addresses on the store's GPU; "host or device" pointers may be either
 *     (unified addressing decides).  No call takes ownership of a caller
 *     array; every array must stay valid until the work on `stream` that
 *     uses it has finished.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 *   - One store must not be used by two batches at the same time: batches on
 *     one store are ordered on one stream, or ordered by the caller.
 *   - Thread safety: a store is not internally locked.
 */
#ifndef INJECT_STORE_H
#define INJECT_STORE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define IS_OK 0
#define IS_ERR_INVALID_ARG (-1)   /* bad pointer, size, geometry or CSR     */
#define IS_ERR_BAD_FACT_ID (-2)   /* a fact id outside [0, num_facts)       */
#define IS_ERR_POSITION (-3)      /* segment runs past the request's table  */
#define IS_ERR_BAD_BLOCK (-4)     /* block-table entry outside the cache    */
#define IS_ERR_CAPACITY (-5)      /* store, batch or slot-output too small  */
#define IS_ERR_OOM (-6)           /* device or pinned allocation failed     */
#define IS_ERR_CUDA (-7)          /* a CUDA runtime call failed             */
#define IS_ERR_TIMEOUT (-8)       /* a bounded host wait ran out            */
#define IS_ERR_NOT_SUPPORTED (-9) /* shape outside what the kernels handle  */

/* ---- configuration ----------------------------------------------------- */
#define IS_ROPE_ROTATE_HALF 0   /* pairs (i, i + D/2): Llama/Mistral/Qwen HF  */
#define IS_ROPE_INTERLEAVED 1   /* pairs (2i, 2i + 1)                         */
#define IS_SCALING_NONE 0
#define IS_SCALING_LLAMA3 1     /* Llama-3.1 wavelength-band frequency rule   */
#define IS_TIER_DEVICE 0        /* whole store in HBM                         */
#define IS_TIER_HOST 1          /* store in pinned host memory + HBM hot set  */

typedef struct {
  int32_t num_layers;        /* L >= 1                                        */
  int32_t num_kv_heads;      /* H >= 1                                        */
  int32_t head_dim;          /* D in {32, 64, 128, 256}                       */
  int32_t rope_style;        /* IS_ROPE_*                                     */
  double rope_theta;         /* base theta > 0; inv_freq_i = theta^(-2i/D)    */
  int32_t rope_scaling;      /* IS_SCALING_*                                  */
  double scale_factor;       /* llama3: factor (8)                            */
  double low_freq_factor;    /* llama3: low (1)                               */
  double high_freq_factor;   /* llama3: high (4)                              */
  int32_t original_max_position; /* llama3: original context (8192)          */
  int64_t capacity_tokens;   /* tokens per (layer, head) plane of the store   */
  int32_t max_facts;         /* fact-id capacity                              */
  int32_t max_batch_requests;/* per-batch request limit (0: 4096)             */
  int32_t max_batch_fact_ids;/* per-batch fact-id limit (0: 1 << 20)          */
  int32_t max_batch_blocks;  /* per-batch touched cache blocks over all
                                requests (0: max(65536, 256 * requests))     */
  int32_t tier;              /* IS_TIER_*                                     */
  int64_t hot_capacity_tokens; /* IS_TIER_HOST: tokens of the HBM hot set     */
} is_store_config_t;

/* Paged KV cache.  Element (layer l, block b, in-block token o, head h,
 * dim d) of K is ((uint16_t*)k_cache)[l*layer_stride + b*block_stride +
 * o*token_stride + h*head_stride + d]; V alike with the same strides.
 * Strides are in elements and multiples of 8; caches 16-byte aligned.
 * [L][num_blocks][B][H][D] (token-major) and [L][num_blocks][H][B][D]
 * (head-major) are both expressible.  Slot s = b*B + o. */
typedef struct {
  void* k_cache;
  void* v_cache;
  int64_t layer_stride;
  int64_t block_stride;
  int64_t token_stride;
  int64_t head_stride;
  int32_t num_blocks;
  int32_t block_size;        /* B in [1, 128]                                 */
} is_cache_t;

typedef struct is_store is_store_t;  /* opaque; owned by the library */

/* ---- store lifetime ---------------------------------------------------- */

/* Create a fact store on `device`.  Pre-RoPE storage (technical summary,
 * Online phase, "Pre-RoPE storage"): K and V arenas, bf16, layout
 * [L][H][capacity_tokens][D] (one token plane per layer and KV head), plus
 * a per-fact offset/length table.  Allocates the arenas (cudaMalloc, or
 * cudaHostAlloc for IS_TIER_HOST), the RoPE frequency table (fp64, computed
 * on the device) and the per-batch work space.  *out receives the store.
 * Errors: INVALID_ARG (null, out-of-range field), NOT_SUPPORTED (head_dim),
 * OOM, CUDA.  Nothing is leaked on error. */
int is_store_create(const is_store_config_t* cfg, int device, is_store_t** out);

/* Free everything the store owns.  Waits for the store's work to finish.
 * A NULL store is ignored. */
void is_store_destroy(is_store_t* store);

/* Append one fact: k_pre and v are bf16 [L][H][len][D] (host or device),
 * the key taken BEFORE RoPE and the raw value (technical summary, Online
 * phase, "Pre-RoPE storage").  The fact gets the next token range of every
 * plane and the next id (ids are dense, in put order).  Synchronous: the
 * caller's buffers may be reused on return.  Errors: INVALID_ARG (null,
 * len <= 0), CAPACITY (tokens or ids exhausted), CUDA. */
int is_store_put_fact(is_store_t* store, const void* k_pre, const void* v, int32_t len,
                      int32_t* fact_id_out);

/* Append one fact from its context-window encoding (technical summary,
 * Offline phase, "Context-Window Encoding": each fact is encoded with a
 * window of w preceding turns and only the fact's KV is kept).  k_pre and v
 * are bf16 [L][H][window_len + fact_len][D] (host or device) -- the pre-RoPE
 * keys and raw values the encoder produced for the window followed by the
 * fact -- and only the last fact_len tokens of every plane are stored.  The
 * window tokens are dropped; positions play no part (keys are pre-RoPE).
 * Synchronous.  Errors as for is_store_put_fact, and INVALID_ARG for
 * window_len < 0. */
int is_store_put_fact_window(is_store_t* store, const void* k_pre, const void* v,
                             int32_t window_len, int32_t fact_len, int32_t* fact_id_out);

/* Number of facts, and a fact's token offset in every plane and length. */
int is_store_num_facts(const is_store_t* store, int32_t* num_facts_out);
int is_store_fact_info(const is_store_t* store, int32_t fact_id, int64_t* offset_out,
                       int32_t* len_out);

/* Copy a stored fact back out as bf16 [L][H][len][D] (host or device
 * destination; synchronous).  Errors: INVALID_ARG, BAD_FACT_ID, CUDA. */
int is_store_read_fact(is_store_t* store, int32_t fact_id, void* k_out, void* v_out);

/* Host tier (IS_TIER_HOST) only: choose the facts whose K/V are also kept in
 * the HBM hot arenas (capacity hot_capacity_tokens per plane), the rest
 * being read from pinned host memory over the host link while a batch runs
 * (technical summary, Results, "Scalability": the KV store can be moved to
 * host DRAM when GPU memory is too small).  fact_ids (host array, n
 * entries; repeats ignored) replaces the previous hot set; the facts are
 * copied in list order.  Waits for the device to go idle first, so no batch
 * reads a half-updated set.  Errors: NOT_SUPPORTED (device tier, or the
 * LRU policy),
 * BAD_FACT_ID, CAPACITY (more tokens than the hot arenas hold; the old set
 * is kept), INVALID_ARG, CUDA. */
int is_store_set_hot(is_store_t* store, const int32_t* fact_ids, int32_t n);

/* Hot-set policy of a host-tier store.
 *   IS_HOT_STATIC  the caller names the hot facts (is_store_set_hot).
 *   IS_HOT_LRU     the hot arenas are cut into slots of slot_tokens tokens;
 *                  is_store_touch (called by is_inject_batch_host for its
 *                  batch) promotes requested cold facts of at most
 *                  slot_tokens tokens into the least recently used slot not
 *                  used by that call, so the batch reads them from HBM.
 * Either way the set starts empty.  Waits for the device to go idle.
 * Errors: NOT_SUPPORTED (device tier), INVALID_ARG, CUDA. */
#define IS_HOT_STATIC 0
#define IS_HOT_LRU 1
int is_store_set_hot_policy(is_store_t* store, int policy, int32_t slot_tokens);

/* IS_HOT_LRU: mark fact_ids (host array) as used now and promote the cold
 * ones (see above).  The copies (host link -> HBM) and the hot-table update
 * are queued on `stream`; work queued after them on the same stream reads
 * the new set.  Ids outside the store are ignored here.  *promoted_out (may
 * be NULL) receives the number of facts promoted.  First waits until the
 * previous touch's queued copies have finished (their lists are reused). */
int is_store_touch(is_store_t* store, const int32_t* fact_ids, int32_t n, void* stream,
                   int32_t* promoted_out);

/* IS_HOT_LRU counters since the policy was set: ids found hot, ids found
 * cold (each counted once per touch), facts promoted and their tokens. */
int is_store_lru_stats(const is_store_t* store, int64_t* hits_out, int64_t* misses_out,
                       int64_t* promoted_out, int64_t* promoted_tokens_out);

/* Tier of the store, hot-arena capacity and use (tokens per plane), and the
 * number of hot facts (0 for a device-tier store). */
int is_store_tier_info(const is_store_t* store, int32_t* tier_out, int64_t* hot_capacity_out,
                       int64_t* hot_used_out, int32_t* hot_facts_out);

/* Device addresses of the K and V arenas and the plane stride in tokens
 * (for callers that fill or inspect the store in place).  For
 * IS_TIER_HOST these are the device-mapped addresses of the host arenas. */
int is_store_arena(const is_store_t* store, void** k_arena_out, void** v_arena_out,
                   int64_t* plane_tokens_out);

/* ---- fact-sharded stores (several GPUs) -------------------------------- */

/* When the facts outgrow one GPU's memory (technical summary, Results,
 * "Scalability" names that limit; its answer there is host DRAM, the host
 * tier above), the store can instead be split by fact over the GPUs of a
 * node: each GPU keeps a store holding its share of the facts, and every
 * GPU injects its own requests reading each fact from the GPU that holds it
 * -- its own HBM, or a peer's over NVLink -- inside the one inject kernel,
 * with no staging copy.  The pages do not describe this partition; the
 * method (positions, rotation, scatter) is unchanged.
 *
 * A view is attached to a device-tier store (its "home": batch work space,
 * stream, status) and lists the shards' arenas and a global fact table.
 * While it is attached, the store's batches take GLOBAL fact ids, in
 * [0, num_global_facts), and read fact g's rows from arena fact_shard[g] at
 * token fact_offset[g] of every plane.  Every arena has the home store's
 * L, H and D and layout [L][H][plane_tokens][D] (another store's
 * is_store_arena, this GPU's or a peer's opened with is_ipc_open).
 *
 * Arguments (host arrays, copied):
 *   num_shards        >= 1
 *   k_arenas, v_arenas  [num_shards] device addresses, 16-byte aligned
 *   plane_tokens      [num_shards] tokens per plane of each arena
 *   num_global_facts  >= 1
 *   fact_shard        int32 [num_global_facts], in [0, num_shards)
 *   fact_offset       int64 [num_global_facts], >= 0
 *   fact_len          int32 [num_global_facts], >= 1, and
 *                     fact_offset + fact_len <= plane_tokens[fact_shard]
 * Replaces a previous view.  Waits for the device to go idle first.  The
 * arenas must stay valid and unchanged while batches that read them run
 * (for peers: keep their stores alive and stop putting facts until every
 * GPU's batches are done).  Errors: INVALID_ARG (null, bad table entry;
 * the previous view is kept), NOT_SUPPORTED (host-tier store), OOM, CUDA. */
int is_store_attach_shards(is_store_t* store, int32_t num_shards, const void* const* k_arenas,
                           const void* const* v_arenas, const int64_t* plane_tokens,
                           int32_t num_global_facts, const int32_t* fact_shard,
                           const int64_t* fact_offset, const int32_t* fact_len);

/* Drop the view: the store's batches read its own facts again.  Waits for
 * the device to go idle first.  A store with no view is left as it is. */
int is_store_detach_shards(is_store_t* store);

/* Number of shards of the attached view (0: none) and of its global facts. */
int is_store_shard_info(const is_store_t* store, int32_t* num_shards_out,
                        int32_t* num_global_facts_out);

/* Inter-process handle of a device allocation (a cudaIpcMemHandle_t). */
typedef struct {
  unsigned char bytes[64];
} is_ipc_handle_t;

/* Handles of a device-tier store's K and V arenas, for other processes on
 * this node to open with is_ipc_open, and its plane stride in tokens.
 * Errors: INVALID_ARG, NOT_SUPPORTED (host-tier store), CUDA. */
int is_store_export(const is_store_t* store, is_ipc_handle_t* k_handle_out,
                    is_ipc_handle_t* v_handle_out, int64_t* plane_tokens_out);

/* Map another process's exported arena into this process on `device`
 * (peer access enabled when the arena is on another GPU); *ptr_out is its
 * base address here.  is_ipc_close unmaps it: only after every batch that
 * reads it has finished.  A handle from this same process is refused by
 * CUDA (use is_store_arena instead).  Errors: INVALID_ARG, CUDA. */
int is_ipc_open(int device, const is_ipc_handle_t* handle, void** ptr_out);
int is_ipc_close(int device, void* ptr);

/* ---- the hot path ------------------------------------------------------ */

/* Inject one batch (technical summary, Online phase, "Dynamic rotation" and
 * "Injection").  Request r owns fact_ids[req_fact_offsets[r] ..
 * req_fact_offsets[r+1]) in retrieval order.  Token t of its j-th fact is
 * placed at position start_pos[r] + (lengths of facts 0..j-1) + t, i.e. the
 * facts form one contiguous segment.  For every such token, every layer and
 * every KV head:
 *     V cache row at slot  <- stored V row                (bit copy)
 *     K cache row at slot  <- bf16_rne(R(pos) . stored pre-RoPE K row)
 * with slot = block_tables[r][pos / B] * B + pos % B and R(pos) the RoPE
 * rotation of the store's configuration (fp64 angles, fp32 rotation).
 * No other cache element is written.
 *
 * Arguments (all arrays on the device):
 *   req_fact_offsets  int32 [num_requests + 1], CSR, non-decreasing,
 *                     [0] = 0, [num_requests] = num_fact_ids
 *   fact_ids          int32 [num_fact_ids]; duplicates allowed
 *   start_pos         int32 [num_requests], first injected position
 *   block_tables      int32 [num_requests][max_blocks_per_req]
 *   cache             geometry and base pointers of the paged cache
 *   slot_mapping_out  optional int64 [slot_mapping_capacity]: the slot of
 *                     every injected token, requests in order, segment order
 *                     within a request; -1 for tokens not written.  NULL
 *                     skips it.
 * Asynchronous on `stream`.  Returns host-side validation errors
 * (INVALID_ARG, CAPACITY when num_requests or num_fact_ids exceed the
 * store's batch limits, NOT_SUPPORTED, CUDA); device-side errors are found
 * by is_last_error():
 *   INVALID_ARG  CSR not starting at 0, not ending at num_fact_ids or with
 *                a decreasing offset (nothing written); a negative start
 *                (that request skipped)
 *   BAD_FACT_ID  id outside the store (its request skipped)
 *   POSITION     segment past max_blocks_per_req * B (request skipped)
 *   BAD_BLOCK    table entry outside [0, num_blocks) (that block skipped)
 *   CAPACITY     more tokens than slot_mapping_capacity (nothing written)
 * Requests must not share slots (the winner is undefined). */
int is_inject_batch(is_store_t* store, int32_t num_requests, const int32_t* req_fact_offsets,
                    const int32_t* fact_ids, int32_t num_fact_ids, const int32_t* start_pos,
                    const int32_t* block_tables, int32_t max_blocks_per_req,
                    const is_cache_t* cache, int64_t* slot_mapping_out,
                    int64_t slot_mapping_capacity, void* stream);

/* The same batch with the four index arrays in HOST memory (pinned memory
 * makes the copies asynchronous) and slot_mapping_out, if not NULL, in host
 * memory.  Copies the arrays into store-owned device buffers, runs the
 * batch, waits for `stream` and returns the batch's status (host-side or
 * device-side, as for is_inject_batch + is_last_error).  The caches stay on
 * the device.  On a device-tier store, slot_mapping_out in page-locked
 * memory mapped for the store's device (cudaHostAlloc, cudaMallocHost, a
 * mapped registration; the whole slot_mapping_capacity entries) is written
 * in place by the kernels, with exactly the entries is_inject_batch writes;
 * any other host buffer, and every buffer of a host-tier store (whose batch
 * keeps the host link busy), receives all slot_mapping_capacity entries of a
 * store-owned device buffer, whose entries past the batch's tokens (all of
 * them on CAPACITY) are stale. */
int is_inject_batch_host(is_store_t* store, int32_t num_requests,
                         const int32_t* req_fact_offsets, const int32_t* fact_ids,
                         int32_t num_fact_ids, const int32_t* start_pos,
                         const int32_t* block_tables, int32_t max_blocks_per_req,
                         const is_cache_t* cache, int64_t* slot_mapping_out,
                         int64_t slot_mapping_capacity, void* stream);

/* is_inject_batch_host for a stream of batches on a host-tier store with the
 * LRU hot set (IS_HOT_LRU): the same batch, and, while it runs, the cold
 * facts of the NEXT batch (next_fact_ids, host array, num_next_ids entries;
 * the caller's retrieval knows them before their injection) start moving
 * into HBM slots on a stream of the store -- slots not used by this batch,
 * in least-recently-used order -- so that batch
 * reads them from HBM (technical summary, Results, "Scalability": the KV
 * store may live in host DRAM; this is its prefetch path).  Every later
 * batch on the store waits for those transfers.  Ids that do not come or
 * are outside the store only cost their transfer; results never depend on
 * the prefetch.  On a store without the LRU policy the next ids are
 * ignored.  Errors as for is_inject_batch_host, and INVALID_ARG for
 * num_next_ids < 0 or a NULL list; when this batch ran clean but the
 * prefetch could not be started (OOM, CUDA), that error is returned after
 * the batch has completed. */
int is_inject_batch_host_next(is_store_t* store, int32_t num_requests,
                              const int32_t* req_fact_offsets, const int32_t* fact_ids,
                              int32_t num_fact_ids, const int32_t* start_pos,
                              const int32_t* block_tables, int32_t max_blocks_per_req,
                              const is_cache_t* cache, int64_t* slot_mapping_out,
                              int64_t slot_mapping_capacity, const int32_t* next_fact_ids,
                              int32_t num_next_ids, void* stream);

/* Wait for `stream`, then return and clear the first device-side error
 * recorded since the previous call (IS_OK if none).  *detail_out, if not
 * NULL, receives the offending index (request, CSR entry or block). */
int is_last_error(is_store_t* store, void* stream, int64_t* detail_out);

/* As is_last_error, but waits at most timeout_ms for `stream` (polling,
 * never blocking the calling thread longer): IS_ERR_TIMEOUT if the stream's
 * work has not finished by then (nothing is cleared; call again later).  For
 * callers that must not hang on a stalled stream. */
int is_last_error_timeout(is_store_t* store, void* stream, int32_t timeout_ms,
                          int64_t* detail_out);

/* Batches with at most max_requests requests (0..32; default 32) and at
 * most 256 fact ids (whose count times the store's longest fact stays below
 * 2^31 tokens) run as one kernel that composes the batch in every CTA
 * instead of a plan kernel followed by the inject kernel (lower latency;
 * same results).  0 always uses the two-kernel path. */
int is_store_set_small_batch_limit(is_store_t* store, int32_t max_requests);

/* ---- measurement -------------------------------------------------------- */

/* Enable (1) or disable (0) CUDA-event timing of the inject kernel itself
 * (the plan kernel excluded; for small batches the single kernel).  While enabled each batch records two events
 * on its stream around the inject kernel. */
int is_store_set_timing(is_store_t* store, int enable);

/* Sum of inject-kernel durations (ms) and number of timed launches since
 * the previous call; waits for the recorded events.  Resets the sums. */
int is_store_kernel_time(is_store_t* store, double* total_ms_out, int64_t* launches_out);

/* Human-readable name of a status code (static string). */
const char* is_status_string(int status);

/* ---- allocation-free variant ------------------------------------------- */

/* Limits of is_inject_batch_noalloc (its fixed work space). */
#define IS_NOALLOC_MAX_REQUESTS 1024
#define IS_NOALLOC_MAX_FACT_IDS 65536
#define IS_NOALLOC_MAX_BLOCKS 65536   /* touched cache blocks per batch */
#define IS_NOALLOC_MAX_HEAD_DIM 256

/* The inject batch of is_inject_batch for callers that cannot allocate
 * device memory.  The paper has no counterpart: this is a deployment
 * variant of the same plan and inject kernels, not a step of the method.
 *
 * Who needs it: code that runs where cudaMalloc is off limits -- inside a
 * serving engine whose memory pool already owns the whole GPU (a call to
 * cudaMalloc would fail or fragment the pool), or in a plugin whose host
 * may not create allocations behind its back.  Such a caller cannot create an is_store_t
 * (creation allocates), so it passes the store's contents itself.
 *
 * The per-batch work space (segment offsets, per-request sums, block
 * descriptors, plan header, status word, RoPE frequencies) lives in one
 * fixed array of about 1.3 MB in the library's device globals, which every
 * GPU that loads the library keeps until the process exits.  The call
 * itself calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * Arguments:
 *   cfg           num_layers, num_kv_heads, head_dim (<= 256) and the RoPE
 *                 fields as for is_store_create; the capacity, batch-limit
 *                 and tier fields are ignored
 *   k_store, v_store  device bf16 arenas [L][H][plane_tokens][D]
 *   fact_offsets  device int64 [num_facts]: first token of each fact in
 *                 every plane
 *   fact_lens     device int32 [num_facts]
 *   the batch arguments, cache and slot mapping as for is_inject_batch
 *   status_out    optional device buffer of 16 bytes that receives the
 *                 batch's device status: int32 code (an IS_* value), int32
 *                 padding, int64 detail (as is_last_error's detail)
 *   stream        as for is_inject_batch; the work is asynchronous
 * The device is the current device; every pointer must be on it.
 *
 * Limits: num_requests <= IS_NOALLOC_MAX_REQUESTS and num_fact_ids <=
 * IS_NOALLOC_MAX_FACT_IDS, else IS_ERR_CAPACITY is returned and nothing is
 * launched; a batch that touches more than IS_NOALLOC_MAX_BLOCKS cache
 * blocks writes nothing and reports IS_ERR_CAPACITY in status_out.
 *
 * The first call on a device looks up the work space's device address
 * (cudaGetSymbolAddress) and the kernels' launch settings; make that first
 * call before any stream capture.  All calls share the one work space and
 * each starts by clearing its status word: calls whose work overlaps on the
 * GPU (two streams, two host threads) race and must be ordered by the
 * caller, for instance by issuing them on one stream. */
int is_inject_batch_noalloc(const is_store_config_t* cfg, const void* k_store,
                            const void* v_store, int64_t plane_tokens,
                            const int64_t* fact_offsets, const int32_t* fact_lens,
                            int32_t num_facts, int32_t num_requests,
                            const int32_t* req_fact_offsets, const int32_t* fact_ids,
                            int32_t num_fact_ids, const int32_t* start_pos,
                            const int32_t* block_tables, int32_t max_blocks_per_req,
                            const is_cache_t* cache, int64_t* slot_mapping_out,
                            int64_t slot_mapping_capacity, void* status_out, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* INJECT_STORE_H */
