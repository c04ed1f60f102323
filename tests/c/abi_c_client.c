/* A plain C client of libinjectstore.so: only include/inject_store.h and the
 * CUDA runtime for device memory.  Creates a small store, puts two facts,
 * injects one request into a paged cache, and checks what it can check
 * without an oracle: V rows are bit copies of the stored rows at the slots
 * the block table gives, a slot outside the segment is untouched, and the
 * first token (position 0) keeps its key unrotated.  Then a fact-sharded
 * view: a second store holds fact 0, the first store's view reads global
 * fact 0 from it and global fact 1 from its own arena, and the same request
 * through the view writes the same cache bytes.  Exit status 0 on success;
 * prints the failing step otherwise. */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "inject_store.h"

#define L 2
#define H 2
#define D 64
#define B 16
#define NB 4

static int fail(const char* what, int rc) {
  fprintf(stderr, "abi_c_client: %s failed: %s (%d)\n", what, is_status_string(rc), rc);
  return 1;
}

/* Put fact f (len tokens, its own bit patterns) from host memory. */
static int put_fact(is_store_t* store, int f, int len, int32_t* id) {
  const size_t n = (size_t)L * H * len * D;
  uint16_t* k = malloc(n * 2);
  uint16_t* v = malloc(n * 2);
  for (size_t i = 0; i < n; ++i) {
    k[i] = (uint16_t)(0x3C00 + ((i * 7 + f * 13) & 0x3FF));
    v[i] = (uint16_t)(0x4000 + ((i * 11 + f * 5) & 0x3FF));
  }
  const int rc = is_store_put_fact(store, k, v, len, id); /* host pointers */
  free(k);
  free(v);
  return rc;
}

int main(void) {
  is_store_config_t cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.num_layers = L;
  cfg.num_kv_heads = H;
  cfg.head_dim = D;
  cfg.rope_style = IS_ROPE_ROTATE_HALF;
  cfg.rope_theta = 10000.0;
  cfg.rope_scaling = IS_SCALING_NONE;
  cfg.capacity_tokens = 64;
  cfg.max_facts = 4;
  cfg.tier = IS_TIER_DEVICE;
  is_store_t* store = NULL;
  int rc = is_store_create(&cfg, 0, &store);
  if (rc != IS_OK) return fail("is_store_create", rc);

  /* two facts of 5 and 9 tokens; value of element (l, h, t, d) of fact f is
   * a distinct bf16 bit pattern */
  const int lens[2] = {5, 9};
  for (int f = 0; f < 2; ++f) {
    int32_t id = -1;
    rc = put_fact(store, f, lens[f], &id);
    if (rc != IS_OK || id != f) return fail("is_store_put_fact", rc);
  }

  /* one request: facts 1 then 0, starting at position 0; blocks 2, 0 */
  const int32_t h_off[2] = {0, 2}, h_ids[2] = {1, 0}, h_start[1] = {0}, h_bt[2] = {2, 0};
  int32_t *d_off, *d_ids, *d_start, *d_bt;
  int64_t* d_slots;
  uint16_t *kc, *vc;
  const size_t cache_elems = (size_t)L * NB * B * H * D;
  if (cudaMalloc((void**)&d_off, 8) || cudaMalloc((void**)&d_ids, 8) || cudaMalloc((void**)&d_start, 4) ||
      cudaMalloc((void**)&d_bt, 8) || cudaMalloc((void**)&d_slots, 14 * 8) ||
      cudaMalloc((void**)&kc, cache_elems * 2) || cudaMalloc((void**)&vc, cache_elems * 2))
    return fail("cudaMalloc", IS_ERR_CUDA);
  cudaMemcpy(d_off, h_off, 8, cudaMemcpyHostToDevice);
  cudaMemcpy(d_ids, h_ids, 8, cudaMemcpyHostToDevice);
  cudaMemcpy(d_start, h_start, 4, cudaMemcpyHostToDevice);
  cudaMemcpy(d_bt, h_bt, 8, cudaMemcpyHostToDevice);
  cudaMemset(kc, 0x55, cache_elems * 2);
  cudaMemset(vc, 0x55, cache_elems * 2);
  is_cache_t cache;
  cache.k_cache = kc;
  cache.v_cache = vc;
  cache.layer_stride = (int64_t)NB * B * H * D;
  cache.block_stride = (int64_t)B * H * D;
  cache.token_stride = H * D;
  cache.head_stride = D;
  cache.num_blocks = NB;
  cache.block_size = B;
  rc = is_inject_batch(store, 1, d_off, d_ids, 2, d_start, d_bt, 2, &cache, d_slots, 14, NULL);
  if (rc != IS_OK) return fail("is_inject_batch", rc);
  int64_t detail = 0;
  rc = is_last_error(store, NULL, &detail);
  if (rc != IS_OK) return fail("device status", rc);

  int64_t slots[14];
  uint16_t* vh = malloc(cache_elems * 2);
  uint16_t* kh = malloc(cache_elems * 2);
  cudaMemcpy(slots, d_slots, sizeof slots, cudaMemcpyDeviceToHost);
  cudaMemcpy(vh, vc, cache_elems * 2, cudaMemcpyDeviceToHost);
  cudaMemcpy(kh, kc, cache_elems * 2, cudaMemcpyDeviceToHost);
  for (int p = 0; p < 14; ++p) {
    const int64_t want = (int64_t)h_bt[p / B] * B + p % B;
    if (slots[p] != want) return fail("slot mapping", IS_ERR_INVALID_ARG);
  }
  /* V of token p (fact 1 for p < 9, then fact 0) at (l, h) */
  uint16_t* vf = malloc((size_t)L * H * 9 * D * 2);
  uint16_t* kf = malloc((size_t)L * H * 9 * D * 2);
  for (int p = 0; p < 14; ++p) {
    const int f = p < 9 ? 1 : 0, t = p < 9 ? p : p - 9;
    if (is_store_read_fact(store, f, kf, vf) != IS_OK) return fail("is_store_read_fact", IS_ERR_CUDA);
    for (int l = 0; l < L; ++l)
      for (int h = 0; h < H; ++h)
        for (int d = 0; d < D; ++d) {
          const uint16_t want = vf[(((size_t)l * H + h) * lens[f] + t) * D + d];
          const uint16_t got = vh[l * cache.layer_stride + slots[p] * H * D + h * D + d];
          if (got != want) return fail("V bit copy", IS_ERR_INVALID_ARG);
          if (p == 0 && kh[l * cache.layer_stride + slots[p] * H * D + h * D + d] !=
                            kf[(((size_t)l * H + h) * lens[f] + t) * D + d])
            return fail("key at position 0", IS_ERR_INVALID_ARG);
        }
  }
  /* slot 14 of the request (block 0, offset 14) is outside the segment */
  for (int d = 0; d < H * D; ++d)
    if (vh[(size_t)(h_bt[0] * B + 14) * H * D + d] != 0x5555) return fail("untouched slot", IS_ERR_INVALID_ARG);

  /* Fact-sharded view: store2 holds fact 0; global fact 0 -> store2, global
   * fact 1 -> this store's own fact 1. */
  is_store_t* store2 = NULL;
  rc = is_store_create(&cfg, 0, &store2);
  if (rc != IS_OK) return fail("is_store_create (shard)", rc);
  int32_t id2 = -1;
  rc = put_fact(store2, 0, lens[0], &id2);
  if (rc != IS_OK || id2 != 0) return fail("is_store_put_fact (shard)", rc);
  void *ka[2], *va[2];
  int64_t plane[2], off1 = 0, off0 = 0;
  int32_t len1 = 0, len0 = 0;
  if (is_store_arena(store, &ka[0], &va[0], &plane[0]) != IS_OK ||
      is_store_arena(store2, &ka[1], &va[1], &plane[1]) != IS_OK ||
      is_store_fact_info(store, 1, &off1, &len1) != IS_OK || is_store_fact_info(store2, 0, &off0, &len0) != IS_OK)
    return fail("arena / fact info", IS_ERR_INVALID_ARG);
  is_ipc_handle_t hk, hv;
  int64_t exported_plane = 0;
  rc = is_store_export(store2, &hk, &hv, &exported_plane);
  if (rc != IS_OK || exported_plane != plane[1]) return fail("is_store_export", rc);
  const int32_t g_shard[2] = {1, 0}, g_len[2] = {len0, len1};
  const int64_t g_off[2] = {off0, off1};
  const int32_t bad_shard[2] = {1, 2};
  if (is_store_attach_shards(store, 2, (const void* const*)ka, (const void* const*)va, plane, 2, bad_shard, g_off,
                             g_len) != IS_ERR_INVALID_ARG)
    return fail("attach rejects a bad shard", IS_ERR_INVALID_ARG);
  rc = is_store_attach_shards(store, 2, (const void* const*)ka, (const void* const*)va, plane, 2, g_shard, g_off,
                              g_len);
  if (rc != IS_OK) return fail("is_store_attach_shards", rc);
  int32_t n_shards = 0, n_global = 0;
  if (is_store_shard_info(store, &n_shards, &n_global) != IS_OK || n_shards != 2 || n_global != 2)
    return fail("is_store_shard_info", IS_ERR_INVALID_ARG);
  uint16_t *kc2, *vc2;
  if (cudaMalloc((void**)&kc2, cache_elems * 2) || cudaMalloc((void**)&vc2, cache_elems * 2))
    return fail("cudaMalloc", IS_ERR_CUDA);
  cudaMemset(kc2, 0x55, cache_elems * 2);
  cudaMemset(vc2, 0x55, cache_elems * 2);
  is_cache_t cache2 = cache;
  cache2.k_cache = kc2;
  cache2.v_cache = vc2;
  rc = is_inject_batch(store, 1, d_off, d_ids, 2, d_start, d_bt, 2, &cache2, NULL, 0, NULL);
  if (rc != IS_OK) return fail("is_inject_batch (view)", rc);
  rc = is_last_error(store, NULL, &detail);
  if (rc != IS_OK) return fail("device status (view)", rc);
  uint16_t* kh2 = malloc(cache_elems * 2);
  uint16_t* vh2 = malloc(cache_elems * 2);
  cudaMemcpy(kh2, kc2, cache_elems * 2, cudaMemcpyDeviceToHost);
  cudaMemcpy(vh2, vc2, cache_elems * 2, cudaMemcpyDeviceToHost);
  if (memcmp(kh2, kh, cache_elems * 2) || memcmp(vh2, vh, cache_elems * 2))
    return fail("sharded view reproduces the cache", IS_ERR_INVALID_ARG);
  if (is_store_detach_shards(store) != IS_OK || is_store_shard_info(store, &n_shards, &n_global) != IS_OK ||
      n_shards != 0)
    return fail("is_store_detach_shards", IS_ERR_INVALID_ARG);
  is_store_destroy(store2);
  is_store_destroy(store);
  printf("abi_c_client: ok\n");
  return 0;
}
