/*
 * CPU oracle for the InferScale retrieve-and-inject path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no
 * code, header, table or constant with the CUDA path.
 *
 * It is the plain definition of what the online phase computes, written as
 * loops in fp64 (page titles below refer to the three summaries of
 * "InferScale: GPU-Native KV Injection for Personalized LLM Serving",
 * gist.science/{ja,nl,it}/paper/2607.27090, technical summary, section
 * "Methodology -- 2. Online phase: Chunked RoPE and KV injection"):
 *
 *   - Pre-RoPE storage: keys are captured before rotary embedding and stored
 *     with the raw values (the fact store, orc_store_put).
 *   - Dynamic rotation: the retrieved facts are composed into one contiguous
 *     segment; each stored key is rotated for its new serving position
 *     (orc_segment, orc_rope_row).
 *   - Injection: the composed K/V are scatter-copied into the paged KV cache
 *     (orc_slot, orc_inject_batch).
 *
 * RoPE itself (inv_freq_i = theta^(-2i/D), pairs rotated by pos * inv_freq_i)
 * and the Llama-3.1 frequency scaling are not printed on the pages; they are
 * the standard published definitions of the named model families.
 *
 * Precision: every angle, cosine, sine and rotation is fp64; a rotated key is
 * rounded once, fp64 -> bf16 round-to-nearest-even.  Values are copied as bit
 * patterns.
 *
 * Parity pins (tests/test_oracle_pins.py): closed-form RoPE values, rotation
 * group laws against a matrix power, the relative-position property
 * (Theorem 6) by brute force, the one-layer prefill equivalence (Theorem 3),
 * the gather view of the paged cache, bf16 rounding by exact comparison.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum {
  ORC_OK = 0,
  ORC_ERR_INVALID_ARG = -1,
  ORC_ERR_BAD_FACT_ID = -2,
  ORC_ERR_POSITION = -3,
  ORC_ERR_BAD_BLOCK = -4,
  ORC_ERR_CAPACITY = -5,
};

/* ------------------------------------------------------------------ bf16 */

/* bf16 is the upper half of an IEEE binary32 word. */
double orc_bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Nearest bf16 to x (8 significant bits, exponent range of binary32), ties to
 * even, taken in one step from the fp64 value. */
uint16_t orc_f64_to_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (a == 0.0) return sign;
  if (isinf(a)) return (uint16_t)(sign | 0x7F80);
  int e;
  frexp(a, &e);                       /* a = m * 2^e, m in [0.5, 1) */
  if (e < -125) e = -125;             /* subnormal bf16 spacing is 2^-133 */
  double spacing = ldexp(1.0, e - 8); /* distance between bf16 neighbours */
  double n = nearbyint(a / spacing);  /* round half to even (default mode) */
  double r = n * spacing;
  if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80);
  float f = (float)r; /* exact: r has <= 8 significant bits in range */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(sign | (u >> 16));
}

void orc_bf16_to_f64_array(const uint16_t* in, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_to_f64(in[i]);
}

void orc_f64_to_bf16_array(const double* in, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_f64_to_bf16(in[i]);
}

/* ------------------------------------------------------------------ RoPE */

/* Llama-3.1 frequency scaling of one frequency (published rule):
 * wavelength lam = 2 pi / f; lam < orig/high keeps f; lam > orig/low gives
 * f/factor; between, f is blended with weight
 * smooth = (orig/lam - low) / (high - low) on the unscaled frequency. */
double orc_llama3_scale(double f, double factor, double low, double high, double orig) {
  double lam = 2.0 * M_PI / f;
  double low_wl = orig / low;   /* longest wavelength kept partly unscaled */
  double high_wl = orig / high; /* shortest wavelength that gets blended */
  if (lam < high_wl) return f;
  if (lam > low_wl) return f / factor;
  double smooth = (orig / lam - low) / (high - low);
  return (1.0 - smooth) * f / factor + smooth * f;
}

/* inv_freq[i] = theta^(-2i/D), i in [0, D/2); scaling 1 applies the Llama-3.1
 * rule above.  Returns ORC_ERR_INVALID_ARG for an odd or non-positive D. */
int orc_rope_inv_freq(int D, double theta, int scaling, double factor, double low,
                      double high, double orig, double* out) {
  if (D <= 0 || D % 2 != 0 || !(theta > 0.0)) return ORC_ERR_INVALID_ARG;
  for (int i = 0; i < D / 2; ++i) {
    double f = pow(theta, -(2.0 * i) / (double)D);
    if (scaling == 1) f = orc_llama3_scale(f, factor, low, high, orig);
    out[i] = f;
  }
  return ORC_OK;
}

/* The pair (a, b) that frequency i rotates.  style 0: rotate-half, pairs
 * (i, i + D/2); style 1: interleaved, pairs (2i, 2i + 1). */
static void pair_of(int i, int D, int style, int* a, int* b) {
  if (style == 0) { *a = i; *b = i + D / 2; }
  else { *a = 2 * i; *b = 2 * i + 1; }
}

/* y = R(pos) x for one head row of D values (D <= 1024; y may alias x):
 *   y_a = x_a cos(pos f_i) - x_b sin(pos f_i)
 *   y_b = x_b cos(pos f_i) + x_a sin(pos f_i).  pos may be negative. */
void orc_rope_row(const double* x, double* y, int D, int64_t pos, const double* inv_freq,
                  int style) {
  double out[1024];
  if (D <= 0 || D > 1024) return;
  for (int i = 0; i < D / 2; ++i) {
    int a, b;
    pair_of(i, D, style, &a, &b);
    double ang = (double)pos * inv_freq[i];
    double c = cos(ang), s = sin(ang);
    out[a] = x[a] * c - x[b] * s;
    out[b] = x[b] * c + x[a] * s;
  }
  memcpy(y, out, sizeof(double) * (size_t)D);
}

/* n rows: y[r] = R(pos[r]) x[r]. */
void orc_rope_rows(const double* x, double* y, int64_t n, int D, const int64_t* pos,
                   const double* inv_freq, int style) {
  for (int64_t r = 0; r < n; ++r)
    orc_rope_row(x + r * D, y + r * D, D, pos[r], inv_freq, style);
}

/* ------------------------------------------------------------- fact store */

/* The store holds, per (layer l, head h), one plane of tokens:
 *   K[((l * H + h) * T_cap + token) * D + d], same for V,
 * and fact f occupies tokens [off[f], off[f] + len[f]) of every plane.
 * Facts are appended in put order, so off[f] = sum of earlier lengths. */
typedef struct {
  int32_t L, H, D;
  int64_t T_cap;      /* tokens per plane */
  int64_t T_used;     /* tokens appended so far */
  int32_t num_facts;
  int32_t max_facts;
  uint16_t* k;        /* [L][H][T_cap][D] */
  uint16_t* v;
  int64_t* off;       /* [max_facts] */
  int32_t* len;       /* [max_facts] */
} orc_store_t;

/* Append one fact given as k, v: bf16 [L][H][len][D].  Returns the new id
 * or a negative error. */
int32_t orc_store_put(orc_store_t* s, const uint16_t* k, const uint16_t* v, int32_t len) {
  if (len <= 0) return ORC_ERR_INVALID_ARG;
  if (s->num_facts >= s->max_facts || s->T_used + len > s->T_cap) return ORC_ERR_CAPACITY;
  int32_t id = s->num_facts;
  int64_t off = s->T_used;
  for (int32_t l = 0; l < s->L; ++l)
    for (int32_t h = 0; h < s->H; ++h)
      for (int32_t t = 0; t < len; ++t)
        for (int32_t d = 0; d < s->D; ++d) {
          int64_t src = (((int64_t)l * s->H + h) * len + t) * s->D + d;
          int64_t dst = (((int64_t)l * s->H + h) * s->T_cap + off + t) * s->D + d;
          s->k[dst] = k[src];
          s->v[dst] = v[src];
        }
  s->off[id] = off;
  s->len[id] = len;
  s->num_facts = id + 1;
  s->T_used = off + len;
  return id;
}

/* --------------------------------------------------- segment and the slot */

/* Paged-cache slot of logical position pos for a request with block table
 * row bt (max_blocks entries): bt[pos / B] * B + pos % B.  Returns -1 when
 * pos is past the table or the entry is outside [0, num_blocks). */
int64_t orc_slot(const int32_t* bt, int32_t max_blocks, int32_t B, int32_t num_blocks,
                 int64_t pos) {
  if (pos < 0 || pos / B >= max_blocks) return -1;
  int32_t blk = bt[pos / B];
  if (blk < 0 || blk >= num_blocks) return -1;
  return (int64_t)blk * B + pos % B;
}

/* Per-request validation and length of the composed segment.  A request
 * whose CSR range is malformed has no tokens.  A fact id outside
 * [0, num_facts) counts as length 0 and makes the request invalid.  Returns
 * the request's status; *seg_len receives the segment length. */
static int request_segment(const orc_store_t* s, const int32_t* req_off, const int32_t* ids,
                           int32_t num_ids, int32_t r, int64_t* seg_len) {
  int32_t a = req_off[r], b = req_off[r + 1];
  *seg_len = 0;
  if (a < 0 || b < a || b > num_ids) return ORC_ERR_INVALID_ARG;
  int st = ORC_OK;
  for (int32_t j = a; j < b; ++j) {
    int32_t f = ids[j];
    if (f < 0 || f >= s->num_facts) { st = ORC_ERR_BAD_FACT_ID; continue; }
    *seg_len += s->len[f];
  }
  return st;
}

/* Segment composition for one batch, token by token in request order, and
 * within a request in the given fact order: token t of the j-th fact of
 * request r sits at position start[r] + (lengths of facts before j) + t.
 * A request that is invalid (bad fact id, negative start, segment past its
 * block table) keeps its token indices but none of its tokens is written.
 * Writes, per token, the request, the store token index, the position and
 * the slot (-1 when not written); arrays may be NULL, at most cap entries.
 * Returns the number of tokens, or ORC_ERR_INVALID_ARG when the CSR of the
 * whole batch is wrong -- first offset not 0, last offset not the number of
 * ids, or an offset smaller than the one before -- (then nothing is
 * composed). */
int64_t orc_segment(const orc_store_t* s, int32_t R, const int32_t* req_off, const int32_t* ids,
                    int32_t num_ids, const int32_t* start, const int32_t* bt, int32_t max_blocks,
                    int32_t B, int32_t num_blocks, int64_t cap, int32_t* tok_req,
                    int64_t* tok_src, int64_t* tok_pos, int64_t* tok_slot, int* status) {
  int st = ORC_OK;
  if (R < 0 || B <= 0 || req_off == NULL || req_off[0] != 0 || req_off[R] != num_ids) {
    if (status) *status = ORC_ERR_INVALID_ARG;
    return ORC_ERR_INVALID_ARG;
  }
  /* A CSR's offsets never decrease; one that does is not a batch. */
  for (int32_t r = 0; r < R; ++r)
    if (req_off[r + 1] < req_off[r]) {
      if (status) *status = ORC_ERR_INVALID_ARG;
      return ORC_ERR_INVALID_ARG;
    }
  int64_t n = 0;
  for (int32_t r = 0; r < R; ++r) {
    int64_t S;
    int rs = request_segment(s, req_off, ids, num_ids, r, &S);
    if (rs == ORC_ERR_INVALID_ARG) { /* malformed range: no tokens */
      if (st == ORC_OK) st = rs;
      continue;
    }
    if (rs == ORC_OK && start[r] < 0) rs = ORC_ERR_INVALID_ARG;
    if (rs == ORC_OK && (int64_t)start[r] + S > (int64_t)max_blocks * B) rs = ORC_ERR_POSITION;
    if (rs != ORC_OK && st == ORC_OK) st = rs;
    int64_t i = 0; /* index inside the segment */
    for (int32_t j = req_off[r]; j < req_off[r + 1]; ++j) {
      int32_t f = ids[j];
      if (f < 0 || f >= s->num_facts) continue;
      for (int32_t t = 0; t < s->len[f]; ++t, ++i, ++n) {
        if (n >= cap) continue;
        int64_t pos = (int64_t)start[r] + i;
        int64_t slot = -1;
        if (rs == ORC_OK) {
          slot = orc_slot(bt + (int64_t)r * max_blocks, max_blocks, B, num_blocks, pos);
          if (slot < 0 && st == ORC_OK) st = ORC_ERR_BAD_BLOCK;
        }
        if (tok_req) tok_req[n] = r;
        if (tok_src) tok_src[n] = s->off[f] + t;
        if (tok_pos) tok_pos[n] = pos;
        if (tok_slot) tok_slot[n] = slot;
      }
    }
  }
  if (status) *status = st;
  return n;
}

/* --------------------------------------------------------------- inject */

/* Paged cache addressing.  Element (layer l, slot s = block * B + o, head h,
 * dim d) of the K cache is k[l * layer_stride + block * block_stride +
 * o * token_stride + h * head_stride + d] (strides in elements); V alike. */
typedef struct {
  uint16_t* k;
  uint16_t* v;
  double* k_ref;          /* optional fp64 rotated keys, same indexing as k */
  int64_t layer_stride, block_stride, token_stride, head_stride;
  int32_t num_blocks, block_size;
} orc_cache_t;

/* The whole online inject for one batch.  For every valid request, every
 * token of its segment, every layer and every KV head:
 *   V cache row at the token's slot  <- stored V row   (bit copy)
 *   K cache row at the token's slot  <- bf16(R(pos) . stored K row)
 * Nothing else in the cache changes.  slot_out (optional) receives each
 * token's slot, -1 where nothing was written; if the batch has more tokens
 * than cap, nothing is written at all and ORC_ERR_CAPACITY is returned.
 * Returns the first error met (in request order), or ORC_OK. */
int orc_inject_batch(const orc_store_t* s, int style, const double* inv_freq, int32_t R,
                     const int32_t* req_off, const int32_t* ids, int32_t num_ids,
                     const int32_t* start, const int32_t* bt, int32_t max_blocks,
                     const orc_cache_t* c, int64_t* slot_out, int64_t cap, int num_threads) {
  const int32_t B = c->block_size;
  if (R < 0 || B <= 0 || s->D <= 0 || s->D % 2 || s->D > 1024) return ORC_ERR_INVALID_ARG;
  int status = ORC_OK;
  int64_t n = orc_segment(s, R, req_off, ids, num_ids, start, bt, max_blocks, B, c->num_blocks,
                          0, NULL, NULL, NULL, NULL, &status);
  if (n < 0) return (int)n;
  if (slot_out && n > cap) return ORC_ERR_CAPACITY;
  size_t m = (size_t)(n > 0 ? n : 1);
  int64_t* tok_src = (int64_t*)malloc(sizeof(int64_t) * m);
  int64_t* tok_pos = (int64_t*)malloc(sizeof(int64_t) * m);
  int64_t* tok_slot = (int64_t*)malloc(sizeof(int64_t) * m);
  if (!tok_src || !tok_pos || !tok_slot) {
    free(tok_src); free(tok_pos); free(tok_slot);
    return ORC_ERR_CAPACITY;
  }
  orc_segment(s, R, req_off, ids, num_ids, start, bt, max_blocks, B, c->num_blocks, n, NULL,
              tok_src, tok_pos, tok_slot, &status);
  if (slot_out)
    for (int64_t i = 0; i < n; ++i) slot_out[i] = tok_slot[i];
  const int32_t L = s->L, H = s->H, D = s->D;
#ifdef _OPENMP
  if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 16)
#endif
  for (int64_t i = 0; i < n; ++i) {
    if (tok_slot[i] < 0) continue;
    const int64_t blk = tok_slot[i] / B, o = tok_slot[i] % B;
    double x[1024], y[1024];
    for (int32_t l = 0; l < L; ++l)
      for (int32_t h = 0; h < H; ++h) {
        const int64_t src = (((int64_t)l * H + h) * s->T_cap + tok_src[i]) * D;
        const int64_t dst = l * c->layer_stride + blk * c->block_stride + o * c->token_stride +
                            h * c->head_stride;
        for (int32_t d = 0; d < D; ++d) {
          c->v[dst + d] = s->v[src + d];
          x[d] = orc_bf16_to_f64(s->k[src + d]);
        }
        orc_rope_row(x, y, D, tok_pos[i], inv_freq, style);
        for (int32_t d = 0; d < D; ++d) {
          c->k[dst + d] = orc_f64_to_bf16(y[d]);
          if (c->k_ref) c->k_ref[dst + d] = y[d];
        }
      }
  }
  free(tok_src); free(tok_pos); free(tok_slot);
  return status;
}

int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
