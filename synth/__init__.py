"""Seeded synthetic inputs for the retrieve-and-inject path.

This module only makes inputs.  It holds none of the method's arithmetic (no
RoPE, no positions, no slot mapping): both the CPU oracle's tests and the CUDA
path's tests and benchmark draw their inputs from here, so the two sides see
the same bytes without sharing any code.

Two kinds of data:

* Bulk bf16 tensors (fact keys/values, cache pre-fill).  These come from a
  counter-based generator, so any single element can be regenerated on the host
  without materialising the whole tensor (the full-size fact store is tens of
  GB and lives only on the GPU).  Element ``n`` of stream ``s`` under ``seed``
  is a standard normal value rounded to bf16 (round to nearest, ties to even),
  drawn by inverting its distribution over the bf16 grid:

      G      = 0x9E3779B97F4A7C15                     (SplitMix64 increment)
      mix(z) = SplitMix64 output function (Steele, Lea, Flood 2014):
               z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
               z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31
      key    = mix(seed * G + s)                      (all arithmetic mod 2^64)
      w_j    = mix(key + (2n + j) * G),  j = 0, 1
      |x|    = the bf16 magnitude code c (0 .. 0x7F7F) whose rounding
               interval holds the quantile w_0 / 2^64 of |X|, X ~ N(0, 1):
               c = number of codes whose upper interval edge h_c (the
               midpoint to the next code) has Q_c <= w_0, with
               Q_c = round(2^64 P(|X| < h_c))           (the table below)
      sign   = top bit of w_1.

  P(|X| < h) = erf(h / sqrt 2) is evaluated once in fp64 (upper tail through
  erfc) into the integer table Q; sampling is integer comparisons only, so
  the host (numpy, here) and the device (``synth/csrc/fill.cu``, handed the
  same table) produce identical bits.  The 2^-64 resolution leaves out
  magnitudes below about 2^-65 and above about 9.3: a sample of 10^10 values
  reaches beyond 6.5 sigma (the largest |x| of such a sample) with room to
  spare.

* Small integer metadata (fact lengths, retrieved ids, block tables, start
  positions), drawn on the host with ``numpy.random.default_rng(seed)``.
"""
from __future__ import annotations

import ctypes
import functools
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_G = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Stream tags: the high bits of a stream id name the tensor family.
TAG_FACT = 1 << 40        # stream = TAG_FACT | (fact_id << 1) | is_value
TAG_CACHE = 2 << 40       # stream = TAG_CACHE | is_value   (cache pre-fill)


def _mix(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * _M1
    z = z ^ (z >> np.uint64(27))
    z = z * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        z = np.array([seed], dtype=np.uint64) * _G + np.array([stream], dtype=np.uint64)
        return _mix(z)[0]


def _bf16_code_value(code: int) -> float:
    return float(np.array([code << 16], np.uint32).view(np.float32)[0])


@functools.lru_cache(maxsize=1)
def normal_table() -> tuple[int, np.ndarray]:
    """(first code, thresholds): Q_c for the codes c = first, first + 1, ...
    whose threshold lies strictly inside (0, 2^64); every code below `first`
    has Q_c = 0 and every code past the table Q_c = 2^64 - 1 (never reached
    but by w_0 = 2^64 - 1).  Q_c = round(2^64 P(|X| < h_c)), h_c the midpoint
    between bf16 codes c and c + 1."""
    two64 = 1 << 64
    q = []
    for c in range(0x7F7F):
        h = 0.5 * (_bf16_code_value(c) + _bf16_code_value(c + 1))
        if h <= 1.0:
            t = int(round(math.ldexp(math.erf(h / math.sqrt(2.0)), 64)))
        else:
            t = two64 - int(round(math.ldexp(math.erfc(h / math.sqrt(2.0)), 64)))
        q.append(min(t, two64 - 1))
    q = np.array(q, dtype=np.uint64)
    first = int(np.argmax(q > 0))
    last = int(np.argmax(q == np.uint64(two64 - 1)))
    return first, q[first:last].copy()


def bf16_bits(seed: int, stream: int, index) -> np.ndarray:
    """bf16 bit patterns (uint16) of elements ``index`` (int array) of a stream."""
    n = np.asarray(index, dtype=np.uint64)
    key = stream_key(seed, stream)
    first, q = normal_table()
    with np.errstate(over="ignore"):
        base = key + (n * np.uint64(2)) * _G
        w0 = _mix(base)
        w1 = _mix(base + _G)
    code = first + np.searchsorted(q, w0, side="right").astype(np.int64)
    sign = (w1 >> np.uint64(63)).astype(np.int64) << 15
    return (code | sign).astype(np.uint16)


def bf16_block(seed: int, stream: int, shape, base: int = 0) -> np.ndarray:
    """A whole tensor of the given shape: elements base .. base + prod(shape)."""
    count = int(np.prod(shape))
    return bf16_bits(seed, stream, np.arange(base, base + count, dtype=np.uint64)).reshape(shape)


def bf16_to_float(bits: np.ndarray) -> np.ndarray:
    """Decode bf16 bit patterns to float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def fact_stream(fact_id: int, is_value: bool) -> int:
    return TAG_FACT | (int(fact_id) << 1) | int(bool(is_value))


def fact_kv(seed: int, fact_id: int, L: int, H: int, length: int, D: int):
    """Pre-RoPE K and raw V of one fact, bf16 bits shaped [L][H][length][D]."""
    shape = (L, H, length, D)
    return (bf16_block(seed, fact_stream(fact_id, False), shape),
            bf16_block(seed, fact_stream(fact_id, True), shape))


def fact_rows(seed: int, fact_id: int, is_value: bool, L: int, H: int, length: int,
              D: int, l, h, t) -> np.ndarray:
    """Rows [.., D] of a fact's K or V at (layer l, head h, token t) (arrays, broadcast)."""
    l, h, t = np.broadcast_arrays(np.asarray(l), np.asarray(h), np.asarray(t))
    row0 = ((l.astype(np.int64) * H + h) * length + t) * D
    idx = row0[..., None] + np.arange(D, dtype=np.int64)
    return bf16_bits(seed, fact_stream(fact_id, is_value), idx.astype(np.uint64))


# ---------------------------------------------------------------------------
# Workload descriptions (shapes, sizes and distributions of the page's setups)
# ---------------------------------------------------------------------------

@dataclass
class Model:
    name: str
    num_layers: int
    num_kv_heads: int
    head_dim: int
    rope_theta: float
    llama3: bool = False            # Llama-3.1 frequency scaling (8, 1, 4, 8192)

    def scaling(self):
        if not self.llama3:
            return None
        return dict(factor=8.0, low_freq_factor=1.0, high_freq_factor=4.0,
                    original_max_position=8192)

    @property
    def bytes_per_token(self) -> int:
        """K+V bytes of one token over all layers and KV heads (bf16)."""
        return 2 * self.num_layers * self.num_kv_heads * self.head_dim * 2


TINY = Model("tiny", 1, 2, 64, 1.0e4)
LLAMA31_8B = Model("llama-3.1-8b", 32, 8, 128, 5.0e5, llama3=True)
MISTRAL_7B = Model("mistral-7b", 32, 8, 128, 1.0e6)
QWEN25_7B = Model("qwen2.5-7b", 28, 4, 128, 1.0e6)
MODELS = {m.name: m for m in (TINY, LLAMA31_8B, MISTRAL_7B, QWEN25_7B)}


@dataclass
class Batch:
    """One inject batch: CSR fact ids, start positions and block tables."""
    req_offsets: np.ndarray          # int32 [R+1]
    fact_ids: np.ndarray             # int32 [req_offsets[R]]
    start_pos: np.ndarray            # int32 [R]
    block_tables: np.ndarray         # int32 [R][max_blocks]
    block_size: int
    num_blocks: int

    @property
    def num_requests(self) -> int:
        return len(self.start_pos)

    @property
    def max_blocks(self) -> int:
        return self.block_tables.shape[1]


@dataclass
class Workload:
    name: str
    model: Model
    fact_lens: np.ndarray            # int32 [num_facts]
    batch: Batch
    seed: int = 0
    notes: dict = field(default_factory=dict)

    def tokens(self) -> int:
        b = self.batch
        return int(self.fact_lens[b.fact_ids].sum()) if len(b.fact_ids) else 0


def uniform_lengths(rng, n, lo, hi):
    return rng.integers(lo, hi + 1, size=n).astype(np.int32)


def lognormal_lengths(rng, n, median=32.0, sigma=0.5, lo=8, hi=96):
    x = rng.lognormal(mean=np.log(median), sigma=sigma, size=n)
    return np.clip(np.rint(x), lo, hi).astype(np.int32)


def distinct_ids(rng, num_facts, k):
    return rng.choice(num_facts, size=k, replace=False).astype(np.int32)


def zipf_distinct_ids(rng, rank_to_fact, probs, k):
    """k distinct facts drawn by Zipf rank (rejection of repeats)."""
    out, seen = [], set()
    while len(out) < k:
        need = 4 * (k - len(out))
        ranks = rng.choice(len(probs), size=need, p=probs)
        for r in ranks:
            f = int(rank_to_fact[r])
            if f not in seen:
                seen.add(f)
                out.append(f)
                if len(out) == k:
                    break
    return np.array(out, dtype=np.int32)


def make_batch(rng, ids_per_request, start_pos, block_size, num_blocks, max_blocks):
    """Requests get disjoint block sets from one seeded shuffle of all blocks."""
    R = len(ids_per_request)
    perm = rng.permutation(num_blocks).astype(np.int32)
    if R * max_blocks > num_blocks:
        raise ValueError("cache too small for disjoint block tables")
    bt = perm[: R * max_blocks].reshape(R, max_blocks).copy()
    offs = np.zeros(R + 1, dtype=np.int32)
    offs[1:] = np.cumsum([len(x) for x in ids_per_request])
    ids = (np.concatenate(ids_per_request).astype(np.int32) if R
           else np.zeros(0, np.int32))
    sp = np.broadcast_to(np.asarray(start_pos, dtype=np.int32), (R,)).copy()
    return Batch(offs, ids, sp, bt, block_size, num_blocks)


def tiny(seed: int = 0, start_pos: int = 32) -> Workload:
    """1 layer, 2 KV heads, D=64; 64 facts of 8-24 tokens; one request, k=5."""
    rng = np.random.default_rng(seed)
    lens = uniform_lengths(rng, 64, 8, 24)
    ids = distinct_ids(rng, 64, 5)
    batch = make_batch(rng, [ids], start_pos, 16, 64, 64)
    return Workload("tiny", TINY, lens, batch, seed)


def llama_single(seed: int = 0, num_facts: int = 10_000, k: int = 5,
                 num_blocks: int = 64) -> Workload:
    """Llama-3.1-8B shapes; 10k facts of 16-64 tokens; one request, k=5 at 64."""
    rng = np.random.default_rng(seed)
    lens = uniform_lengths(rng, num_facts, 16, 64)
    ids = distinct_ids(rng, num_facts, k)
    batch = make_batch(rng, [ids], 64, 16, num_blocks, num_blocks)
    return Workload("llama3.1-8b R=1 k=5", LLAMA31_8B, lens, batch, seed)


def llama_batch(seed: int = 0, num_facts: int = 10_000, R: int = 100, k: int = 50,
                slots_per_request: int = 4096, distinct_batch: bool = False) -> Workload:
    """Llama-3.1-8B shapes; 100 requests x k=50 distinct facts after a 64-token
    prefix, each request owning 4096 slots (256 blocks) of a shuffled cache.
    distinct_batch: no fact repeats anywhere in the batch (R * k ids drawn
    without replacement)."""
    rng = np.random.default_rng(seed)
    lens = uniform_lengths(rng, num_facts, 16, 64)
    if distinct_batch:
        ids = list(distinct_ids(rng, num_facts, R * k).reshape(R, k))
    else:
        ids = [distinct_ids(rng, num_facts, k) for _ in range(R)]
    mb = slots_per_request // 16
    batch = make_batch(rng, ids, 64, 16, R * mb, mb)
    return Workload(f"llama3.1-8b R={R} k={k}", LLAMA31_8B, lens, batch, seed)


def sweep(model: Model, R: int, k: int, seed: int = 0, num_facts: int = 50_000) -> Workload:
    """Mistral / Qwen sweep point: lognormal lengths (median 32, sigma 0.5,
    clamped to 8..96), cache sized to what each request needs."""
    rng = np.random.default_rng(seed)
    lens = lognormal_lengths(rng, num_facts)
    ids = [distinct_ids(rng, num_facts, k) for _ in range(R)]
    need = [-(-(64 + int(lens[x].sum())) // 16) for x in ids]
    mb = max(need) if need else 1
    batch = make_batch(rng, ids, 64, 16, R * mb, mb)
    return Workload(f"{model.name} R={R} k={k}", model, lens, batch, seed)


def offload(seed: int = 0, num_facts: int = 100_000, R: int = 100, k: int = 50,
            zipf_s: float = 1.1, hot_fraction: float = 0.2,
            slots_per_request: int = 4096, extra_batches: int = 0) -> Workload:
    """Qwen2.5-7B shapes; facts of 16..48 tokens (mean 32) in pinned host
    memory; requests draw k distinct facts by Zipf(zipf_s) over a seeded rank
    order; the hot set is the top hot_fraction of facts by rank.  The hot fact
    ids go to notes["hot"]; notes["more_ids"] holds extra_batches further
    draws of the same shape (CSR ids, same offsets) for streams of batches."""
    rng = np.random.default_rng(seed)
    lens = uniform_lengths(rng, num_facts, 16, 48)
    rank_to_fact = rng.permutation(num_facts).astype(np.int32)
    w = np.arange(1, num_facts + 1, dtype=np.float64) ** -zipf_s
    probs = w / w.sum()
    ids = [zipf_distinct_ids(rng, rank_to_fact, probs, k) for _ in range(R)]
    mb = slots_per_request // 16
    batch = make_batch(rng, ids, 64, 16, R * mb, mb)
    n_hot = int(round(hot_fraction * num_facts))
    more = [np.concatenate([zipf_distinct_ids(rng, rank_to_fact, probs, k) for _ in range(R)])
            for _ in range(extra_batches)]
    return Workload(f"{QWEN25_7B.name} offload R={R} k={k}", QWEN25_7B, lens, batch, seed,
                    notes=dict(hot=rank_to_fact[:n_hot].copy(), zipf_s=zipf_s,
                               hot_fraction=hot_fraction, more_ids=more))


# ---------------------------------------------------------------------------
# Device-side bulk fill (same definition as bf16_bits), for full-size inputs
# ---------------------------------------------------------------------------

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "csrc", "fill.cu")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        cmd = ["nvcc", "-O3", "-shared", "-Xcompiler", "-fPIC", "-lineinfo",
               "-gencode", "arch=compute_100a,code=sm_100a", "-o", _LIB_PATH, src]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.synth_fill_bf16.restype = ctypes.c_int
        _lib.synth_fill_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                         ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    return _lib


def fill_device(ptr: int, count: int, seed: int, stream: int, base: int = 0,
                cuda_stream: int = 0) -> None:
    """Fill ``count`` bf16 values at device address ``ptr`` with elements
    base .. base+count of the given stream (asynchronous on ``cuda_stream``)."""
    first, q = normal_table()
    rc = _load().synth_fill_bf16(ctypes.c_void_p(ptr), count, seed, stream, base,
                                 q.ctypes.data, len(q), first, ctypes.c_void_p(cuda_stream))
    if rc != 0:
        raise RuntimeError(f"synth_fill_bf16 failed: cuda error {rc}")
