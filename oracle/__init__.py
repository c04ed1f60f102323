"""CPU oracle for the InferScale retrieve-and-inject path (numpy wrapper).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline leg, never by the product package.  The
arithmetic lives in ``inject_oracle.c`` (plain C, fp64); this module compiles
it with gcc, marshals numpy arrays and holds no arithmetic of its own.

Functions and the passages they follow (summaries of "InferScale: GPU-Native
KV Injection for Personalized LLM Serving", gist.science/{ja,nl,it}/paper/
2607.27090, technical summary, "Methodology -- 2. Online phase"):

* ``Store`` / ``Store.put``     -- Pre-RoPE storage (keys captured before RoPE,
                                   stored with raw values on the GPU).
* ``rope_inv_freq``, ``rope_rows`` -- Dynamic rotation (RoPE for the new
                                   serving position; standard RoPE frequencies,
                                   Llama-3.1 scaling where configured).
* ``segment``                   -- the retrieved facts composed into one
                                   contiguous segment.
* ``inject_batch``              -- Injection: scatter-copy into the paged KV
                                   cache.

Every function is pinned by ``tests/test_oracle_pins.py``; none is "parity
unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "inject_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

OK, ERR_INVALID_ARG, ERR_BAD_FACT_ID, ERR_POSITION, ERR_BAD_BLOCK, ERR_CAPACITY = 0, -1, -2, -3, -4, -5

ROTATE_HALF, INTERLEAVED = 0, 1

_P = ctypes.c_void_p
_I32, _I64, _F64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double


class _StoreC(ctypes.Structure):
    _fields_ = [("L", _I32), ("H", _I32), ("D", _I32), ("T_cap", _I64), ("T_used", _I64),
                ("num_facts", _I32), ("max_facts", _I32), ("k", _P), ("v", _P),
                ("off", _P), ("len", _P)]


class _CacheC(ctypes.Structure):
    _fields_ = [("k", _P), ("v", _P), ("k_ref", _P), ("layer_stride", _I64),
                ("block_stride", _I64), ("token_stride", _I64), ("head_stride", _I64),
                ("num_blocks", _I32), ("block_size", _I32)]


def build(force: bool = False) -> str:
    """Compile the oracle (gcc, -O2, OpenMP) into oracle/liboracle.so."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", tmp, _SRC, "-lm"],
                       check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    # ORACLE_LIB names a different build of inject_oracle.c; the mutation
    # tests use it to check that the pins catch planted mistakes.
    lib = ctypes.CDLL(os.environ.get("ORACLE_LIB") or build())
    lib.orc_bf16_to_f64_array.argtypes = [_P, _P, _I64]
    lib.orc_f64_to_bf16_array.argtypes = [_P, _P, _I64]
    lib.orc_llama3_scale.restype = _F64
    lib.orc_llama3_scale.argtypes = [_F64, _F64, _F64, _F64, _F64]
    lib.orc_rope_inv_freq.restype = ctypes.c_int
    lib.orc_rope_inv_freq.argtypes = [ctypes.c_int, _F64, ctypes.c_int, _F64, _F64, _F64, _F64, _P]
    lib.orc_rope_rows.argtypes = [_P, _P, _I64, ctypes.c_int, _P, _P, ctypes.c_int]
    lib.orc_store_put.restype = _I32
    lib.orc_store_put.argtypes = [ctypes.POINTER(_StoreC), _P, _P, _I32]
    lib.orc_slot.restype = _I64
    lib.orc_slot.argtypes = [_P, _I32, _I32, _I32, _I64]
    lib.orc_segment.restype = _I64
    lib.orc_segment.argtypes = [ctypes.POINTER(_StoreC), _I32, _P, _P, _I32, _P, _P, _I32, _I32,
                                _I32, _I64, _P, _P, _P, _P, ctypes.POINTER(ctypes.c_int)]
    lib.orc_inject_batch.restype = ctypes.c_int
    lib.orc_inject_batch.argtypes = [ctypes.POINTER(_StoreC), ctypes.c_int, _P, _I32, _P, _P, _I32,
                                     _P, _P, _I32, ctypes.POINTER(_CacheC), _P, _I64,
                                     ctypes.c_int]
    lib.orc_max_threads.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


def max_threads() -> int:
    return int(_load().orc_max_threads())


# ------------------------------------------------------------------- bf16

def bf16_to_f64(bits) -> np.ndarray:
    b = _c(bits, np.uint16)
    out = np.empty(b.shape, np.float64)
    _load().orc_bf16_to_f64_array(_ptr(b), _ptr(out), b.size)
    return out


def f64_to_bf16(x) -> np.ndarray:
    """Round fp64 values to bf16 bit patterns, nearest, ties to even (one step)."""
    a = _c(x, np.float64)
    out = np.empty(a.shape, np.uint16)
    _load().orc_f64_to_bf16_array(_ptr(a), _ptr(out), a.size)
    return out


# ------------------------------------------------------------------- RoPE

def llama3_scale(freq: float, factor=8.0, low=1.0, high=4.0, orig=8192.0) -> float:
    return float(_load().orc_llama3_scale(freq, factor, low, high, orig))


def rope_inv_freq(head_dim: int, theta: float, scaling: dict | None = None) -> np.ndarray:
    out = np.empty(head_dim // 2, np.float64)
    if scaling is None:
        rc = _load().orc_rope_inv_freq(head_dim, theta, 0, 1.0, 1.0, 1.0, 1.0, _ptr(out))
    else:
        rc = _load().orc_rope_inv_freq(head_dim, theta, 1, scaling["factor"],
                                       scaling["low_freq_factor"], scaling["high_freq_factor"],
                                       float(scaling["original_max_position"]), _ptr(out))
    if rc != OK:
        raise ValueError(f"rope_inv_freq: status {rc}")
    return out


def rope_rows(x, pos, inv_freq, style: int = ROTATE_HALF) -> np.ndarray:
    """Rotate rows x[..., D] (fp64) to positions pos[...] (int)."""
    x = _c(x, np.float64)
    D = x.shape[-1]
    p = _c(np.broadcast_to(np.asarray(pos, dtype=np.int64), x.shape[:-1]), np.int64)
    f = _c(inv_freq, np.float64)
    y = np.empty_like(x)
    _load().orc_rope_rows(_ptr(x), _ptr(y), x.size // D, D, _ptr(p), _ptr(f), style)
    return y


# ------------------------------------------------------------- fact store

class Store:
    """The fact store: K and V planes bf16 [L][H][T_cap][D], offsets, lengths."""

    def __init__(self, L: int, H: int, D: int, capacity_tokens: int, max_facts: int):
        self.L, self.H, self.D = L, H, D
        self.k = np.zeros((L, H, capacity_tokens, D), np.uint16)
        self.v = np.zeros((L, H, capacity_tokens, D), np.uint16)
        self.off = np.zeros(max_facts, np.int64)
        self.len = np.zeros(max_facts, np.int32)
        self._c = _StoreC(L, H, D, capacity_tokens, 0, 0, max_facts, _ptr(self.k), _ptr(self.v),
                          _ptr(self.off), _ptr(self.len))

    @property
    def num_facts(self) -> int:
        return int(self._c.num_facts)

    def put(self, k_pre, v) -> int:
        """Append one fact (bf16 bits [L][H][len][D]); returns its id."""
        k = _c(k_pre, np.uint16)
        v = _c(v, np.uint16)
        if k.shape != v.shape or k.shape[:2] != (self.L, self.H) or k.shape[3] != self.D:
            raise ValueError("fact shape mismatch")
        fid = int(_load().orc_store_put(ctypes.byref(self._c), _ptr(k), _ptr(v), k.shape[2]))
        if fid < 0:
            raise ValueError(f"put: status {fid}")
        return fid


def slot(bt_row, block_size: int, num_blocks: int, pos: int) -> int:
    bt = _c(bt_row, np.int32)
    return int(_load().orc_slot(_ptr(bt), bt.size, block_size, num_blocks, pos))


def segment(store: Store, req_offsets, fact_ids, start_pos, block_tables, block_size: int,
            num_blocks: int):
    """Per-token (request, store token, position, slot) of a batch, and status."""
    ro, ids, sp = _c(req_offsets, np.int32), _c(fact_ids, np.int32), _c(start_pos, np.int32)
    bt = _c(block_tables, np.int32).reshape(len(sp), -1) if len(sp) else np.zeros((0, 1), np.int32)
    st = ctypes.c_int(0)
    n = int(_load().orc_segment(ctypes.byref(store._c), len(sp), _ptr(ro), _ptr(ids), ids.size,
                                _ptr(sp), _ptr(bt), bt.shape[1], block_size, num_blocks, 0, None,
                                None, None, None, ctypes.byref(st)))
    if n < 0:
        return None, int(st.value)
    req = np.empty(n, np.int32)
    src, pos, slt = (np.empty(n, np.int64) for _ in range(3))
    _load().orc_segment(ctypes.byref(store._c), len(sp), _ptr(ro), _ptr(ids), ids.size, _ptr(sp),
                        _ptr(bt), bt.shape[1], block_size, num_blocks, n, _ptr(req), _ptr(src),
                        _ptr(pos), _ptr(slt), ctypes.byref(st))
    return dict(request=req, src=src, pos=pos, slot=slt), int(st.value)


def cache_strides(num_blocks: int, block_size: int, H: int, D: int, head_major: bool = False):
    """Element strides (layer, block, token, head) of a dense paged cache,
    [L][num_blocks][B][H][D] (token-major) or [L][num_blocks][H][B][D]."""
    blk = block_size * H * D
    if head_major:
        return (num_blocks * blk, blk, D, block_size * D)
    return (num_blocks * blk, blk, H * D, D)


def inject_batch(store: Store, inv_freq, req_offsets, fact_ids, start_pos, block_tables,
                 k_cache, v_cache, block_size: int, strides=None, style: int = ROTATE_HALF,
                 k_ref=None, slot_capacity: int | None = None, num_threads: int = 0):
    """Run the whole inject on host arrays (k_cache / v_cache uint16, updated
    in place; k_ref optional float64 of the same shape).  Returns
    (status, slot_mapping)."""
    ro, ids, sp = _c(req_offsets, np.int32), _c(fact_ids, np.int32), _c(start_pos, np.int32)
    R = len(sp)
    bt = _c(block_tables, np.int32).reshape(R, -1) if R else np.zeros((0, 1), np.int32)
    assert k_cache.dtype == np.uint16 and k_cache.flags.c_contiguous
    assert v_cache.dtype == np.uint16 and v_cache.flags.c_contiguous
    num_blocks = k_cache.shape[1]
    if strides is None:
        strides = cache_strides(num_blocks, block_size, store.H, store.D)
    if k_ref is not None:
        assert k_ref.dtype == np.float64 and k_ref.shape == k_cache.shape
    cache = _CacheC(_ptr(k_cache), _ptr(v_cache), _ptr(k_ref), *strides, num_blocks, block_size)
    seg, st0 = segment(store, ro, ids, sp, bt, block_size, num_blocks)
    n = 0 if seg is None else len(seg["pos"])
    cap = n if slot_capacity is None else slot_capacity
    slots = np.full(max(n, 1), -1, np.int64)
    f = _c(inv_freq, np.float64)
    rc = int(_load().orc_inject_batch(ctypes.byref(store._c), style, _ptr(f), R, _ptr(ro),
                                      _ptr(ids), ids.size, _ptr(sp), _ptr(bt), bt.shape[1],
                                      ctypes.byref(cache), _ptr(slots), cap, num_threads))
    return rc, slots[:n]
