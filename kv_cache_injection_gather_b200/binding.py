"""ctypes binding of libinjectstore.so (include/inject_store.h).

Argument marshalling only: every step of the inject path runs in the CUDA
library.  Pointers are plain integers (``tensor.data_ptr()``) and streams are
``torch.cuda.Stream.cuda_stream`` integers; no torch type crosses the C-ABI.
If the shared library is missing this module raises at import: there is no
fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libinjectstore.so")

IS_OK = 0
IS_ERR_INVALID_ARG = -1
IS_ERR_BAD_FACT_ID = -2
IS_ERR_POSITION = -3
IS_ERR_BAD_BLOCK = -4
IS_ERR_CAPACITY = -5
IS_ERR_OOM = -6
IS_ERR_CUDA = -7
IS_ERR_TIMEOUT = -8
IS_ERR_NOT_SUPPORTED = -9

IS_ROPE_ROTATE_HALF = 0
IS_ROPE_INTERLEAVED = 1
IS_SCALING_NONE = 0
IS_SCALING_LLAMA3 = 1
IS_TIER_DEVICE = 0
IS_TIER_HOST = 1
IS_HOT_STATIC = 0
IS_HOT_LRU = 1

IS_NOALLOC_MAX_REQUESTS = 1024
IS_NOALLOC_MAX_FACT_IDS = 65536
IS_NOALLOC_MAX_BLOCKS = 65536
IS_NOALLOC_MAX_HEAD_DIM = 256

_I32, _I64, _F64, _P = ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p


class is_store_config_t(ctypes.Structure):
    _fields_ = [
        ("num_layers", _I32), ("num_kv_heads", _I32), ("head_dim", _I32), ("rope_style", _I32),
        ("rope_theta", _F64), ("rope_scaling", _I32), ("scale_factor", _F64),
        ("low_freq_factor", _F64), ("high_freq_factor", _F64), ("original_max_position", _I32),
        ("capacity_tokens", _I64), ("max_facts", _I32), ("max_batch_requests", _I32),
        ("max_batch_fact_ids", _I32), ("max_batch_blocks", _I32), ("tier", _I32),
        ("hot_capacity_tokens", _I64),
    ]


class is_cache_t(ctypes.Structure):
    _fields_ = [
        ("k_cache", _P), ("v_cache", _P), ("layer_stride", _I64), ("block_stride", _I64),
        ("token_stride", _I64), ("head_stride", _I64), ("num_blocks", _I32), ("block_size", _I32),
    ]


class is_ipc_handle_t(ctypes.Structure):
    _fields_ = [("bytes", ctypes.c_ubyte * 64)]


class InjectError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m kv_cache_injection_gather_b200.build` "
        "(the inject path has no Python or CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

_SIGNATURES = {
    "is_store_create": (ctypes.c_int, [ctypes.POINTER(is_store_config_t), ctypes.c_int,
                                       ctypes.POINTER(_P)]),
    "is_store_destroy": (None, [_P]),
    "is_store_put_fact": (ctypes.c_int, [_P, _P, _P, _I32, ctypes.POINTER(_I32)]),
    "is_store_put_fact_window": (ctypes.c_int, [_P, _P, _P, _I32, _I32, ctypes.POINTER(_I32)]),
    "is_store_num_facts": (ctypes.c_int, [_P, ctypes.POINTER(_I32)]),
    "is_store_fact_info": (ctypes.c_int, [_P, _I32, ctypes.POINTER(_I64), ctypes.POINTER(_I32)]),
    "is_store_read_fact": (ctypes.c_int, [_P, _I32, _P, _P]),
    "is_store_arena": (ctypes.c_int, [_P, ctypes.POINTER(_P), ctypes.POINTER(_P),
                                      ctypes.POINTER(_I64)]),
    "is_inject_batch": (ctypes.c_int, [_P, _I32, _P, _P, _I32, _P, _P, _I32,
                                       ctypes.POINTER(is_cache_t), _P, _I64, _P]),
    "is_inject_batch_host": (ctypes.c_int, [_P, _I32, _P, _P, _I32, _P, _P, _I32,
                                            ctypes.POINTER(is_cache_t), _P, _I64, _P]),
    "is_inject_batch_host_next": (ctypes.c_int, [_P, _I32, _P, _P, _I32, _P, _P, _I32,
                                                 ctypes.POINTER(is_cache_t), _P, _I64, _P, _I32,
                                                 _P]),
    "is_last_error": (ctypes.c_int, [_P, _P, ctypes.POINTER(_I64)]),
    "is_last_error_timeout": (ctypes.c_int, [_P, _P, _I32, ctypes.POINTER(_I64)]),
    "is_store_set_timing": (ctypes.c_int, [_P, ctypes.c_int]),
    "is_store_set_small_batch_limit": (ctypes.c_int, [_P, _I32]),
    "is_store_kernel_time": (ctypes.c_int, [_P, ctypes.POINTER(_F64), ctypes.POINTER(_I64)]),
    "is_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "is_store_set_hot": (ctypes.c_int, [_P, _P, _I32]),
    "is_store_set_hot_policy": (ctypes.c_int, [_P, ctypes.c_int, _I32]),
    "is_store_touch": (ctypes.c_int, [_P, _P, _I32, _P, ctypes.POINTER(_I32)]),
    "is_store_lru_stats": (ctypes.c_int, [_P, ctypes.POINTER(_I64), ctypes.POINTER(_I64),
                                          ctypes.POINTER(_I64), ctypes.POINTER(_I64)]),
    "is_store_tier_info": (ctypes.c_int, [_P, ctypes.POINTER(_I32), ctypes.POINTER(_I64),
                                          ctypes.POINTER(_I64), ctypes.POINTER(_I32)]),
    "is_store_attach_shards": (ctypes.c_int, [_P, _I32, _P, _P, _P, _I32, _P, _P, _P]),
    "is_store_detach_shards": (ctypes.c_int, [_P]),
    "is_store_shard_info": (ctypes.c_int, [_P, ctypes.POINTER(_I32), ctypes.POINTER(_I32)]),
    "is_store_export": (ctypes.c_int, [_P, ctypes.POINTER(is_ipc_handle_t),
                                       ctypes.POINTER(is_ipc_handle_t), ctypes.POINTER(_I64)]),
    "is_ipc_open": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(is_ipc_handle_t),
                                   ctypes.POINTER(_P)]),
    "is_ipc_close": (ctypes.c_int, [ctypes.c_int, _P]),
    "is_inject_batch_noalloc": (ctypes.c_int, [ctypes.POINTER(is_store_config_t), _P, _P, _I64,
                                               _P, _P, _I32, _I32, _P, _P, _I32, _P, _P, _I32,
                                               ctypes.POINTER(is_cache_t), _P, _I64, _P, _P]),
}
for _name, (_res, _args) in _SIGNATURES.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def lib() -> ctypes.CDLL:
    return _lib


def status_string(status: int) -> str:
    return _lib.is_status_string(status).decode()


def check(status: int, where: str = "call") -> None:
    if status != IS_OK:
        raise InjectError(status, where)


# ---- the C-ABI, same names -------------------------------------------------

def is_store_create(cfg: is_store_config_t, device: int = 0) -> int:
    out = _P()
    check(_lib.is_store_create(ctypes.byref(cfg), device, ctypes.byref(out)), "is_store_create")
    return out.value


def is_store_destroy(store: int) -> None:
    _lib.is_store_destroy(store)


def is_store_put_fact(store: int, k_pre_ptr: int, v_ptr: int, length: int) -> int:
    fid = _I32()
    check(_lib.is_store_put_fact(store, k_pre_ptr, v_ptr, length, ctypes.byref(fid)),
          "is_store_put_fact")
    return fid.value


def is_store_put_fact_window(store: int, k_pre_ptr: int, v_ptr: int, window_len: int,
                             fact_len: int) -> int:
    fid = _I32()
    check(_lib.is_store_put_fact_window(store, k_pre_ptr, v_ptr, window_len, fact_len,
                                        ctypes.byref(fid)), "is_store_put_fact_window")
    return fid.value


def is_store_num_facts(store: int) -> int:
    n = _I32()
    check(_lib.is_store_num_facts(store, ctypes.byref(n)), "is_store_num_facts")
    return n.value


def is_store_fact_info(store: int, fact_id: int) -> tuple[int, int]:
    off, ln = _I64(), _I32()
    check(_lib.is_store_fact_info(store, fact_id, ctypes.byref(off), ctypes.byref(ln)),
          "is_store_fact_info")
    return off.value, ln.value


def is_store_read_fact(store: int, fact_id: int, k_out_ptr: int, v_out_ptr: int) -> None:
    check(_lib.is_store_read_fact(store, fact_id, k_out_ptr, v_out_ptr), "is_store_read_fact")


def is_store_arena(store: int) -> tuple[int, int, int]:
    k, v, t = _P(), _P(), _I64()
    check(_lib.is_store_arena(store, ctypes.byref(k), ctypes.byref(v), ctypes.byref(t)),
          "is_store_arena")
    return k.value, v.value, t.value


def is_store_attach_shards(store: int, k_arenas: list[int], v_arenas: list[int],
                           plane_tokens: list[int], fact_shard, fact_offset, fact_len) -> None:
    """fact_shard / fact_offset / fact_len: int32 / int64 / int32 sequences
    of one length (host; copied)."""
    n, nf = len(k_arenas), len(fact_shard)
    if len(v_arenas) != n or len(plane_tokens) != n or len(fact_offset) != nf or len(fact_len) != nf:
        raise ValueError("is_store_attach_shards: array lengths differ")
    ka = (_P * max(n, 1))(*k_arenas)
    va = (_P * max(n, 1))(*v_arenas)
    pt = (_I64 * max(n, 1))(*plane_tokens)
    fs = (_I32 * max(nf, 1))(*[int(x) for x in fact_shard])
    fo = (_I64 * max(nf, 1))(*[int(x) for x in fact_offset])
    fl = (_I32 * max(nf, 1))(*[int(x) for x in fact_len])
    check(_lib.is_store_attach_shards(store, n, ka, va, pt, nf, fs, fo, fl), "is_store_attach_shards")


def is_store_detach_shards(store: int) -> None:
    check(_lib.is_store_detach_shards(store), "is_store_detach_shards")


def is_store_shard_info(store: int) -> tuple[int, int]:
    n, nf = _I32(), _I32()
    check(_lib.is_store_shard_info(store, ctypes.byref(n), ctypes.byref(nf)), "is_store_shard_info")
    return n.value, nf.value


def is_store_export(store: int) -> tuple[bytes, bytes, int]:
    """(K handle, V handle, plane tokens); handles as 64-byte strings."""
    hk, hv, t = is_ipc_handle_t(), is_ipc_handle_t(), _I64()
    check(_lib.is_store_export(store, ctypes.byref(hk), ctypes.byref(hv), ctypes.byref(t)),
          "is_store_export")
    return bytes(hk.bytes), bytes(hv.bytes), t.value


def is_ipc_open(device: int, handle: bytes) -> int:
    if len(handle) != 64:
        raise ValueError("is_ipc_open: a handle is 64 bytes")
    h = is_ipc_handle_t()
    ctypes.memmove(h.bytes, handle, 64)
    out = _P()
    check(_lib.is_ipc_open(device, ctypes.byref(h), ctypes.byref(out)), "is_ipc_open")
    return out.value


def is_ipc_close(device: int, ptr: int) -> None:
    check(_lib.is_ipc_close(device, ptr), "is_ipc_close")


def is_inject_batch(store: int, num_requests: int, req_fact_offsets: int, fact_ids: int,
                    num_fact_ids: int, start_pos: int, block_tables: int,
                    max_blocks_per_req: int, cache: is_cache_t, slot_mapping_out: int | None,
                    slot_mapping_capacity: int, stream: int = 0) -> int:
    """Asynchronous; returns the host-side status (raises on error)."""
    rc = _lib.is_inject_batch(store, num_requests, req_fact_offsets, fact_ids, num_fact_ids,
                              start_pos, block_tables, max_blocks_per_req, ctypes.byref(cache),
                              slot_mapping_out, slot_mapping_capacity, stream)
    check(rc, "is_inject_batch")
    return rc


def is_inject_batch_host(store: int, num_requests: int, req_fact_offsets: int, fact_ids: int,
                         num_fact_ids: int, start_pos: int, block_tables: int,
                         max_blocks_per_req: int, cache: is_cache_t,
                         slot_mapping_out: int | None, slot_mapping_capacity: int,
                         stream: int = 0) -> int:
    """Host index arrays in, status out (waits for the stream).  Returns the
    batch status without raising, so callers can inspect device errors."""
    return _lib.is_inject_batch_host(store, num_requests, req_fact_offsets, fact_ids,
                                     num_fact_ids, start_pos, block_tables, max_blocks_per_req,
                                     ctypes.byref(cache), slot_mapping_out,
                                     slot_mapping_capacity, stream)


def is_inject_batch_host_next(store: int, num_requests: int, req_fact_offsets: int,
                              fact_ids: int, num_fact_ids: int, start_pos: int,
                              block_tables: int, max_blocks_per_req: int, cache: is_cache_t,
                              slot_mapping_out: int | None, slot_mapping_capacity: int,
                              next_fact_ids: int | None, num_next_ids: int,
                              stream: int = 0) -> int:
    """is_inject_batch_host, and on an LRU host-tier store the next batch's
    cold facts (host array) start moving into HBM while this batch runs.
    Returns the batch status without raising."""
    return _lib.is_inject_batch_host_next(store, num_requests, req_fact_offsets, fact_ids,
                                          num_fact_ids, start_pos, block_tables,
                                          max_blocks_per_req, ctypes.byref(cache),
                                          slot_mapping_out, slot_mapping_capacity,
                                          next_fact_ids, num_next_ids, stream)


def is_last_error(store: int, stream: int = 0) -> tuple[int, int]:
    detail = _I64()
    rc = _lib.is_last_error(store, stream, ctypes.byref(detail))
    return rc, detail.value


def is_last_error_timeout(store: int, stream: int, timeout_ms: int) -> tuple[int, int]:
    detail = _I64()
    rc = _lib.is_last_error_timeout(store, stream, timeout_ms, ctypes.byref(detail))
    return rc, detail.value


def is_store_set_small_batch_limit(store: int, max_requests: int) -> None:
    check(_lib.is_store_set_small_batch_limit(store, max_requests), "is_store_set_small_batch_limit")


def is_store_set_timing(store: int, enable: bool) -> None:
    check(_lib.is_store_set_timing(store, int(bool(enable))), "is_store_set_timing")


def is_store_kernel_time(store: int) -> tuple[float, int]:
    ms, n = _F64(), _I64()
    check(_lib.is_store_kernel_time(store, ctypes.byref(ms), ctypes.byref(n)),
          "is_store_kernel_time")
    return ms.value, n.value


def is_status_string(status: int) -> str:
    return status_string(status)


def is_store_set_hot(store: int, fact_ids_host_ptr: int, n: int) -> None:
    check(_lib.is_store_set_hot(store, fact_ids_host_ptr, n), "is_store_set_hot")


def is_store_set_hot_policy(store: int, policy: int, slot_tokens: int = 0) -> None:
    check(_lib.is_store_set_hot_policy(store, policy, slot_tokens), "is_store_set_hot_policy")


def is_store_touch(store: int, fact_ids_host_ptr: int, n: int, stream: int = 0) -> int:
    promoted = _I32()
    check(_lib.is_store_touch(store, fact_ids_host_ptr, n, stream, ctypes.byref(promoted)),
          "is_store_touch")
    return promoted.value


def is_store_lru_stats(store: int) -> tuple[int, int, int, int]:
    h, m, p, t = _I64(), _I64(), _I64(), _I64()
    check(_lib.is_store_lru_stats(store, ctypes.byref(h), ctypes.byref(m), ctypes.byref(p),
                                  ctypes.byref(t)), "is_store_lru_stats")
    return h.value, m.value, p.value, t.value


def is_store_tier_info(store: int) -> tuple[int, int, int, int]:
    t, cap, used, nf = _I32(), _I64(), _I64(), _I32()
    check(_lib.is_store_tier_info(store, ctypes.byref(t), ctypes.byref(cap), ctypes.byref(used),
                                  ctypes.byref(nf)), "is_store_tier_info")
    return t.value, cap.value, used.value, nf.value


def is_inject_batch_noalloc(cfg: is_store_config_t, k_store: int, v_store: int,
                            plane_tokens: int, fact_offsets: int, fact_lens: int, num_facts: int,
                            num_requests: int, req_fact_offsets: int, fact_ids: int,
                            num_fact_ids: int, start_pos: int, block_tables: int,
                            max_blocks_per_req: int, cache: is_cache_t,
                            slot_mapping_out: int | None, slot_mapping_capacity: int,
                            status_out: int | None, stream: int = 0) -> int:
    """The batch for callers that cannot allocate device memory: the store's
    arenas and fact table are passed in, the work space is the library's
    fixed device array.  Asynchronous; returns the host-side status
    without raising.  The device status lands in status_out (16 bytes)."""
    return _lib.is_inject_batch_noalloc(ctypes.byref(cfg), k_store, v_store, plane_tokens,
                                        fact_offsets, fact_lens, num_facts, num_requests,
                                        req_fact_offsets, fact_ids, num_fact_ids, start_pos,
                                        block_tables, max_blocks_per_req, ctypes.byref(cache),
                                        slot_mapping_out, slot_mapping_capacity, status_out,
                                        stream)
