"""Torch-facing convenience over the C-ABI (marshalling only).

``FactStore`` owns one ``is_store_t``; tensors are passed to the library as
raw device pointers with their strides checked here.  Every byte of the
inject path is produced by the CUDA kernels in libinjectstore.so.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import binding as B


@dataclass
class RopeConfig:
    theta: float
    style: int = B.IS_ROPE_ROTATE_HALF
    llama3: dict | None = None   # factor, low_freq_factor, high_freq_factor, original_max_position


def _i32(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype != torch.int32 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous int32 tensor")
    return t


class _DeviceArray:
    """__cuda_array_interface__ wrapper so torch can view library memory."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = dict(shape=tuple(shape), typestr=typestr,
                                             data=(ptr, False), version=3, strides=None)


def cache_desc(k_cache: torch.Tensor, v_cache: torch.Tensor, head_major: bool = False) -> B.is_cache_t:
    """Describe bf16 caches shaped [L][num_blocks][B][H][D] (token-major) or
    [L][num_blocks][H][B][D] (head-major) to the library."""
    for t in (k_cache, v_cache):
        if t.dtype != torch.bfloat16 or t.dim() != 5 or not t.is_cuda or t.stride(-1) != 1:
            raise ValueError("caches must be CUDA bf16 [L][num_blocks][.][.][D] with unit last stride")
    if k_cache.shape != v_cache.shape or k_cache.stride() != v_cache.stride():
        raise ValueError("K and V caches must share shape and strides")
    L, nb, a, b, D = k_cache.shape
    ls, bs, sa, sb, _ = k_cache.stride()
    if head_major:
        H, blk, hs, ts = a, b, sa, sb
    else:
        blk, H, ts, hs = a, b, sa, sb
    return B.is_cache_t(k_cache.data_ptr(), v_cache.data_ptr(), ls, bs, ts, hs, nb, blk)


class FactStore:
    """A GPU-resident fact store of pre-RoPE keys and raw values."""

    def __init__(self, num_layers: int, num_kv_heads: int, head_dim: int, rope: RopeConfig,
                 capacity_tokens: int, max_facts: int, device: int = 0,
                 max_batch_requests: int = 0, max_batch_fact_ids: int = 0,
                 max_batch_blocks: int = 0, host_tier: bool = False, hot_capacity_tokens: int = 0):
        cfg = B.is_store_config_t()
        cfg.num_layers, cfg.num_kv_heads, cfg.head_dim = num_layers, num_kv_heads, head_dim
        cfg.rope_style, cfg.rope_theta = rope.style, rope.theta
        if rope.llama3:
            cfg.rope_scaling = B.IS_SCALING_LLAMA3
            cfg.scale_factor = rope.llama3["factor"]
            cfg.low_freq_factor = rope.llama3["low_freq_factor"]
            cfg.high_freq_factor = rope.llama3["high_freq_factor"]
            cfg.original_max_position = int(rope.llama3["original_max_position"])
        cfg.capacity_tokens, cfg.max_facts = capacity_tokens, max_facts
        cfg.max_batch_requests, cfg.max_batch_fact_ids = max_batch_requests, max_batch_fact_ids
        cfg.max_batch_blocks = max_batch_blocks
        cfg.tier = B.IS_TIER_HOST if host_tier else B.IS_TIER_DEVICE
        cfg.hot_capacity_tokens = hot_capacity_tokens
        self.L, self.H, self.D = num_layers, num_kv_heads, head_dim
        self.device = device
        self.capacity_tokens = capacity_tokens
        self.handle = B.is_store_create(cfg, device)

    # ---- lifetime
    def close(self) -> None:
        if getattr(self, "handle", None):
            B.is_store_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # ---- facts
    def put_fact(self, k_pre: torch.Tensor, v: torch.Tensor) -> int:
        """k_pre, v: bf16 [L][H][len][D] on the host or this device."""
        if k_pre.shape != v.shape or k_pre.dim() != 4 or k_pre.shape[0] != self.L \
                or k_pre.shape[1] != self.H or k_pre.shape[3] != self.D:
            raise ValueError("fact must be [L][H][len][D]")
        if k_pre.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
            raise ValueError("fact tensors must be bf16")
        k_pre, v = k_pre.contiguous(), v.contiguous()
        return B.is_store_put_fact(self.handle, k_pre.data_ptr(), v.data_ptr(), k_pre.shape[2])

    def put_fact_window(self, k_pre: torch.Tensor, v: torch.Tensor, window_len: int) -> int:
        """K/V of an encoded [window | fact], bf16 [L][H][window_len + len][D]:
        store only the fact's tokens (context-window encoding)."""
        if k_pre.shape != v.shape or k_pre.dim() != 4 or k_pre.shape[0] != self.L \
                or k_pre.shape[1] != self.H or k_pre.shape[3] != self.D:
            raise ValueError("encoding must be [L][H][window_len + len][D]")
        if k_pre.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
            raise ValueError("tensors must be bf16")
        n = k_pre.shape[2] - window_len
        if window_len < 0 or n <= 0:
            raise ValueError("window_len must leave at least one fact token")
        k_pre, v = k_pre.contiguous(), v.contiguous()
        return B.is_store_put_fact_window(self.handle, k_pre.data_ptr(), v.data_ptr(),
                                          window_len, n)

    @property
    def num_facts(self) -> int:
        return B.is_store_num_facts(self.handle)

    def fact_info(self, fact_id: int) -> tuple[int, int]:
        return B.is_store_fact_info(self.handle, fact_id)

    def read_fact(self, fact_id: int) -> tuple[torch.Tensor, torch.Tensor]:
        _, n = self.fact_info(fact_id)
        dev = torch.device("cuda", self.device)
        k = torch.empty((self.L, self.H, n, self.D), dtype=torch.bfloat16, device=dev)
        v = torch.empty_like(k)
        B.is_store_read_fact(self.handle, fact_id, k.data_ptr(), v.data_ptr())
        return k, v

    def arena(self) -> tuple[torch.Tensor, torch.Tensor]:
        """Views of the K and V arenas as bf16 [L][H][capacity_tokens][D]."""
        kp, vp, t = B.is_store_arena(self.handle)
        shape = (self.L, self.H, t, self.D)
        dev = torch.device("cuda", self.device)
        k = torch.as_tensor(_DeviceArray(kp, shape, "<i2"), device=dev).view(torch.bfloat16)
        v = torch.as_tensor(_DeviceArray(vp, shape, "<i2"), device=dev).view(torch.bfloat16)
        return k, v

    # ---- fact-sharded view
    def export(self) -> tuple[bytes, bytes, int]:
        """IPC handles of the K and V arenas (for peers' is_ipc_open) and the
        plane stride in tokens."""
        return B.is_store_export(self.handle)

    def arena_ptrs(self) -> tuple[int, int, int]:
        """Device addresses of the K and V arenas and the plane stride."""
        return B.is_store_arena(self.handle)

    def attach_shards(self, arenas, fact_shard, fact_offset, fact_len) -> None:
        """arenas: [(k_ptr, v_ptr, plane_tokens)] per shard; the global fact
        table as three host sequences.  Batches then take global fact ids."""
        B.is_store_attach_shards(self.handle, [a[0] for a in arenas], [a[1] for a in arenas],
                                 [a[2] for a in arenas], fact_shard, fact_offset, fact_len)

    def detach_shards(self) -> None:
        B.is_store_detach_shards(self.handle)

    def shard_info(self) -> tuple[int, int]:
        """(shards, global facts) of the attached view; (0, 0) when none."""
        return B.is_store_shard_info(self.handle)

    def set_hot(self, fact_ids) -> None:
        """Host tier: keep these facts (host int sequence) in the HBM hot arenas."""
        import numpy as np
        ids = np.ascontiguousarray(np.asarray(fact_ids, dtype=np.int32))
        B.is_store_set_hot(self.handle, ids.ctypes.data, ids.size)

    def set_hot_policy(self, lru: bool, slot_tokens: int = 0) -> None:
        """Host tier: LRU hot set with slots of slot_tokens, or back to static."""
        B.is_store_set_hot_policy(self.handle, B.IS_HOT_LRU if lru else B.IS_HOT_STATIC,
                                  slot_tokens)

    def touch(self, fact_ids, stream: int | None = None) -> int:
        """LRU: promote these facts (host ints) on the stream; returns how many."""
        import numpy as np
        ids = np.ascontiguousarray(np.asarray(fact_ids, dtype=np.int32))
        if stream is None:
            stream = torch.cuda.current_stream(self.device).cuda_stream
        return B.is_store_touch(self.handle, ids.ctypes.data, ids.size, stream)

    def lru_stats(self) -> dict:
        h, m, p, t = B.is_store_lru_stats(self.handle)
        return dict(hits=h, misses=m, promoted=p, promoted_tokens=t)

    def tier_info(self) -> dict:
        t, cap, used, nf = B.is_store_tier_info(self.handle)
        return dict(tier=t, hot_capacity=cap, hot_used=used, hot_facts=nf)

    # ---- the hot path
    def inject(self, req_offsets: torch.Tensor, fact_ids: torch.Tensor, start_pos: torch.Tensor,
               block_tables: torch.Tensor, cache: B.is_cache_t,
               slot_mapping: torch.Tensor | None = None, stream: int | None = None) -> None:
        """Asynchronous inject of one batch; all index tensors on the device."""
        _i32(req_offsets, "req_offsets"), _i32(fact_ids, "fact_ids")
        _i32(start_pos, "start_pos"), _i32(block_tables, "block_tables")
        R = start_pos.numel()
        if block_tables.dim() != 2 or block_tables.shape[0] != R:
            raise ValueError("block_tables must be [R][max_blocks]")
        if slot_mapping is not None and (slot_mapping.dtype != torch.int64 or not slot_mapping.is_contiguous()):
            raise ValueError("slot_mapping must be contiguous int64")
        if stream is None:
            stream = torch.cuda.current_stream(self.device).cuda_stream
        B.is_inject_batch(self.handle, R, req_offsets.data_ptr(), fact_ids.data_ptr(),
                          fact_ids.numel(), start_pos.data_ptr(), block_tables.data_ptr(),
                          block_tables.shape[1], cache,
                          None if slot_mapping is None else slot_mapping.data_ptr(),
                          0 if slot_mapping is None else slot_mapping.numel(), stream)

    def inject_host(self, req_offsets: torch.Tensor, fact_ids: torch.Tensor,
                    start_pos: torch.Tensor, block_tables: torch.Tensor, cache: B.is_cache_t,
                    slot_mapping: torch.Tensor | None = None, stream: int | None = None,
                    next_fact_ids: torch.Tensor | None = None) -> int:
        """Index tensors in host memory (pinned for asynchronous copies);
        waits and returns the batch status.  next_fact_ids (host int32): the
        next batch's ids, whose cold facts an LRU host-tier store prefetches
        into HBM while this batch runs."""
        for t in (req_offsets, fact_ids, start_pos, block_tables):
            if t.is_cuda:
                raise ValueError("inject_host takes host tensors")
        if stream is None:
            stream = torch.cuda.current_stream(self.device).cuda_stream
        args = (self.handle, start_pos.numel(), req_offsets.data_ptr(), fact_ids.data_ptr(),
                fact_ids.numel(), start_pos.data_ptr(), block_tables.data_ptr(),
                block_tables.shape[1], cache,
                None if slot_mapping is None else slot_mapping.data_ptr(),
                0 if slot_mapping is None else slot_mapping.numel())
        if next_fact_ids is None:
            return B.is_inject_batch_host(*args, stream)
        nxt = _i32(next_fact_ids, "next_fact_ids")
        if nxt.is_cuda:
            raise ValueError("next_fact_ids is a host tensor")
        return B.is_inject_batch_host_next(*args, nxt.data_ptr(), nxt.numel(), stream)

    def last_error(self, stream: int | None = None) -> tuple[int, int]:
        if stream is None:
            stream = torch.cuda.current_stream(self.device).cuda_stream
        return B.is_last_error(self.handle, stream)

    def last_error_timeout(self, timeout_ms: int, stream: int | None = None) -> tuple[int, int]:
        """As last_error, waiting at most timeout_ms (IS_ERR_TIMEOUT otherwise)."""
        if stream is None:
            stream = torch.cuda.current_stream(self.device).cuda_stream
        return B.is_last_error_timeout(self.handle, stream, timeout_ms)

    def set_small_batch_limit(self, max_requests: int) -> None:
        """Batches up to max_requests (<= 32) requests and 256 ids run as one
        kernel; 0: never."""
        B.is_store_set_small_batch_limit(self.handle, max_requests)

    def set_timing(self, enable: bool) -> None:
        B.is_store_set_timing(self.handle, enable)

    def kernel_time(self) -> tuple[float, int]:
        return B.is_store_kernel_time(self.handle)
