"""Device-side inputs of a seeded synthetic workload: a FactStore holding
its facts, a paged cache pre-filled with seeded values, the batch's index
arrays as device tensors.  Used by the GPU tests, the smoke check and the
benchmark.

Input construction only (the generator of this package, then marshalling
into the library's store); no part of the inject arithmetic lives here.
The library is imported when a store is built, never at import time, so
the host-side generator stays importable without it.
"""
from __future__ import annotations

import numpy as np
import torch

import synth

CACHE_FILL_SEED = 7


def rope_of(model: synth.Model, style: int = 0):
    from kv_cache_injection_gather_b200 import RopeConfig
    return RopeConfig(theta=model.rope_theta, style=style, llama3=model.scaling())


def make_store(wl: synth.Workload, style: int = 0, on_device_gen: bool | None = None,
               device: int = 0, extra_tokens: int = 0, small_limit: int | None = None,
               heads: tuple[int, int] | None = None, facts=None, **limits):
    """Put every fact of the workload, in id order (ids equal indices).

    Small stores are generated on the host (numpy) and copied; large ones are
    generated on the device by the same counter-based definition.  heads =
    (h0, h1) keeps KV heads [h0, h1) of every fact (a head-sharded store; the
    workload's model then names the full head count).  facts = increasing
    global ids keeps only those facts, local id i holding facts[i] (a
    fact-sharded store)."""
    from kv_cache_injection_gather_b200 import FactStore
    full = wl.model
    m = full if heads is None else synth.Model(full.name, full.num_layers, heads[1] - heads[0],
                                               full.head_dim, full.rope_theta, full.llama3)
    ids = np.arange(len(wl.fact_lens)) if facts is None else np.asarray(facts, np.int64)
    total = int(wl.fact_lens[ids].sum()) + extra_tokens
    store = FactStore(m.num_layers, m.num_kv_heads, m.head_dim, rope_of(m, style), max(total, 1),
                      max(len(ids), 1), device=device, **limits)
    if small_limit is not None:  # 0: always the plan + inject kernels
        store.set_small_batch_limit(small_limit)
    if on_device_gen is None:
        on_device_gen = total * m.bytes_per_token > (64 << 20)
    dev = torch.device("cuda", device)
    if on_device_gen:
        maxlen = int(wl.fact_lens.max())
        kbuf = torch.empty(full.num_layers * full.num_kv_heads * maxlen * full.head_dim,
                           dtype=torch.bfloat16, device=dev)
        vbuf = torch.empty_like(kbuf)
        stream = torch.cuda.current_stream(dev).cuda_stream
        for i, f in enumerate(ids):
            f, n = int(f), int(wl.fact_lens[f])
            cnt = full.num_layers * full.num_kv_heads * n * full.head_dim
            synth.fill_device(kbuf.data_ptr(), cnt, wl.seed, synth.fact_stream(f, False), 0, stream)
            synth.fill_device(vbuf.data_ptr(), cnt, wl.seed, synth.fact_stream(f, True), 0, stream)
            shape = (full.num_layers, full.num_kv_heads, n, full.head_dim)
            k, v = kbuf[:cnt].view(shape), vbuf[:cnt].view(shape)
            if heads is not None:
                k, v = k[:, heads[0]:heads[1]], v[:, heads[0]:heads[1]]
            fid = store.put_fact(k, v)
            assert fid == i
        torch.cuda.synchronize(dev)
    else:
        for i, f in enumerate(ids):
            f, n = int(f), int(wl.fact_lens[f])
            k, v = synth.fact_kv(wl.seed, f, full.num_layers, full.num_kv_heads, n, full.head_dim)
            if heads is not None:
                k, v = k[:, heads[0]:heads[1]], v[:, heads[0]:heads[1]]
            k, v = np.ascontiguousarray(k), np.ascontiguousarray(v)
            kt = torch.from_numpy(k.view(np.int16)).view(torch.bfloat16)
            vt = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16)
            assert store.put_fact(kt, vt) == i
    return store


def cache_shape(wl: synth.Workload, head_major: bool = False):
    m, b = wl.model, wl.batch
    if head_major:
        return (m.num_layers, b.num_blocks, m.num_kv_heads, b.block_size, m.head_dim)
    return (m.num_layers, b.num_blocks, b.block_size, m.num_kv_heads, m.head_dim)


def make_cache(wl: synth.Workload, device: int = 0, fill: bool = True, head_major: bool = False,
               num_kv_heads: int | None = None):
    """K and V caches (bf16, device); filled with seeded values so untouched
    slots can be checked, or left uninitialised.  num_kv_heads overrides the
    model's (a head-sharded cache)."""
    from kv_cache_injection_gather_b200 import cache_desc
    shape = list(cache_shape(wl, head_major))
    if num_kv_heads is not None:
        shape[2 if head_major else 3] = num_kv_heads
    shape = tuple(shape)
    dev = torch.device("cuda", device)
    k = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    v = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    if fill:
        stream = torch.cuda.current_stream(dev).cuda_stream
        synth.fill_device(k.data_ptr(), k.numel(), CACHE_FILL_SEED, synth.TAG_CACHE | 0, 0, stream)
        synth.fill_device(v.data_ptr(), v.numel(), CACHE_FILL_SEED, synth.TAG_CACHE | 1, 0, stream)
    return k, v, cache_desc(k, v, head_major)


def batch_tensors(batch: synth.Batch, device: int = 0):
    dev = torch.device("cuda", device)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)  # noqa: E731
    return (t(batch.req_offsets), t(batch.fact_ids), t(batch.start_pos), t(batch.block_tables))


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)
