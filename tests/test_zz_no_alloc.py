"""is_inject_batch_noalloc, the entry point for callers that cannot allocate
device memory (an engine whose memory pool owns the GPU, a region captured
into a CUDA graph, a plugin host that forbids hidden allocations), gives the
same cache, slot mapping and status as is_inject_batch on the same inputs.

Called through the C-ABI twice in a row with two different batches, so the
second call runs on the work space the first one left behind.  Collected
last (file name) so that a run stopping at the first failure has already run
every other test; it also passes alone in a fresh process.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from gpu_common import batch_tensors, make_cache, make_store, to_bits
from kv_cache_injection_gather_b200 import binding as B

pytestmark = pytest.mark.gpu

REL, ABS = 2.0 ** -8, 1e-3  # the K tolerance of the other GPU tests


def _batch(rng, lens, R, max_k, B_, starts):
    nf = len(lens)
    ids = [rng.choice(nf, int(rng.integers(1, max_k + 1)), replace=False) for _ in range(R)]
    need = max(-(-(int(starts[r]) + int(lens[ids[r]].sum())) // B_) for r in range(R)) + 2
    return synth.make_batch(rng, ids, starts, B_, R * need, need)


def test_no_alloc_matches_store_entry_point_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    rng = np.random.default_rng(2024)
    model = synth.Model("llama-like", 4, 8, 128, 5e5, llama3=True)
    lens = rng.integers(16, 65, 300).astype(np.int32)
    b1 = _batch(rng, lens, 12, 20, 16, rng.integers(0, 100, 12).astype(np.int32))
    b2 = _batch(rng, lens, 5, 30, 16, np.array([64, 0, 17, 300, 5], np.int32))
    wl = synth.Workload("noalloc", model, lens, b1, seed=3)
    store = make_store(wl)
    kp, vp, plane = B.is_store_arena(store.handle)
    info = [store.fact_info(f) for f in range(len(lens))]
    offs = torch.tensor([o for o, _ in info], dtype=torch.int64, device="cuda")
    lns = torch.tensor([n for _, n in info], dtype=torch.int32, device="cuda")
    cfg = B.is_store_config_t(num_layers=model.num_layers, num_kv_heads=model.num_kv_heads,
                              head_dim=model.head_dim, rope_theta=model.rope_theta,
                              rope_scaling=B.IS_SCALING_LLAMA3, scale_factor=8.0,
                              low_freq_factor=1.0, high_freq_factor=4.0,
                              original_max_position=8192)
    stream = torch.cuda.current_stream().cuda_stream
    status = torch.full((2,), -99, dtype=torch.int64, device="cuda")

    for batch in (b1, b2):
        wlb = synth.Workload("noalloc", model, lens, batch, seed=3)
        n_tok = wlb.tokens()
        ro, ids, sp, bt = batch_tensors(batch)
        # existing entry point
        k1, v1, d1 = make_cache(wlb)
        s1 = torch.empty(n_tok, dtype=torch.int64, device="cuda")
        store.inject(ro, ids, sp, bt, d1, s1)
        assert store.last_error()[0] == B.IS_OK
        # allocation-free entry point, same inputs, fresh caches with the same fill
        k2, v2, d2 = make_cache(wlb)
        s2 = torch.full((n_tok,), -5, dtype=torch.int64, device="cuda")
        rc = B.is_inject_batch_noalloc(cfg, kp, vp, plane, offs.data_ptr(), lns.data_ptr(),
                                       len(lens), batch.num_requests, ro.data_ptr(),
                                       ids.data_ptr(), ids.numel(), sp.data_ptr(), bt.data_ptr(),
                                       batch.max_blocks, d2, s2.data_ptr(), n_tok,
                                       status.data_ptr(), stream)
        assert rc == B.IS_OK
        torch.cuda.synchronize()
        assert int(status[0].item()) == 0, "device status not ok"
        assert torch.equal(s1, s2)
        assert torch.equal(v1, v2)
        f1 = (to_bits(k1).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        f2 = (to_bits(k2).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        assert np.all(np.abs(f2 - f1) <= REL * np.abs(f1) + ABS)

    # sizes beyond the fixed work space are refused before any launch
    ro, ids, sp, bt = batch_tensors(b1)
    rc = B.is_inject_batch_noalloc(cfg, kp, vp, plane, offs.data_ptr(), lns.data_ptr(),
                                   len(lens), B.IS_NOALLOC_MAX_REQUESTS + 1, ro.data_ptr(),
                                   ids.data_ptr(), ids.numel(), sp.data_ptr(), bt.data_ptr(),
                                   b1.max_blocks, d2, None, 0, None, stream)
    assert rc == B.IS_ERR_CAPACITY
    store.close()
