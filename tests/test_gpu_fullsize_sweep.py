"""Full-size parity at the other large configurations, in the launch
configuration the benchmark times (the checks of fullsize_check: every slot,
every row of K and V against the oracle request by request, every untouched
element):

  * Qwen2.5-7B shapes, 50k-fact store (~103 GB), 256 requests x k=50 (the
    plan + inject kernels) and, on the same store, 16 requests x k=10 (the
    single kernel, past two waves of units);
  * Mistral-7B shapes, 20k-fact store (~95 GB: 50k would not fit in HBM),
    100 requests x k=20 and 16 requests x k=5 alike;
  * the host tier: Qwen2.5-7B shapes, 10k facts of 16-48 tokens in pinned
    host memory with the top 20% by Zipf rank in the HBM hot set, 100
    requests x k=50 drawn Zipf(1.1) -- the offload configuration at a store
    size a test can allocate.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from fullsize_check import check_full_size
from synth.device import make_store

pytestmark = pytest.mark.gpu


def _room(wl, extra=8 << 30, host_store=False):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    m, b = wl.model, wl.batch
    dev = (0 if host_store else int(wl.fact_lens.sum())) + b.num_blocks * b.block_size
    need = dev * m.bytes_per_token
    free, _ = torch.cuda.mem_get_info()
    if free < need + extra:
        pytest.skip(f"needs {need / 1e9:.0f} GB free on the device")


@pytest.mark.parametrize("model,points,facts", [("qwen", [(256, 50), (16, 10)], 50_000),
                                                ("mistral", [(100, 20), (16, 5)], 20_000)])
def test_sweep_point_full_size(model, points, facts):
    m = synth.QWEN25_7B if model == "qwen" else synth.MISTRAL_7B
    wls = [synth.sweep(m, R, k, 0, num_facts=facts) for R, k in points]
    # the sweep draws its fact lengths first: every point uses the same pool
    assert all(np.array_equal(w.fact_lens, wls[0].fact_lens) for w in wls)
    _room(wls[0])
    store = make_store(wls[0], on_device_gen=True)
    try:
        for wl in wls:
            check_full_size(wl, store)
            torch.cuda.empty_cache()
    finally:
        store.close()
        torch.cuda.empty_cache()


def test_host_tier_offload_full_batch():
    wl = synth.offload(0, num_facts=10_000)
    _room(wl, host_store=True)
    hot = np.asarray(wl.notes["hot"], np.int32)
    hot_tokens = int(wl.fact_lens[hot].sum())
    store = make_store(wl, on_device_gen=True, host_tier=True, hot_capacity_tokens=hot_tokens)
    try:
        store.set_hot(hot)
        info = store.tier_info()
        assert info["hot_facts"] == len(hot)
        check_full_size(wl, store)
    finally:
        store.close()
        torch.cuda.empty_cache()
