"""Edge cases at the limits of the boundary, against the CPU oracle: the
largest positions a block table can address (fp64 angles near 2e9 rad),
batches exactly at and just past the store's batch limits, the touched-block
limit, and a block table that is exactly as long as the segment needs."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from synth.device import make_store
from kv_cache_injection_gather_b200 import binding as B
from test_gpu_parity import assert_parity, gpu_run, oracle_run

pytestmark = pytest.mark.gpu


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_positions_near_the_int32_limit():
    """A request whose segment ends 17 positions below 2^31: the block table
    has 2^27 - 1 entries (every position below 2^31 - 16 addressable) and only
    the touched entries point into a small cache."""
    _need_gpu()
    model = synth.Model("llama-like", 2, 8, 128, 5e5, llama3=True)
    rng = np.random.default_rng(11)
    lens = rng.integers(16, 64, 12).astype(np.int32)
    ids = np.array([3, 7, 1], np.int32)
    S = int(lens[ids].sum())
    Bs = 16
    max_blocks = (1 << 27) - 1
    start = max_blocks * Bs - 17 - S
    first, last = start // Bs, (start + S - 1) // Bs
    nblk = last - first + 1
    bt = np.zeros((1, max_blocks), np.int32)
    bt[0, first:last + 1] = rng.permutation(nblk + 4)[:nblk]
    batch = synth.Batch(np.array([0, 3], np.int32), ids, np.array([start], np.int32), bt, Bs, nblk + 4)
    wl = synth.Workload("far", model, lens, batch, seed=12)
    o = oracle_run(wl)
    assert o[0] == oracle.OK
    assert_parity(o, gpu_run(wl))


def test_batch_limits_are_enforced():
    _need_gpu()
    model = synth.Model("m", 1, 2, 64, 1e4)
    rng = np.random.default_rng(12)
    lens = rng.integers(4, 20, 10).astype(np.int32)
    ids = [rng.choice(10, 2, replace=False) for _ in range(4)]
    batch = synth.make_batch(rng, ids, [0, 5, 9, 30], 16, 4 * 4, 4)
    wl = synth.Workload("lim", model, lens, batch, seed=13)
    store = make_store(wl, max_batch_requests=4, max_batch_fact_ids=8, max_batch_blocks=12)
    assert_parity(oracle_run(wl), gpu_run(wl, store=store))  # exactly at the limits
    # one request, one id or one touched block too many
    more = synth.make_batch(rng, ids + [ids[0]], [0, 5, 9, 30, 2], 16, 5 * 4, 4)
    with pytest.raises(B.InjectError) as e:
        gpu_run(synth.Workload("lim", model, lens, more, seed=13), store=store)
    assert e.value.status == B.IS_ERR_CAPACITY
    store.close()
    store = make_store(wl, max_batch_blocks=3)
    n_blocks = sum(-(-(s + int(lens[i].sum())) // 16) - s // 16 for s, i in zip([0, 5, 9, 30], ids))
    assert n_blocks > 3
    rc, slots, kc, vc = gpu_run(wl, store=store)
    assert rc == B.IS_ERR_CAPACITY  # reported on the device, nothing written
    o = oracle_run(synth.Workload("lim", model, lens,
                                  synth.Batch(batch.req_offsets, batch.fact_ids, batch.start_pos,
                                              batch.block_tables, 16, batch.num_blocks), 13))
    unwritten = synth.bf16_block(7, synth.TAG_CACHE | 0, kc.shape)
    assert np.array_equal(kc, unwritten)
    store.close()


def test_block_table_exactly_as_long_as_needed():
    _need_gpu()
    model = synth.Model("m", 2, 4, 128, 1e6)
    rng = np.random.default_rng(14)
    lens = rng.integers(5, 40, 20).astype(np.int32)
    ids = [rng.choice(20, 4, replace=False) for _ in range(3)]
    starts = np.array([0, 7, 16], np.int32)
    need = max(-(-(int(starts[r]) + int(lens[ids[r]].sum())) // 16) for r in range(3))
    batch = synth.make_batch(rng, ids, starts, 16, 3 * need, need)
    wl = synth.Workload("exact", model, lens, batch, seed=15)
    assert_parity(oracle_run(wl), gpu_run(wl))
