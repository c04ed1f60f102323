"""Host-tier store (pinned host memory + HBM hot set), against the CPU oracle.

The tier changes where rows are read from, never what is written: every
parity bar of the device tier applies unchanged (the oracle knows no tiers).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from synth.device import make_store
from kv_cache_injection_gather_b200 import binding as B
from test_gpu_parity import _ragged, assert_parity, gpu_run, oracle_run

pytestmark = pytest.mark.gpu


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("path", ["fused", "two-kernel"])
@pytest.mark.parametrize("hot_part", ["none", "some", "all"])
def test_host_tier_parity(hot_part, path):
    _need_gpu()
    model = synth.Model("qwen-like", 2, 4, 128, 1e6)
    wl = _ragged(model, seed=21, R=6, max_k=8, lens=(1, 40), num_facts=30)
    total = int(wl.fact_lens.sum())
    store = make_store(wl, host_tier=True, hot_capacity_tokens=total,
                       small_limit=None if path == "fused" else 0)
    if hot_part == "some":
        store.set_hot(np.arange(0, 30, 3))
    elif hot_part == "all":
        store.set_hot(np.arange(30))
    info = store.tier_info()
    assert info["tier"] == B.IS_TIER_HOST
    assert info["hot_facts"] == {"none": 0, "some": 10, "all": 30}[hot_part]
    assert_parity(oracle_run(wl), gpu_run(wl, store=store))
    store.close()


def test_host_tier_llama_shapes_with_llama3_scaling():
    _need_gpu()
    model = synth.Model("llama-like", 3, 8, 128, 5e5, llama3=True)
    wl = _ragged(model, seed=22, R=4, max_k=6, lens=(16, 64), num_facts=25)
    store = make_store(wl, host_tier=True, hot_capacity_tokens=200)
    lens = wl.fact_lens
    hot, used = [], 0
    for f in np.argsort(-lens):          # fill the hot set as far as it goes
        if used + lens[f] <= 200:
            hot.append(int(f))
            used += int(lens[f])
    store.set_hot(hot)
    assert store.tier_info()["hot_used"] == used
    assert_parity(oracle_run(wl), gpu_run(wl, store=store))
    store.close()


def test_set_hot_errors_keep_previous_set():
    _need_gpu()
    wl = synth.tiny(0)
    store = make_store(wl, host_tier=True, hot_capacity_tokens=40)
    store.set_hot([0])
    before = store.tier_info()
    with pytest.raises(B.InjectError) as e:
        store.set_hot(list(range(64)))            # far more than 40 tokens
    assert e.value.status == B.IS_ERR_CAPACITY
    with pytest.raises(B.InjectError) as e:
        store.set_hot([64])
    assert e.value.status == B.IS_ERR_BAD_FACT_ID
    assert store.tier_info() == before
    assert_parity(oracle_run(wl), gpu_run(wl, store=store))
    store.close()
    dev = make_store(wl)
    with pytest.raises(B.InjectError) as e:
        dev.set_hot([0])
    assert e.value.status == B.IS_ERR_NOT_SUPPORTED
    assert dev.tier_info()["tier"] == B.IS_TIER_DEVICE
    dev.close()


def _host_inject(store, wl):
    from synth.device import make_cache
    from test_gpu_parity import to_bits
    b = wl.batch
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).pin_memory()  # noqa: E731
    k, v, desc = make_cache(wl)
    n_tok = wl.tokens()
    slots = torch.empty(max(n_tok, 1), dtype=torch.int64).pin_memory()
    rc = store.inject_host(pin(b.req_offsets), pin(b.fact_ids), pin(b.start_pos), pin(b.block_tables),
                           desc, slots[:n_tok])
    return rc, slots[:n_tok].numpy().copy(), to_bits(k), to_bits(v)


def test_lru_hot_set_parity_and_promotion():
    """LRU policy: the host entry point promotes each batch's cold facts into
    HBM slots before injecting; results equal the oracle's every time, the
    second pass over the same ids finds them hot, and a slot that is too
    small for a fact leaves it on the host."""
    _need_gpu()
    model = synth.Model("qwen-like", 2, 4, 128, 1e6)
    wl = _ragged(model, seed=31, R=5, max_k=8, lens=(1, 40), num_facts=30)
    lens = wl.fact_lens
    slot = 32
    store = make_store(wl, host_tier=True, hot_capacity_tokens=slot * 6)
    store.set_hot_policy(True, slot)
    want = oracle_run(wl)
    for rep in range(3):
        rc, slots, gk, gv = _host_inject(store, wl)
        assert_parity(want, (rc, slots, gk, gv))
    st = store.lru_stats()
    ids = wl.batch.fact_ids
    assert st["promoted"] >= 1 and st["hits"] >= 1
    assert st["hits"] + st["misses"] == 3 * len(np.unique(ids))  # each call counts distinct ids
    info = store.tier_info()
    assert info["hot_facts"] <= 6 and info["hot_used"] == info["hot_facts"] * slot
    # explicit touch of facts that fit: all become hot (6 slots, 3 facts)
    fit = [int(f) for f in np.flatnonzero(lens <= slot)[:3]]
    store.touch(fit)
    torch.cuda.synchronize()
    assert_parity(want, _host_inject(store, wl))
    with pytest.raises(B.InjectError):
        store.set_hot([0])  # static API refused under LRU
    store.close()


def test_lru_eviction_keeps_results_exact():
    """Far more distinct facts than slots: every batch evicts; results stay
    exact."""
    _need_gpu()
    model = synth.Model("llama-like", 2, 8, 128, 5e5, llama3=True)
    rng = np.random.default_rng(5)
    lens = rng.integers(4, 20, 60).astype(np.int32)
    store = None
    for rep in range(4):
        ids = [rng.choice(60, 6, replace=False) for _ in range(3)]
        batch = synth.make_batch(rng, ids, [0, 17, 40], 16, 3 * 12, 12)
        wl = synth.Workload("lru", model, lens, batch, seed=4)
        if store is None:
            store = make_store(wl, host_tier=True, hot_capacity_tokens=20 * 5)
            store.set_hot_policy(True, 20)
        assert_parity(oracle_run(wl), _host_inject(store, wl))
    assert store.lru_stats()["promoted"] > 5
    store.close()


def test_lru_promotion_survives_a_batch_with_errors():
    """The host entry point fuses each batch's promotions into the batch (the
    kernel writes the promoted facts' rows into their HBM slots as it reads
    them from host memory).  A batch with a bad block-table entry skips some
    rows, so the library copies its promoted facts whole instead; the next
    batches, reading those facts from HBM through either entry point, must
    still equal the oracle."""
    _need_gpu()
    model = synth.Model("llama-like", 2, 8, 128, 5e5, llama3=True)
    wl = _ragged(model, seed=47, R=5, max_k=8, lens=(1, 30), num_facts=30)
    b = wl.batch
    store = make_store(wl, host_tier=True, hot_capacity_tokens=32 * 40)
    store.set_hot_policy(True, 32)
    bad_bt = b.block_tables.copy()
    r = int(np.argmax(np.diff(b.req_offsets) > 0))        # a request with facts
    bad_bt[r, int(b.start_pos[r]) // b.block_size] = b.num_blocks + 5
    bad = synth.Workload(wl.name, model, wl.fact_lens,
                         synth.Batch(b.req_offsets, b.fact_ids, b.start_pos, bad_bt, b.block_size,
                                     b.num_blocks), wl.seed)
    o_bad = oracle_run(bad)
    assert o_bad[0] == oracle.ERR_BAD_BLOCK
    assert_parity(o_bad, _host_inject(store, bad))
    promoted = store.lru_stats()["promoted"]
    assert promoted >= 1
    want = oracle_run(wl)
    assert_parity(want, _host_inject(store, wl))           # hot now: read from HBM
    assert store.lru_stats()["promoted"] == promoted       # nothing left to promote
    assert_parity(want, gpu_run(wl, store=store))          # device entry point, same hot set
    store.close()


def test_lru_prefetch_of_the_next_batch():
    """A stream of batches through is_inject_batch_host_next: each call
    injects its batch and starts moving the next batch's cold facts into HBM
    slots (copy-engine transfers, slots not used by the running batch) while
    it runs.  With 30 slots and 20 facts per batch, part of each next batch
    fits beside the running one and the rest is promoted by its own batch.
    Every batch equals the oracle -- also when the announced next ids are not
    the ones that come, and through the device entry point after a
    prefetch."""
    _need_gpu()
    from synth.device import make_cache
    from test_gpu_parity import to_bits
    model = synth.Model("qwen-like", 2, 4, 128, 1e6)
    rng = np.random.default_rng(71)
    lens = rng.integers(4, 33, 80).astype(np.int32)
    slot = 32
    store = None
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).pin_memory()  # noqa: E731
    batches = []
    for _ in range(6):
        ids = [rng.choice(80, 5, replace=False) for _ in range(4)]
        batches.append(synth.make_batch(rng, ids, [0, 17, 40, 64], 16, 4 * 10, 10))
    wls = [synth.Workload("pf", model, lens, bb, seed=9) for bb in batches]
    store = make_store(wls[0], host_tier=True, hot_capacity_tokens=slot * 30)
    store.set_hot_policy(True, slot)
    promoted = []
    for i, wl in enumerate(wls):
        b = wl.batch
        nxt = batches[(i + 1) % len(batches)].fact_ids if i != 3 else rng.choice(80, 12)
        k, v, desc = make_cache(wl)
        n_tok = wl.tokens()
        slots = torch.empty(max(n_tok, 1), dtype=torch.int64).pin_memory()
        before = store.lru_stats()["promoted"]
        rc = store.inject_host(pin(b.req_offsets), pin(b.fact_ids), pin(b.start_pos),
                               pin(b.block_tables), desc, slots[:n_tok],
                               next_fact_ids=pin(nxt))
        assert_parity(oracle_run(wl), (rc, slots[:n_tok].numpy().copy(), to_bits(k), to_bits(v)))
        promoted.append(store.lru_stats()["promoted"] - before)
    assert promoted[0] > 0
    assert_parity(oracle_run(wls[0]), gpu_run(wls[0], store=store))
    store.close()
