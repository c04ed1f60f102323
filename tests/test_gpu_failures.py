"""Failure detection without a GPU fault: a stream held back by a short
device sleep on another stream (the GPU stays responsive), ids and tables
that the device-side checks reject; every wait is bounded.  No kernel of
this library spins or waits on another."""
from __future__ import annotations

import time

import numpy as np
import pytest
import torch

import synth
from synth.device import batch_tensors, make_cache, make_store
from kv_cache_injection_gather_b200 import binding as B

pytestmark = pytest.mark.gpu


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_bounded_wait_times_out_then_recovers():
    _need_gpu()
    from kv_cache_injection_gather_b200 import binding
    wl = synth.tiny(0)
    store = make_store(wl)
    k, v, desc = make_cache(wl)
    ro, ids, sp, bt = batch_tensors(wl.batch)
    s = torch.cuda.Stream()
    # the batch's stream waits for a bounded device sleep (~0.3 s at ~2 GHz)
    # queued on another stream
    gate = torch.cuda.Event()
    blocker = torch.cuda.Stream()
    with torch.cuda.stream(blocker):
        torch.cuda._sleep(int(6e8))
        gate.record(blocker)
    s.wait_event(gate)
    with torch.cuda.stream(s):
        store.inject(ro, ids, sp, bt, desc, stream=s.cuda_stream)
    t0 = time.perf_counter()
    rc, _ = store.last_error_timeout(50, s.cuda_stream)
    waited = time.perf_counter() - t0
    assert rc == binding.IS_ERR_TIMEOUT and waited < 0.25
    rc, _ = store.last_error_timeout(30_000, s.cuda_stream)
    assert rc == binding.IS_OK
    store.close()


def test_device_status_is_cleared_after_reading():
    _need_gpu()
    wl = synth.tiny(0)
    store = make_store(wl)
    k, v, desc = make_cache(wl)
    ro, ids, sp, bt = batch_tensors(wl.batch)
    bad = ids.clone()
    bad[0] = 10_000
    store.inject(ro, bad, sp, bt, desc)
    rc, detail = store.last_error()
    assert rc == B.IS_ERR_BAD_FACT_ID and detail == 0  # request 0
    assert store.last_error()[0] == B.IS_OK          # read once, then cleared
    store.inject(ro, ids, sp, bt, desc)               # the store keeps working
    assert store.last_error()[0] == B.IS_OK
    store.close()


@pytest.mark.parametrize("small_limit", [None, 0], ids=["single-kernel", "two-kernel"])
def test_host_entry_point_reports_device_errors(small_limit):
    """The host entry point returns the status the batch's kernels recorded
    (they also write it into the store's mapped pinned copy): a bad block,
    a malformed CSR, slot capacity, an error left by an earlier asynchronous
    batch on the store (then cleared), and OK."""
    _need_gpu()
    wl = synth.tiny(0)
    store = make_store(wl, small_limit=small_limit)
    k, v, desc = make_cache(wl)
    b = wl.batch
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).pin_memory()  # noqa: E731
    ro, ids, sp, bt = pin(b.req_offsets), pin(b.fact_ids), pin(b.start_pos), pin(b.block_tables)
    bad_bt = b.block_tables.copy()
    bad_bt[0, 2] = 9999  # the first fact's tokens start at position 32: block 2
    assert store.inject_host(ro, ids, sp, pin(bad_bt), desc) == B.IS_ERR_BAD_BLOCK
    assert store.inject_host(ro, ids, sp, bt, desc) == B.IS_OK
    bad_ro = b.req_offsets.copy()
    bad_ro[-1] -= 1
    assert store.inject_host(pin(bad_ro), ids, sp, bt, desc) == B.IS_ERR_INVALID_ARG
    n_tok = wl.tokens()
    short = torch.empty(n_tok - 1, dtype=torch.int64).pin_memory()
    assert store.inject_host(ro, ids, sp, bt, desc, short) == B.IS_ERR_CAPACITY
    # an asynchronous batch's error, not yet read, comes back with the next
    # host-entry batch, which clears it
    d_ro, d_ids, d_sp, d_bt = batch_tensors(b)
    bad_ids = d_ids.clone()
    bad_ids[0] = 9999
    store.inject(d_ro, bad_ids, d_sp, d_bt, desc)
    assert store.inject_host(ro, ids, sp, bt, desc) == B.IS_ERR_BAD_FACT_ID
    assert store.inject_host(ro, ids, sp, bt, desc) == B.IS_OK
    assert store.last_error()[0] == B.IS_OK
    store.close()


@pytest.mark.parametrize("host_tier", [False, True], ids=["device-tier", "host-tier"])
def test_failed_allocation_returns_oom_and_leaves_the_device_usable(host_tier):
    """An HBM arena no device can hold (2^31 - 1 tokens per plane of
    Llama-3.1-8B shapes, ~140 TB): the store's arena on the device tier, the
    hot arena on the host tier (whose pinned store arena is small and is
    freed again).  cudaMalloc refuses at once, create returns IS_ERR_OOM with
    nothing leaked, and a normal store created afterwards injects correctly."""
    _need_gpu()
    from synth.device import rope_of
    from kv_cache_injection_gather_b200 import FactStore
    m = synth.LLAMA31_8B
    huge = (1 << 31) - 1
    free0, _ = torch.cuda.mem_get_info()
    with pytest.raises(B.InjectError) as e:
        FactStore(m.num_layers, m.num_kv_heads, m.head_dim, rope_of(m), 64 if host_tier else huge, 16,
                  host_tier=host_tier, hot_capacity_tokens=huge if host_tier else 0)
    assert e.value.status == B.IS_ERR_OOM
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 >= free0 - (64 << 20)  # nothing of the failed store stays allocated
    wl = synth.tiny(0)
    store = make_store(wl)
    k, v, desc = make_cache(wl)
    ro, ids, sp, bt = batch_tensors(wl.batch)
    store.inject(ro, ids, sp, bt, desc)
    assert store.last_error()[0] == 0
    store.close()
