"""GPU path (through the C-ABI) against the CPU oracle on the same seeded
inputs.

Bar: V, slot mapping, status and every untouched cache element bit-exact;
rotated K within |err| <= 2^-8 |ref| + 1e-3 elementwise, ref = the oracle's
fp64 rotation before rounding (the stated tolerance; one bf16 rounding alone
stays inside it, a rounding flip next to a midpoint too).  Non-finite
values follow IEEE arithmetic on both sides: where ref is NaN the output is a
NaN (any sign or payload), where ref is an infinity the output is that
infinity, and an output that overflowed to an infinity stands for every
magnitude from the bf16 overflow threshold (2^128 - 2^119) up, with its
sign, against a finite ref.  The absolute term 1e-3 is the allowance for the
fp32 angle and arithmetic error on unit-scale inputs; where the test knows
the input pair (x_a, x_b) of an element (stores holding values far beyond
the unit scale) it scales with it: + 2^-20 (|x_a| + |x_b|), below 1e-5 on
the N(0, 1) inputs.
"""
from __future__ import annotations

import functools

import numpy as np
import pytest
import torch

import oracle
import synth
from synth.device import (CACHE_FILL_SEED, batch_tensors, make_cache, make_store, to_bits)
from kv_cache_injection_gather_b200 import binding as B
from kv_cache_injection_gather_b200 import cache_desc

pytestmark = pytest.mark.gpu

REL, ABS = 2.0 ** -8, 1e-3
# fp64 marker of K elements the oracle did not write: a signalling NaN, which
# no arithmetic result (always a quiet NaN) can equal bit for bit.
UNWRITTEN = np.uint64(0x7FF4DEADBEEF0000)


def new_kref(shape) -> np.ndarray:
    return np.full(shape, UNWRITTEN, np.uint64).view(np.float64)


def written_mask(kref: np.ndarray) -> np.ndarray:
    return kref.view(np.uint64) != UNWRITTEN


# Round-to-nearest-even to bf16 gives an infinity from this magnitude up: the
# midpoint between the largest finite bf16, 2^128 - 2^120, and 2^128.
BF16_OVERFLOW = 2.0 ** 128 - 2.0 ** 119


# Scale of the fp32 error per unit of input magnitude: the kernel's sine and
# cosine carry a relative error below 2^-22 (single-precision sin/cos of an
# angle reduced exactly in fp64 and rounded once to fp32), the product and the
# fused add round at 2^-24 each: together below 2^-21, and 2^-20 leaves room.
INPUT_REL = 2.0 ** -20


def k_out_of_tolerance(got_bits: np.ndarray, ref: np.ndarray, mag=None) -> np.ndarray:
    """Mask of rotated K elements (bf16 bits) outside the bar against the
    oracle's fp64 values.  An infinity in the output stands for every
    magnitude from BF16_OVERFLOW up, so against a finite ref its error is the
    distance from ref to that range (with the same sign).  mag (optional, the
    same shape): |x_a| + |x_b| of each element's input rotation pair."""
    got = oracle.bf16_to_f64(got_bits)
    bad = np.isnan(got) != np.isnan(ref)
    inf = np.isinf(ref)
    bad |= inf & (got != ref)
    fin = ~np.isnan(ref) & ~inf
    with np.errstate(invalid="ignore"):
        over = np.where(np.sign(got) == np.sign(ref), np.maximum(BF16_OVERFLOW - np.abs(ref), 0.0),
                        np.inf)
        err = np.where(np.isinf(got), over, np.abs(got - ref))
        tol = REL * np.abs(ref) + ABS
        if mag is not None:
            tol = tol + INPUT_REL * np.nan_to_num(mag, nan=0.0, posinf=0.0)
        bad |= fin & ~(err <= tol)
    return bad


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


# ------------------------------------------------------------------ oracle side

def oracle_store(wl: synth.Workload):
    """The oracle's store of every fact of wl (read-only for inject_batch,
    so batches over the same facts may share it)."""
    m = wl.model
    st = oracle.Store(m.num_layers, m.num_kv_heads, m.head_dim, max(int(wl.fact_lens.sum()), 1),
                      len(wl.fact_lens))
    for f, n in enumerate(wl.fact_lens):
        st.put(*synth.fact_kv(wl.seed, f, m.num_layers, m.num_kv_heads, int(n), m.head_dim))
    return st


def oracle_run(wl: synth.Workload, style=0, head_major=False, slot_capacity=None, st=None):
    m, b = wl.model, wl.batch
    if st is None:
        st = oracle_store(wl)
    shape = ((m.num_layers, b.num_blocks, m.num_kv_heads, b.block_size, m.head_dim) if head_major
             else (m.num_layers, b.num_blocks, b.block_size, m.num_kv_heads, m.head_dim))
    kc = synth.bf16_block(CACHE_FILL_SEED, synth.TAG_CACHE | 0, shape)
    vc = synth.bf16_block(CACHE_FILL_SEED, synth.TAG_CACHE | 1, shape)
    kref = new_kref(shape)
    strides = oracle.cache_strides(b.num_blocks, b.block_size, m.num_kv_heads, m.head_dim,
                                   head_major)
    f = oracle.rope_inv_freq(m.head_dim, m.rope_theta, m.scaling())
    rc, slots = oracle.inject_batch(st, f, b.req_offsets, b.fact_ids, b.start_pos, b.block_tables,
                                    kc, vc, b.block_size, strides=strides, style=style, k_ref=kref,
                                    slot_capacity=slot_capacity)
    return rc, slots, kc, vc, kref


# Small batches run as one kernel by default; "two-kernel" forces the plan +
# inject path on the same inputs.
PATHS = {"fused": None, "two-kernel": 0}


def gpu_run(wl: synth.Workload, style=0, head_major=False, slot_capacity=None, store=None,
            path="fused"):
    _need_gpu()
    own = store is None
    if own:
        store = make_store(wl, style, small_limit=PATHS[path])
    k, v, desc = make_cache(wl, head_major=head_major)
    ro, ids, sp, bt = batch_tensors(wl.batch)
    n_tok = int(wl.fact_lens[wl.batch.fact_ids[(wl.batch.fact_ids >= 0) &
                                               (wl.batch.fact_ids < len(wl.fact_lens))]].sum())
    cap = n_tok if slot_capacity is None else slot_capacity
    slots = torch.full((max(cap, 1),), -7, dtype=torch.int64, device="cuda")
    store.inject(ro, ids, sp, bt, desc, slots[:cap] if cap else slots[:0])
    rc, _ = store.last_error()
    out = rc, slots[:cap].cpu().numpy(), to_bits(k), to_bits(v)
    if own:
        store.close()
    return out


def assert_parity(o, g, kmag=None):
    """o: the oracle's (status, slots, K bits, V bits, fp64 K); g: the
    library's (status, slots, K bits, V bits); kmag (optional, the cache's
    shape): input pair magnitudes of the rotated K elements."""
    orc, oslots, okc, ovc, kref = o
    grc, gslots, gkc, gvc = g
    assert grc == orc
    assert np.array_equal(gslots[: len(oslots)], oslots)
    assert np.array_equal(gvc, ovc), "V or untouched V slots differ"
    written = written_mask(kref)
    assert np.array_equal(gkc[~written], okc[~written]), "untouched K slots changed"
    ref = kref[written]
    bad = k_out_of_tolerance(gkc[written], ref, None if kmag is None else kmag[written])
    assert not bad.any(), f"{bad.sum()} K elements out of tolerance, first at ref {ref[bad][:4]}"
    # bit-identical to the oracle's own rounding, NaNs (free payloads) aside,
    # and, where the inputs are known, pairs far beyond the unit scale or so
    # small that fp32's subnormal range decides the last bit
    keep = ~np.isnan(ref)
    if kmag is not None:
        keep &= (kmag[written] <= 64.0) & (kmag[written] >= 2.0 ** -100)
    same = (gkc[written] == okc[written])[keep]
    exact = np.mean(same) if same.size else 1.0
    assert exact > 0.999, f"only {exact:.5f} of K bit-identical to the oracle's rounding"
    return exact


# ------------------------------------------------------------------ tests

def test_device_generator_matches_host():
    _need_gpu()
    n = 1 << 20
    t = torch.empty(n, dtype=torch.int16, device="cuda")
    synth.fill_device(t.data_ptr(), n, 123, synth.fact_stream(77, True), 5000,
                      torch.cuda.current_stream().cuda_stream)
    host = synth.bf16_bits(123, synth.fact_stream(77, True), np.arange(5000, 5000 + n))
    assert np.array_equal(t.cpu().numpy().view(np.uint16), host)


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("style", [0, 1])
@pytest.mark.parametrize("start", [32, 37, 0])
def test_tiny_parity(start, style, path):
    wl = synth.tiny(0, start_pos=start)
    assert_parity(oracle_run(wl, style), gpu_run(wl, style, path=path))


def _ragged(model, seed, B=16, R=7, max_k=9, lens=(1, 40), num_facts=40, starts=None,
            spare_blocks=3):
    rng = np.random.default_rng(seed)
    fl = rng.integers(lens[0], lens[1] + 1, num_facts).astype(np.int32)
    ids = [rng.choice(num_facts, int(rng.integers(0, max_k + 1)), replace=True) for _ in range(R)]
    if R > 1:
        ids[1] = np.zeros(0, np.int64)  # an empty request
    sp = (rng.integers(0, 70, R) if starts is None else np.asarray(starts)).astype(np.int32)
    need = max(-(-(int(sp[r]) + int(fl[ids[r]].sum())) // B) for r in range(R)) + spare_blocks
    batch = synth.make_batch(rng, ids, sp, B, R * need, need)
    return synth.Workload("ragged", model, fl, batch, seed)


SHAPES = [
    # name, L, H, D, theta, llama3, B, style, head_major
    ("llama-like", 3, 8, 128, 5e5, True, 16, 0, False),
    ("qwen-like", 2, 4, 128, 1e6, False, 16, 0, False),
    ("interleaved", 2, 4, 128, 1e4, False, 16, 1, False),
    ("head-major", 2, 8, 128, 5e5, True, 16, 0, True),
    ("qwen-head-major", 3, 4, 128, 1e6, False, 16, 0, True),
    ("h3-generic", 2, 3, 128, 1e4, False, 16, 0, False),
    ("d64-b8", 2, 2, 64, 1e4, False, 8, 0, False),
    ("d256-b32", 1, 2, 256, 1e4, False, 32, 1, False),
    ("d32-b1", 2, 1, 32, 1e4, False, 1, 0, False),
    ("b128", 1, 2, 64, 1e4, False, 128, 0, False),
    ("b12-generic", 2, 2, 64, 1e4, False, 12, 0, True),
]


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_ragged_batches_parity(shape, path):
    name, L, H, D, theta, ll3, B_, style, hm = shape
    model = synth.Model(name, L, H, D, theta, llama3=ll3)
    wl = _ragged(model, seed=sum(name.encode()), B=B_)
    assert_parity(oracle_run(wl, style, hm), gpu_run(wl, style, hm, path=path))


@pytest.mark.parametrize("R,k", [(1024, 2), (1025, 2), (9, 2048), (9, 2049)],
                         ids=["1024-requests", "1025-requests", "16384-ids", "16392-ids"])
def test_plan_in_shared_and_global_memory(R, k):
    """The plan kernel keeps batches of at most 1024 requests and 16384 fact
    ids in shared memory and runs larger ones on its global work space:
    both sides of both limits, against the oracle."""
    model = synth.Model("m", 1, 1, 32, 1e4)
    rng = np.random.default_rng(R * 7 + k)
    F = 64
    fl = rng.integers(1, 4, F).astype(np.int32)
    ids = [rng.integers(0, F, k) for _ in range(R)]
    ids[1] = np.zeros(0, np.int64)
    sp = rng.integers(0, 40, R).astype(np.int32)
    need = max(-(-(int(sp[r]) + int(fl[ids[r]].sum())) // 16) for r in range(R)) + 1
    batch = synth.make_batch(rng, ids, sp, 16, R * need, need)
    wl = synth.Workload("plan-limits", model, fl, batch, R)
    assert len(wl.batch.fact_ids) == k * (R - 1)
    assert_parity(oracle_run(wl), gpu_run(wl, path="two-kernel"))


@pytest.mark.parametrize("path", list(PATHS))
def test_many_requests_many_ids(path):
    """Past the single-kernel limits (9 requests; 300 ids): the two-kernel
    path in both settings."""
    model = synth.Model("m", 2, 4, 64, 1e4)
    wl = _ragged(model, seed=77, R=9, max_k=9, lens=(1, 12), num_facts=50)
    assert_parity(oracle_run(wl), gpu_run(wl, path=path))
    wl2 = _ragged(model, seed=78, R=6, max_k=150, lens=(1, 6), num_facts=400, spare_blocks=1)
    assert len(wl2.batch.fact_ids) > 256
    assert_parity(oracle_run(wl2), gpu_run(wl2, path=path))


@pytest.mark.parametrize("path", list(PATHS))
def test_long_segments_many_blocks(path):
    """Facts longer than several blocks; positions up to ~5k (fp32 angle range
    the kernel must handle with fp64 angles)."""
    model = synth.Model("long", 2, 2, 128, 5e5, llama3=True)
    wl = _ragged(model, seed=3, R=3, max_k=6, lens=(100, 300), num_facts=12,
                 starts=[0, 3000, 4097])
    assert_parity(oracle_run(wl), gpu_run(wl, path=path))


@pytest.mark.parametrize("path", list(PATHS))
def test_empty_batch_and_empty_requests(path):
    model = synth.Model("e", 1, 2, 64, 1e4)
    rng = np.random.default_rng(0)
    fl = rng.integers(1, 20, 10).astype(np.int32)
    b0 = synth.make_batch(rng, [], np.zeros(0), 16, 4, 1)
    wl0 = synth.Workload("empty", model, fl, b0)
    assert_parity(oracle_run(wl0), gpu_run(wl0, path=path))
    b1 = synth.make_batch(rng, [np.zeros(0, int)] * 3, [5, 0, 16], 16, 6, 2)
    wl1 = synth.Workload("empty-requests", model, fl, b1)
    assert_parity(oracle_run(wl1), gpu_run(wl1, path=path))


def _error_wl(kind):
    wl = synth.tiny(0)
    b = wl.batch
    ids = np.concatenate([b.fact_ids[:2], b.fact_ids[2:4]]).astype(np.int32)
    ro = np.array([0, 2, 4], np.int32)
    sp = np.array([0, 40], np.int32)
    bt = np.stack([np.arange(0, 20), np.arange(20, 40)]).astype(np.int32)
    if kind == "bad_fact":
        ids[2] = 9999
    elif kind == "position":
        sp[1] = 20 * 16 - 3
    elif kind == "bad_block":
        bt[1, 3] = 64
    elif kind == "negative_block":
        bt[0, 0] = -5
    elif kind == "negative_start":
        sp[0] = -1
    elif kind == "csr":
        ro = np.array([0, 2, 3], np.int32)
    elif kind == "csr_range":
        # request 0 ends past the id list, request 1 ends before it starts
        ro = np.array([0, 5, 4], np.int32)
    elif kind == "block_then_fact":
        # errors in both requests: the first in request order is reported
        bt[0, 1] = 64
        ids[2] = 9999
    elif kind == "fact_then_block":
        ids[0] = -3
        bt[1, 3] = 70
    elif kind == "position_then_block":
        sp[0] = 20 * 16 - 3
        bt[1, 2] = -1
    batch = synth.Batch(ro, ids, sp, bt, 16, 64)
    return synth.Workload("err-" + kind, wl.model, wl.fact_lens, batch, wl.seed)


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("kind", ["bad_fact", "position", "bad_block", "negative_block",
                                  "negative_start", "csr", "csr_range", "block_then_fact",
                                  "fact_then_block", "position_then_block"])
def test_device_errors_match_oracle(kind, path):
    wl = _error_wl(kind)
    o = oracle_run(wl)
    assert o[0] != oracle.OK
    assert_parity(o, gpu_run(wl, path=path))


@pytest.mark.parametrize("path", list(PATHS))
def test_slot_capacity_error_writes_nothing(path):
    wl = synth.tiny(0)
    o = oracle_run(wl, slot_capacity=3)
    g = gpu_run(wl, slot_capacity=3, path=path)
    assert o[0] == g[0] == oracle.ERR_CAPACITY
    assert np.array_equal(g[2], o[2]) and np.array_equal(g[3], o[3])


def test_host_entry_point_matches_device_entry_point():
    _need_gpu()
    wl = _ragged(synth.Model("h", 2, 4, 128, 1e6), seed=11)
    store = make_store(wl)
    b = wl.batch
    n_tok = int(wl.fact_lens[b.fact_ids].sum())
    k1, v1, d1 = make_cache(wl)
    k2, v2, d2 = make_cache(wl)
    ro, ids, sp, bt = batch_tensors(b)
    s1 = torch.empty(n_tok, dtype=torch.int64, device="cuda")
    store.inject(ro, ids, sp, bt, d1, s1)
    assert store.last_error()[0] == 0
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).pin_memory()  # noqa: E731
    s2 = torch.empty(n_tok, dtype=torch.int64).pin_memory()
    rc = store.inject_host(pin(b.req_offsets), pin(b.fact_ids), pin(b.start_pos),
                           pin(b.block_tables), d2, s2)
    assert rc == 0
    assert torch.equal(k1, k2) and torch.equal(v1, v2)
    assert torch.equal(s1.cpu(), s2)
    store.close()


def test_host_entry_point_slot_buffers():
    """The slot mapping of the host entry point: a pinned buffer is written in
    place (entries past the batch's tokens untouched, nothing at all on
    CAPACITY); a pageable buffer gets the same slots through a copy."""
    _need_gpu()
    wl = _ragged(synth.Model("h", 2, 4, 128, 1e6), seed=12)
    store = make_store(wl)
    b = wl.batch
    n_tok = wl.tokens()
    o = oracle_run(wl)
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).pin_memory()  # noqa: E731
    args = (pin(b.req_offsets), pin(b.fact_ids), pin(b.start_pos), pin(b.block_tables))
    sentinel = 0x5A5A5A5A5A5A5A5A
    # pinned, with room to spare
    k, v, d = make_cache(wl)
    buf = torch.full((n_tok + 37,), sentinel, dtype=torch.int64).pin_memory()
    rc = store.inject_host(*args, d, buf)
    assert_parity(o, (rc, buf[:n_tok].numpy().copy(), to_bits(k), to_bits(v)))
    assert (buf[n_tok:] == sentinel).all()
    # a pinned slice that starts inside the allocation
    k, v, d = make_cache(wl)
    buf = torch.full((n_tok + 64,), sentinel, dtype=torch.int64).pin_memory()
    rc = store.inject_host(*args, d, buf[13:13 + n_tok])
    assert_parity(o, (rc, buf[13:13 + n_tok].numpy().copy(), to_bits(k), to_bits(v)))
    assert (buf[:13] == sentinel).all() and (buf[13 + n_tok:] == sentinel).all()
    # pageable
    k, v, d = make_cache(wl)
    page = torch.full((n_tok,), sentinel, dtype=torch.int64)
    assert not page.is_pinned()
    rc = store.inject_host(*args, d, page)
    assert_parity(o, (rc, page.numpy().copy(), to_bits(k), to_bits(v)))
    # pinned, one entry short: CAPACITY, buffer and cache untouched
    k, v, d = make_cache(wl)
    k0, v0 = k.clone(), v.clone()
    buf = torch.full((n_tok,), sentinel, dtype=torch.int64).pin_memory()
    rc = store.inject_host(*args, d, buf[:n_tok - 1])
    assert rc == oracle.ERR_CAPACITY
    assert (buf == sentinel).all()
    assert torch.equal(k, k0) and torch.equal(v, v0)
    store.close()


def test_store_put_read_and_arena():
    _need_gpu()
    wl = synth.tiny(0)
    m = wl.model
    store = make_store(wl)
    ka, va = store.arena()
    for f in (0, 5, 63):
        off, n = store.fact_info(f)
        k, v = synth.fact_kv(wl.seed, f, m.num_layers, m.num_kv_heads, n, m.head_dim)
        kr, vr = store.read_fact(f)
        assert np.array_equal(to_bits(kr), k) and np.array_equal(to_bits(vr), v)
        assert np.array_equal(to_bits(ka[:, :, off:off + n]), k)
        assert np.array_equal(to_bits(va[:, :, off:off + n]), v)
    assert store.num_facts == 64
    with pytest.raises(B.InjectError):
        store.fact_info(64)
    store.close()


def test_repeatable_and_stream_ordered():
    """Two batches in a row on a side stream give identical bytes; the timing
    hook counts one launch per batch."""
    _need_gpu()
    wl = _ragged(synth.Model("r", 2, 8, 128, 5e5, llama3=True), seed=5)
    store = make_store(wl)
    s = torch.cuda.Stream()
    k, v, d = make_cache(wl)
    k2, v2, d2 = make_cache(wl)
    ro, ids, sp, bt = batch_tensors(wl.batch)
    torch.cuda.synchronize()
    store.set_timing(True)
    with torch.cuda.stream(s):
        store.inject(ro, ids, sp, bt, d)
        store.inject(ro, ids, sp, bt, d2)
    assert store.last_error(s.cuda_stream)[0] == 0
    ms, n = store.kernel_time()
    assert n == 2 and ms > 0
    assert torch.equal(k, k2) and torch.equal(v, v2)
    store.close()


def test_llama_single_request_full_store():
    """Llama-3.1-8B shapes, 10k facts of 16-64 tokens (about 52 GB of store),
    one request of k=5 after a 64-token prefix; whole cache compared."""
    _need_gpu()
    wl = synth.llama_single(0)
    store = make_store(wl, on_device_gen=True)
    g = gpu_run(wl, store=store)
    store.close()
    # the oracle needs only the five injected facts: renumber them 0..4
    ids = wl.batch.fact_ids
    sub = synth.Workload(wl.name, wl.model, wl.fact_lens[ids],
                         synth.Batch(wl.batch.req_offsets, np.arange(len(ids), dtype=np.int32),
                                     wl.batch.start_pos, wl.batch.block_tables,
                                     wl.batch.block_size, wl.batch.num_blocks), wl.seed)
    # regenerate the injected facts under their original ids
    m = wl.model
    st = oracle.Store(m.num_layers, m.num_kv_heads, m.head_dim, int(sub.fact_lens.sum()), len(ids))
    for f in ids:
        st.put(*synth.fact_kv(wl.seed, int(f), m.num_layers, m.num_kv_heads,
                              int(wl.fact_lens[f]), m.head_dim))
    b = sub.batch
    shape = (m.num_layers, b.num_blocks, b.block_size, m.num_kv_heads, m.head_dim)
    kc = synth.bf16_block(CACHE_FILL_SEED, synth.TAG_CACHE | 0, shape)
    vc = synth.bf16_block(CACHE_FILL_SEED, synth.TAG_CACHE | 1, shape)
    kref = new_kref(shape)
    f = oracle.rope_inv_freq(m.head_dim, m.rope_theta, m.scaling())
    rc, slots = oracle.inject_batch(st, f, b.req_offsets, b.fact_ids, b.start_pos, b.block_tables,
                                    kc, vc, b.block_size, k_ref=kref)
    assert_parity((rc, slots, kc, vc, kref), g)


@functools.lru_cache(maxsize=None)
def _block_count_case(nblk):
    k = 5
    T = 16 * nblk - 8
    lens = np.array([T // k + (i < T % k) for i in range(k)], np.int32)
    batch = synth.make_batch(np.random.default_rng(nblk), [np.arange(k)], 64, 16, 24, 24)
    wl = synth.Workload("llama-blocks", synth.LLAMA31_8B, lens, batch, seed=nblk)
    assert wl.tokens() == T
    return wl, oracle_run(wl)


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("nblk", [13, 15, 16, 17, 18])
def test_llama_single_request_block_counts(nblk, path):
    """One Llama-3.1-8B request of k=5 after a 64-token prefix touching nblk
    cache blocks (the last one half full).  With one wave of work units per
    batch this size, 15 to 17 blocks are where rounding the units' row ranges
    once gave more units than the 296-CTA grid; every count, on both paths,
    gives the oracle's cache."""
    _need_gpu()
    wl, o = _block_count_case(nblk)  # the oracle's cache, shared by both paths
    assert_parity(o, gpu_run(wl, path=path))


def test_single_kernel_takes_units_from_its_counter_back_to_back():
    """The single kernel past two waves: 32 requests and up to 256 ids with
    more than twice the work units a 296-CTA grid holds, so CTAs take units
    from the store's counter, which the launch's last fetch sets back to
    zero.  Three such batches queued back to back on one stream (each needs
    the counter at zero) all give the oracle's cache."""
    from test_unit_sizing_model import unit_size
    _need_gpu()
    model = synth.Model("l4h8", 4, 8, 128, 5e5, llama3=True)
    base = _ragged(model, seed=41, R=32, max_k=8, lens=(8, 40), num_facts=64)
    wls = []
    for i in range(3):
        rng = np.random.default_rng(100 + i)
        ids = [rng.choice(64, int(rng.integers(6, 9)), replace=False) for _ in range(32)]
        sp = rng.integers(0, 70, 32).astype(np.int32)
        need = max(-(-(int(sp[r]) + int(base.fact_lens[ids[r]].sum())) // 16) for r in range(32)) + 2
        b = synth.make_batch(rng, ids, sp, 16, 32 * need, need)
        wl = synth.Workload("dyn", model, base.fact_lens, b, base.seed)
        blocks = sum(-(-(int(sp[r]) + int(base.fact_lens[ids[r]].sum())) // 16) - int(sp[r]) // 16
                     for r in range(32))
        upb = unit_size(blocks, model.num_layers, model.num_kv_heads, 296, True)[1]
        assert len(b.fact_ids) <= 256 and blocks * upb > 2 * 296
        wls.append(wl)
    store = make_store(base)
    runs = []
    for wl in wls:
        k, v, desc = make_cache(wl)
        ro, ids, sp, bt = batch_tensors(wl.batch)
        slots = torch.full((wl.tokens(),), -7, dtype=torch.int64, device="cuda")
        store.inject(ro, ids, sp, bt, desc, slots)
        runs.append((k, v, slots, (ro, ids, sp, bt)))
    rc, _ = store.last_error()
    ost = oracle_store(base)
    for wl, (k, v, slots, _) in zip(wls, runs):
        assert_parity(oracle_run(wl, st=ost), (rc, slots.cpu().numpy(), to_bits(k), to_bits(v)))
    store.close()


def test_single_kernel_counter_across_batches_with_errors():
    """The single kernel's counter through batches with errors: past two
    waves, a batch with a block-table entry outside the cache in request 5
    (those units are taken and skip their stores) and an id outside the
    store in request 9 (its blocks make no units); then a batch whose CSR
    does not end at the id count (rejected before any unit); then a clean
    batch past two waves.  Each gives the oracle's status and cache."""
    from test_unit_sizing_model import unit_size
    _need_gpu()
    model = synth.Model("l4h8", 4, 8, 128, 5e5, llama3=True)
    base = _ragged(model, seed=41, R=32, max_k=8, lens=(8, 40), num_facts=64)

    def batch(seed, skip=()):
        rng = np.random.default_rng(seed)
        ids = [rng.choice(64, int(rng.integers(6, 9)), replace=False) for _ in range(32)]
        sp = rng.integers(0, 70, 32).astype(np.int32)
        span = [-(-(int(sp[r]) + int(base.fact_lens[ids[r]].sum())) // 16) for r in range(32)]
        b = synth.make_batch(rng, ids, sp, 16, 32 * (max(span) + 2), max(span) + 2)
        blocks = sum(span[r] - int(sp[r]) // 16 for r in range(32) if r not in skip)
        upb = unit_size(blocks, model.num_layers, model.num_kv_heads, 296, True)[1]
        assert len(b.fact_ids) <= 256 and blocks * upb > 2 * 296
        return b

    b = batch(200, skip=(9,))
    bt = b.block_tables.copy()
    bt[5, int(b.start_pos[5]) // 16 + 1] = b.num_blocks + 3
    fids = b.fact_ids.copy()
    fids[b.req_offsets[9]] = 9999
    b1 = synth.Batch(b.req_offsets, fids, b.start_pos, bt, 16, b.num_blocks)
    b = batch(201)
    ro = b.req_offsets.copy()
    ro[-1] -= 1
    b2 = synth.Batch(ro, b.fact_ids, b.start_pos, b.block_tables, 16, b.num_blocks)
    b3 = batch(202)
    store = make_store(base)
    ost = oracle_store(base)
    for bb, code in ((b1, oracle.ERR_BAD_BLOCK), (b2, oracle.ERR_INVALID_ARG), (b3, oracle.OK)):
        wl = synth.Workload("dyn-err", model, base.fact_lens, bb, base.seed)
        o = oracle_run(wl, st=ost)
        assert o[0] == code
        assert_parity(o, gpu_run(wl, store=store))
    store.close()


def test_single_kernel_random_stream_of_batches():
    """Twelve seeded batches of 1..32 requests queued back to back on one
    stream through the single kernel -- one wave or several, some with an id
    outside the store, a block-table entry outside the cache or a CSR that
    does not end at the id count -- each into its own cache: every cache is
    the oracle's, and the status read once at the end is the first error in
    stream order (each batch's own first error in request order)."""
    _need_gpu()
    model = synth.Model("l4h8", 4, 8, 128, 5e5, llama3=True)
    base = _ragged(model, seed=43, R=32, max_k=8, lens=(4, 48), num_facts=64)
    rng = np.random.default_rng(2024)
    wls = []
    for i in range(12):
        R = int(rng.integers(1, 33))
        kmax = int(rng.choice([2, 8]))
        ids = [rng.choice(64, int(rng.integers(0, kmax + 1)), replace=False) for _ in range(R)]
        sp = rng.integers(0, 100, R).astype(np.int32)
        need = max(-(-(int(sp[r]) + int(base.fact_lens[ids[r]].sum())) // 16) for r in range(R)) + 1
        b = synth.make_batch(rng, ids, sp, 16, R * need, need)
        fids, bt, ro = b.fact_ids.copy(), b.block_tables.copy(), b.req_offsets.copy()
        kind = rng.choice(["clean"] * 5 + ["bad_id", "bad_block", "csr"])
        if kind == "bad_id" and len(fids):
            fids[int(rng.integers(0, len(fids)))] = 64 + int(rng.integers(0, 5))
        elif kind == "bad_block":
            r = int(rng.integers(0, R))
            bt[r, int(sp[r]) // 16] = -2
        elif kind == "csr" and R > 1:
            ro[-1] += 1
        wls.append(synth.Workload("stream", model, base.fact_lens,
                                  synth.Batch(ro, fids, sp, bt, 16, b.num_blocks), base.seed))
    store = make_store(base)
    runs = []
    for wl in wls:
        k, v, desc = make_cache(wl)
        ro_t, ids_t, sp_t, bt_t = batch_tensors(wl.batch)
        fids = wl.batch.fact_ids
        n_tok = int(wl.fact_lens[fids[(fids >= 0) & (fids < 64)]].sum())
        slots = torch.full((max(n_tok, 1),), -7, dtype=torch.int64, device="cuda")
        store.inject(ro_t, ids_t, sp_t, bt_t, desc, slots[:n_tok])
        runs.append((k, v, slots, n_tok, (ro_t, ids_t, sp_t, bt_t)))
    rc, _ = store.last_error()
    first = oracle.OK
    ost = oracle_store(base)
    for wl, (k, v, slots, n_tok, _) in zip(wls, runs):
        o = oracle_run(wl, st=ost)
        if first == oracle.OK:
            first = o[0]
        assert_parity((oracle.OK,) + tuple(o[1:]), (oracle.OK, slots[:n_tok].cpu().numpy(), to_bits(k),
                                                    to_bits(v)))
    assert rc == first
    store.close()


def test_head_sharded_stores_reproduce_the_full_cache():
    """KV-head shards (the multi-GPU tensor-parallel partition): a store and
    cache holding heads [h0, h1) only, fed the whole batch, produce exactly
    the oracle's full cache restricted to those heads."""
    _need_gpu()
    from synth.device import make_cache
    model = synth.Model("llama-like", 2, 8, 128, 5e5, llama3=True)
    wl = _ragged(model, seed=41, R=5)
    orc, oslots, okc, ovc, kref = oracle_run(wl)
    kfull, vfull, _ = make_cache(wl)  # the oracle's fill, all heads
    for h0, h1 in ((0, 4), (4, 8), (6, 8)):
        store = make_store(wl, heads=(h0, h1))
        # The shard's cache starts as the full cache's head slice, so its
        # untouched slots hold the values the oracle's cache holds there.
        k = kfull[:, :, :, h0:h1].contiguous()
        v = vfull[:, :, :, h0:h1].contiguous()
        desc = cache_desc(k, v)
        ro, ids, sp, bt = batch_tensors(wl.batch)
        store.inject(ro, ids, sp, bt, desc)
        assert store.last_error()[0] == orc
        gk, gv = to_bits(k), to_bits(v)
        assert np.array_equal(gv, ovc[:, :, :, h0:h1])
        w = written_mask(np.ascontiguousarray(kref[:, :, :, h0:h1]))
        assert np.array_equal(gk[~w], okc[:, :, :, h0:h1][~w])
        assert not k_out_of_tolerance(gk[w], kref[:, :, :, h0:h1][w]).any()
        store.close()
