"""is_inject_batch_noalloc, the entry point for callers that cannot allocate
device memory: an engine whose memory pool already owns the whole GPU, a
plugin whose host forbids allocations behind its back.  Such a caller hands over the store's arenas and
fact table as its own buffers; the per-batch work space is the library's
fixed device array.

Checked here, through the C-ABI:
  * the same cache, slot mapping and status as is_inject_batch on the same
    inputs, two calls in a row (the second on the work space the first left);
  * against the CPU oracle on ragged batches: token-major and head-major
    caches, the fixed model shapes and a generic shape (3 heads, head_dim 64,
    block size 12), both RoPE pairings;
  * the device status it writes for a bad fact id, for fact-table entries
    that leave the arenas (refused before any read) and for a batch touching
    more cache blocks than the work space holds (nothing written), and a good
    batch right after each of them.

Collected last (file name) so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from synth.device import batch_tensors, make_cache, make_store, to_bits
from kv_cache_injection_gather_b200 import binding as B
from test_gpu_parity import _ragged, assert_parity, oracle_run

pytestmark = pytest.mark.gpu

REL, ABS = 2.0 ** -8, 1e-3  # the K tolerance of the other GPU tests


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _cfg(model: synth.Model, style: int = 0) -> B.is_store_config_t:
    return B.is_store_config_t(num_layers=model.num_layers, num_kv_heads=model.num_kv_heads,
                               head_dim=model.head_dim, rope_style=style,
                               rope_theta=model.rope_theta,
                               rope_scaling=B.IS_SCALING_LLAMA3 if model.llama3 else B.IS_SCALING_NONE,
                               scale_factor=8.0, low_freq_factor=1.0, high_freq_factor=4.0,
                               original_max_position=8192)


class _CallerBuffers:
    """A store built by the library whose arenas and fact table are then used
    the way a caller's own buffers would be: passed to the allocation-free
    entry point, which owns none of them."""

    def __init__(self, wl: synth.Workload, style: int = 0):
        self.store = make_store(wl, style)
        self.k, self.v, self.plane = B.is_store_arena(self.store.handle)
        info = [self.store.fact_info(f) for f in range(len(wl.fact_lens))]
        self.offs = torch.tensor([o for o, _ in info], dtype=torch.int64, device="cuda")
        self.lens = torch.tensor([n for _, n in info], dtype=torch.int32, device="cuda")
        self.num_facts = len(info)
        self.cfg = _cfg(wl.model, style)

    def run(self, wl: synth.Workload, head_major=False, slot_capacity=None, offs=None, lens=None):
        """One batch into a fresh seeded cache; returns (device status code,
        detail, slots, K bits, V bits)."""
        b = wl.batch
        k, v, desc = make_cache(wl, head_major=head_major)
        ro, ids, sp, bt = batch_tensors(b)
        cap = slot_capacity if slot_capacity is not None else 0
        slots = torch.full((max(cap, 1),), -7, dtype=torch.int64, device="cuda")
        status = torch.full((2,), -99, dtype=torch.int64, device="cuda")
        offs = self.offs if offs is None else offs
        lens = self.lens if lens is None else lens
        rc = B.is_inject_batch_noalloc(self.cfg, self.k, self.v, self.plane, offs.data_ptr(),
                                       lens.data_ptr(), self.num_facts, b.num_requests,
                                       ro.data_ptr(), ids.data_ptr(), ids.numel(), sp.data_ptr(),
                                       bt.data_ptr(), b.max_blocks, desc,
                                       slots.data_ptr() if cap else None, cap, status.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
        assert rc == B.IS_OK, B.status_string(rc)
        torch.cuda.synchronize()
        code = int(status.view(torch.int32)[0].item())
        detail = int(status[1].item())
        return code, detail, slots[:cap].cpu().numpy(), to_bits(k), to_bits(v)

    def close(self):
        self.store.close()


def _parity(buf, wl, style=0, head_major=False):
    """The allocation-free batch against the oracle on the same inputs."""
    o = oracle_run(wl, style, head_major)
    code, _, slots, kb, vb = buf.run(wl, head_major, slot_capacity=len(o[1]))
    assert_parity(o, (code, slots, kb, vb))
    return code


def _batch(rng, lens, R, max_k, B_, starts):
    nf = len(lens)
    ids = [rng.choice(nf, int(rng.integers(1, max_k + 1)), replace=False) for _ in range(R)]
    need = max(-(-(int(starts[r]) + int(lens[ids[r]].sum())) // B_) for r in range(R)) + 2
    return synth.make_batch(rng, ids, starts, B_, R * need, need)


def test_no_alloc_matches_store_entry_point_two_calls():
    _need_gpu()
    rng = np.random.default_rng(2024)
    model = synth.Model("llama-like", 4, 8, 128, 5e5, llama3=True)
    lens = rng.integers(16, 65, 300).astype(np.int32)
    b1 = _batch(rng, lens, 12, 20, 16, rng.integers(0, 100, 12).astype(np.int32))
    b2 = _batch(rng, lens, 5, 30, 16, np.array([64, 0, 17, 300, 5], np.int32))
    buf = _CallerBuffers(synth.Workload("noalloc", model, lens, b1, seed=3))
    for batch in (b1, b2):
        wlb = synth.Workload("noalloc", model, lens, batch, seed=3)
        n_tok = wlb.tokens()
        ro, ids, sp, bt = batch_tensors(batch)
        # the store's own entry point
        k1, v1, d1 = make_cache(wlb)
        s1 = torch.empty(n_tok, dtype=torch.int64, device="cuda")
        buf.store.inject(ro, ids, sp, bt, d1, s1)
        assert buf.store.last_error()[0] == B.IS_OK
        # allocation-free entry point, same inputs, a fresh cache with the same fill
        code, _, s2, k2, v2 = buf.run(wlb, slot_capacity=n_tok)
        assert code == B.IS_OK, "device status not ok"
        assert np.array_equal(s1.cpu().numpy(), s2)
        assert np.array_equal(to_bits(v1), v2)
        f1 = oracle.bf16_to_f64(to_bits(k1))
        f2 = oracle.bf16_to_f64(k2)
        assert np.all(np.abs(f2 - f1) <= REL * np.abs(f1) + ABS)

    # sizes beyond the fixed work space are refused before any launch
    ro, ids, sp, bt = batch_tensors(b1)
    _, _, d = make_cache(synth.Workload("noalloc", model, lens, b1, seed=3))
    rc = B.is_inject_batch_noalloc(buf.cfg, buf.k, buf.v, buf.plane, buf.offs.data_ptr(),
                                   buf.lens.data_ptr(), buf.num_facts,
                                   B.IS_NOALLOC_MAX_REQUESTS + 1, ro.data_ptr(), ids.data_ptr(),
                                   ids.numel(), sp.data_ptr(), bt.data_ptr(), b1.max_blocks, d,
                                   None, 0, None, torch.cuda.current_stream().cuda_stream)
    assert rc == B.IS_ERR_CAPACITY
    buf.close()


SHAPES = [
    # name, L, H, D, theta, llama3, B, style, head_major
    ("llama-token-major", 3, 8, 128, 5e5, True, 16, 0, False),
    ("llama-head-major", 2, 8, 128, 5e5, True, 16, 0, True),
    ("qwen-head-major", 3, 4, 128, 1e6, False, 16, 0, True),
    ("interleaved", 2, 4, 128, 1e4, False, 16, 1, False),
    ("h3-d64-b12-head-major", 2, 3, 64, 1e4, False, 12, 0, True),
    ("h3-d64-b12-interleaved", 2, 3, 64, 1e4, False, 12, 1, False),
]


@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_no_alloc_matches_oracle(shape):
    """Two ragged batches in a row through the allocation-free entry point,
    each against the oracle: V, slots and untouched slots bit-exact, K within
    the tolerance."""
    _need_gpu()
    name, L, H, D, theta, ll3, B_, style, hm = shape
    model = synth.Model(name, L, H, D, theta, llama3=ll3)
    seed = sum(name.encode())
    wl = _ragged(model, seed=seed, B=B_)
    buf = _CallerBuffers(wl, style)
    try:
        for batch in (wl.batch, _rebatch(wl, seed + 1, B_)):
            wlb = synth.Workload(wl.name, model, wl.fact_lens, batch, wl.seed)
            assert _parity(buf, wlb, style, hm) == B.IS_OK
    finally:
        buf.close()


def _rebatch(wl, seed, B_):
    """Another ragged batch over the same facts."""
    rng = np.random.default_rng(seed)
    nf = len(wl.fact_lens)
    R = 6
    ids = [rng.choice(nf, int(rng.integers(0, 10)), replace=True) for _ in range(R)]
    sp = rng.integers(0, 70, R).astype(np.int32)
    need = max(-(-(int(sp[r]) + int(wl.fact_lens[ids[r]].sum())) // B_) for r in range(R)) + 2
    return synth.make_batch(rng, ids, sp, B_, R * need, need)


def _with_ids(wl, ids):
    b = wl.batch
    return synth.Workload(wl.name, wl.model, wl.fact_lens,
                          synth.Batch(b.req_offsets, np.asarray(ids, np.int32), b.start_pos,
                                      b.block_tables, b.block_size, b.num_blocks), wl.seed)


def test_no_alloc_device_errors_and_recovery():
    """The device status of refused batches, what they leave in the cache and
    the slot mapping (as the oracle says), and a good batch right after each."""
    _need_gpu()
    model = synth.Model("llama-like", 2, 8, 128, 5e5, llama3=True)
    wl = _ragged(model, seed=314, R=5)
    b = wl.batch
    buf = _CallerBuffers(wl)
    try:
        r0 = b.fact_ids[b.req_offsets[0]:b.req_offsets[1]]
        r2 = b.fact_ids[b.req_offsets[2]:b.req_offsets[3]]
        assert len(r0) and len(r2)
        # a fact id outside the table: its request is skipped
        ids = b.fact_ids.copy()
        ids[b.req_offsets[2]] = buf.num_facts + 3
        assert _parity(buf, _with_ids(wl, ids)) == B.IS_ERR_BAD_FACT_ID
        assert _parity(buf, wl) == B.IS_OK
        # fact-table entries that leave the arenas: past the plane, negative,
        # empty -- each id refused as outside the store, before any read
        f = int(r0[0])
        for off, n in ((buf.plane, 5), (buf.plane - 3, 4), (-16, 8), (0, 0)):
            offs, lens = buf.offs.clone(), buf.lens.clone()
            offs[f], lens[f] = off, n
            bad_ids = np.where(b.fact_ids == f, buf.num_facts + 7, b.fact_ids)
            o = oracle_run(_with_ids(wl, bad_ids))
            assert o[0] == oracle.ERR_BAD_FACT_ID
            code, detail, slots, kb, vb = buf.run(wl, slot_capacity=len(o[1]), offs=offs, lens=lens)
            assert code == B.IS_ERR_BAD_FACT_ID and detail == 0
            assert_parity(o, (code, slots, kb, vb))
            assert _parity(buf, wl) == B.IS_OK
    finally:
        buf.close()


def test_no_alloc_block_capacity_writes_nothing():
    """A batch touching more cache blocks than the fixed work space holds
    (block size 1) writes nothing -- cache and slot mapping untouched -- and
    reports IS_ERR_CAPACITY; the next batch runs normally."""
    _need_gpu()
    model = synth.Model("m", 1, 1, 32, 1e4)
    rng = np.random.default_rng(5)
    lens = rng.integers(30, 50, 40).astype(np.int32)
    ids = [rng.integers(0, 40, 1000), rng.integers(0, 40, 800)]
    sp = np.array([0, 3], np.int32)
    need = max(int(sp[r]) + int(lens[ids[r]].sum()) for r in range(2)) + 1
    big = synth.make_batch(rng, ids, sp, 1, 2 * need, need)
    wl = synth.Workload("cap", model, lens, big, 0)
    assert wl.tokens() > B.IS_NOALLOC_MAX_BLOCKS
    buf = _CallerBuffers(wl)
    try:
        k0, v0, _ = make_cache(wl)
        code, _, slots, kb, vb = buf.run(wl, slot_capacity=wl.tokens())
        assert code == B.IS_ERR_CAPACITY
        assert np.all(slots == -7), "slot mapping written"
        assert np.array_equal(kb, to_bits(k0)) and np.array_equal(vb, to_bits(v0)), "cache written"
        small = synth.make_batch(rng, [rng.integers(0, 40, 7), rng.integers(0, 40, 3)], sp, 1,
                                 2 * need, need)
        assert _parity(buf, synth.Workload("cap-small", model, lens, small, 0)) == B.IS_OK
    finally:
        buf.close()
