"""Parity on the whole bf16 range: stores holding signed zeros, subnormals,
magnitudes next to the largest finite bf16, infinities and NaNs with
payloads (signalling ones too), against the CPU oracle.

The pages call injection exact ("not an approximation": Significance /
Claims section of the technical summary) and the values are a bit copy
(Online phase, "Injection"), so V and every untouched slot must match bit
for bit whatever the pattern.  Rotated K follows IEEE arithmetic on both
sides (fp64 in the oracle, fp32 in the kernel): a NaN in a rotation pair
makes both elements of the pair NaN, an infinity times a sine of exactly 0
(position 0) is NaN, sums past the bf16 range round to an infinity.  The
comparison rule (test_gpu_parity.k_out_of_tolerance): NaN where the oracle
has NaN, the same infinity where it has one, and the tolerance elsewhere,
an overflowed output standing for every magnitude from the bf16 overflow
threshold up, with the absolute term scaled by the element's input pair
(|x_a| + |x_b|) -- fp32 arithmetic on inputs near 1e38 is exact only to a
few units in their last place, not in the output's.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from synth.device import CACHE_FILL_SEED, batch_tensors, make_cache, rope_of, to_bits
from kv_cache_injection_gather_b200 import FactStore
from test_gpu_parity import PATHS, assert_parity, new_kref, written_mask

pytestmark = pytest.mark.gpu

SPECIAL = np.array([
    0x0000, 0x8000,                  # +0, -0
    0x0001, 0x8001, 0x007F, 0x803F,  # subnormals
    0x0080, 0x8080,                  # smallest normals
    0x7F7F, 0xFF7F, 0x7F7E, 0xFF00,  # next to the largest finite
    0x7F80, 0xFF80,                  # +inf, -inf
    0x7FC0, 0xFFC0, 0x7FC1, 0xFFFF,  # quiet NaNs, payloads
    0x7F81, 0xFFA5,                  # signalling NaNs with payloads
], np.uint16)


def _special_facts(model, lens, seed):
    """Fact K/V: seeded normal-range values with about a tenth of the
    elements (and some whole rotation pairs) replaced by special patterns."""
    rng = np.random.default_rng(seed)
    L, H, D = model.num_layers, model.num_kv_heads, model.head_dim
    out = []
    for f, n in enumerate(lens):
        k, v = synth.fact_kv(seed, f, L, H, int(n), D)
        for t in (k, v):
            flat = t.reshape(-1)
            pos = rng.choice(flat.size, flat.size // 10, replace=False)
            flat[pos] = SPECIAL[rng.integers(0, len(SPECIAL), len(pos))]
        # both members of some rotate-half and interleaved pairs
        rows = k.reshape(-1, D)
        sel = rng.choice(rows.shape[0], max(1, rows.shape[0] // 8), replace=False)
        i = rng.integers(0, D // 2, len(sel))
        rows[sel, i] = SPECIAL[rng.integers(0, len(SPECIAL), len(sel))]
        rows[sel, i + D // 2] = SPECIAL[rng.integers(0, len(SPECIAL), len(sel))]
        rows[sel, (2 * i) % D] = SPECIAL[rng.integers(0, len(SPECIAL), len(sel))]
        rows[sel, (2 * i + 1) % D] = SPECIAL[rng.integers(0, len(SPECIAL), len(sel))]
        out.append((k, v))
    return out


def _pair_magnitudes(st, b, shape, style, head_major):
    """|x_a| + |x_b| of the stored key pair each injected K element rotates
    (the input scale of the tolerance), placed like the cache; 0 elsewhere."""
    L, H, D = st.L, st.H, st.D
    Bs = b.block_size
    seg, _ = oracle.segment(st, b.req_offsets, b.fact_ids, b.start_pos, b.block_tables, Bs,
                            b.num_blocks)
    ok = seg["slot"] >= 0
    src, slot = seg["src"][ok], seg["slot"][ok]
    x = np.abs(oracle.bf16_to_f64(st.k[:, :, src, :]))           # [L][H][n][D]
    d = np.arange(D)
    partner = (d + D // 2) % D if style == oracle.ROTATE_HALF else d ^ 1
    m = x + x[..., partner]
    out = np.zeros(shape)
    if head_major:
        out[:, slot // Bs, :, slot % Bs] = m.transpose(2, 0, 1, 3)  # [n][L][H][D]
    else:
        out[:, slot // Bs, slot % Bs] = m.transpose(0, 2, 1, 3)     # [L][n][H][D]
    return out


CASES = [
    # name, L, H, D, theta, llama3, B, style, head_major
    ("llama-fixed", 2, 8, 128, 5e5, True, 16, 0, False),
    ("llama-head-major", 2, 8, 128, 5e5, True, 16, 0, True),
    ("interleaved", 2, 4, 128, 1e4, False, 16, 1, False),
    ("generic-h3-d64-b12", 2, 3, 64, 1e4, False, 12, 0, False),
]


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_special_values_parity(case, path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    name, L, H, D, theta, ll3, B_, style, hm = case
    model = synth.Model(name, L, H, D, theta, llama3=ll3)
    rng = np.random.default_rng(sum(name.encode()))
    lens = rng.integers(3, 30, 12).astype(np.int32)
    facts = _special_facts(model, lens, seed=11)
    # requests: one at position 0 (sine exactly 0), unaligned starts, repeats
    ids = [rng.choice(12, 4, replace=False), np.array([3, 3, 7]), rng.choice(12, 6, replace=True),
           np.array([0, 11])]
    sp = np.array([0, 37, 5000, 16], np.int32)
    need = max(-(-(int(sp[r]) + int(lens[ids[r]].sum())) // B_) for r in range(4)) + 1
    batch = synth.make_batch(rng, ids, sp, B_, 4 * need, need)
    wl = synth.Workload(name, model, lens, batch, 11)

    # oracle
    st = oracle.Store(L, H, D, int(lens.sum()), len(lens))
    for k, v in facts:
        st.put(k, v)
    b = batch
    shape = ((L, b.num_blocks, H, B_, D) if hm else (L, b.num_blocks, B_, H, D))
    kc = synth.bf16_block(CACHE_FILL_SEED, synth.TAG_CACHE | 0, shape)
    vc = synth.bf16_block(CACHE_FILL_SEED, synth.TAG_CACHE | 1, shape)
    kref = new_kref(shape)
    strides = oracle.cache_strides(b.num_blocks, B_, H, D, hm)
    f = oracle.rope_inv_freq(D, theta, model.scaling())
    n_tok = wl.tokens()
    rc, oslots = oracle.inject_batch(st, f, b.req_offsets, b.fact_ids, b.start_pos, b.block_tables,
                                     kc, vc, B_, strides=strides, style=style, k_ref=kref)
    assert rc == oracle.OK
    ref = kref[written_mask(kref)]
    assert np.isnan(ref).any() and np.isinf(ref).any(), "no NaN or infinity reached rotated K"
    kmag = _pair_magnitudes(st, b, shape, style, hm)

    # GPU, through the C-ABI
    store = FactStore(L, H, D, rope_of(model, style), int(lens.sum()), len(lens))
    if PATHS[path] is not None:
        store.set_small_batch_limit(PATHS[path])
    for k, v in facts:
        kt = torch.from_numpy(k.view(np.int16)).view(torch.bfloat16)
        vt = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16)
        store.put_fact(kt, vt)
    kg, vg, desc = make_cache(wl, head_major=hm)
    ro, fids, spd, bt = batch_tensors(b)
    slots = torch.full((n_tok,), -7, dtype=torch.int64, device="cuda")
    store.inject(ro, fids, spd, bt, desc, slots)
    grc, _ = store.last_error()
    store.close()
    assert_parity((rc, oslots, kc, vc, kref), (grc, slots.cpu().numpy(), to_bits(kg), to_bits(vg)),
                  kmag)
