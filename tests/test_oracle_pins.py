"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here compares the oracle with itself: each check uses an independent
formulation (complex multiplication, a matrix power, exact rational
arithmetic, torch's own rounding, a gather read of the paged cache, a direct
re-derivation of the prefill) or a closed form, chosen so that a dropped term,
a wrong sign or index or a transposed operand in the oracle fails one of them.

Passages (summaries of "InferScale: GPU-Native KV Injection for Personalized
LLM Serving", gist.science/{ja,nl,it}/paper/2607.27090, technical summary):
  * Online phase, "Dynamic rotation": stored keys get the RoPE rotation of
    their new serving positions in one contiguous segment.
  * Online phase, "Theoretical guarantee" and Contributions, "Chunked RoPE"
    (Theorem 6): re-rotation is exact; scores equal prefill at those positions.
  * Contributions, "Retrieve-and-inject inference" (Theorem 3): injecting
    precomputed KV at the intended positions equals prompt injection.
  * Online phase, "Injection": scatter-copy into the paged KV cache.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LLAMA3 = dict(factor=8.0, low_freq_factor=1.0, high_freq_factor=4.0, original_max_position=8192)


# ----------------------------------------------------------------- bf16 rounding

def _bf16_value(b: int) -> Fraction:
    return Fraction(float(oracle.bf16_to_f64(np.array([b], np.uint16))[0]))


def test_bf16_roundtrip_exhaustive():
    """Every finite bf16 value converts to fp64 and back to itself."""
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    finite = (b & 0x7F80) != 0x7F80
    back = oracle.f64_to_bf16(oracle.bf16_to_f64(b[finite]))
    assert np.array_equal(back, b[finite])


def test_bf16_rounding_is_nearest_ties_even():
    """Exact rational check: the result is a nearest bf16, and exact midpoints
    go to the neighbour with an even last mantissa bit."""
    rng = np.random.default_rng(1)
    xs = list(rng.standard_normal(300) * 10.0 ** rng.integers(-40, 38, 300))
    xs += [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 2.0 ** -130 * 1.5, 3.0e38, 1.0 - 2.0 ** -10]
    # exact midpoints between random neighbouring positive bf16 values
    for b in rng.integers(0x0080, 0x7F00, 200):
        lo, hi = _bf16_value(int(b)), _bf16_value(int(b) + 1)
        xs.append(float((lo + hi) / 2))
    out = oracle.f64_to_bf16(np.array(xs))
    for x, r in zip(xs, out):
        r = int(r)
        X = Fraction(x)
        mag = r & 0x7FFF
        assert (r >> 15) == (1 if x < 0 else 0)
        val = _bf16_value(r)
        dist = abs(X - val)
        for nb in (mag - 1, mag + 1):
            if 0 <= nb < 0x7F80:
                nv = _bf16_value(nb | (r & 0x8000))
                d2 = abs(X - nv)
                assert dist <= d2, (x, hex(r))
                if dist == d2:  # tie: must take the even mantissa
                    assert mag % 2 == 0, (x, hex(r))


def test_bf16_matches_torch_on_fp32_inputs():
    """For values already in fp32, one RNE step to bf16 is what torch does."""
    import torch
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(100_000) * 10.0 ** rng.integers(-30, 30, 100_000)).astype(np.float32)
    ours = oracle.f64_to_bf16(x.astype(np.float64))
    theirs = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)


def test_bf16_special_values_and_overflow():
    """Outside the finite range: signed zeros keep their sign, infinities map
    to themselves, a NaN stays a NaN (quiet), and the overflow threshold of
    round-to-nearest-even is the midpoint between the largest finite bf16
    (2^128 - 2^120) and 2^128 -- the tie rounds up to the infinity, whose
    mantissa is the even one.  torch's fp32 -> bf16 (an independent
    implementation) agrees on fp32 inputs next to the threshold, at the
    subnormal end and on the specials."""
    b = oracle.f64_to_bf16(np.array([0.0, -0.0, np.inf, -np.inf, np.nan, -np.nan]))
    assert list(b[:4]) == [0x0000, 0x8000, 0x7F80, 0xFF80]
    for x in b[4:]:
        assert (x & 0x7F80) == 0x7F80 and (x & 0x007F) != 0 and (x & 0x0040), hex(x)
    top = 2.0 ** 128 - 2.0 ** 120
    mid = 2.0 ** 128 - 2.0 ** 119
    xs = np.array([top, np.nextafter(mid, 0.0), mid, np.nextafter(mid, np.inf), 2.0 ** 128, 1e300,
                   -np.nextafter(mid, 0.0), -mid])
    assert list(oracle.f64_to_bf16(xs)) == [0x7F7F, 0x7F7F, 0x7F80, 0x7F80, 0x7F80, 0x7F80,
                                             0xFF7F, 0xFF80]
    import torch
    f32 = np.array([3.38e38, 3.3953e38, 3.3961e38, 3.3962e38, 3.4e38, np.finfo(np.float32).max,
                    -3.3962e38, 1e-45, -1e-45, 9.2e-41, 1.17e-38, 2.0 ** -133, 3 * 2.0 ** -134,
                    0.0, -0.0, np.inf, -np.inf], np.float32)
    ours = oracle.f64_to_bf16(f32.astype(np.float64))
    theirs = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs), (ours, theirs)


# --------------------------------------------------------------- RoPE frequencies

@pytest.mark.parametrize("D,theta", [(64, 1.0e4), (128, 5.0e5), (128, 1.0e6), (4, 100.0)])
def test_inv_freq_closed_form(D, theta):
    f = oracle.rope_inv_freq(D, theta)
    assert f[0] == 1.0
    # constant ratio theta^(-2/D) between neighbours
    assert np.allclose(f[1:] / f[:-1], theta ** (-2.0 / D), rtol=1e-13, atol=0)
    if D % 4 == 0:  # the middle frequency is theta^(-1/2)
        assert math.isclose(f[D // 4], 1.0 / math.sqrt(theta), rel_tol=1e-14)


def test_llama3_scaling_band_edges_and_identity():
    """Llama-3.1 rule: wavelengths below orig/high keep their frequency,
    above orig/low are divided by the factor, and the blend joins both
    continuously at the two edges; factor 1 leaves every frequency alone."""
    lo_wl, hi_wl = 8192.0, 2048.0
    for lam in (100.0, 2047.9, 8192.1, 1.0e6):
        f = 2 * math.pi / lam
        expect = f if lam < hi_wl else f / 8.0
        assert math.isclose(oracle.llama3_scale(f), expect, rel_tol=1e-15)
    for edge, target in ((hi_wl, 1.0), (lo_wl, 1.0 / 8.0)):
        for eps in (1e-9, -1e-9):
            lam = edge * (1 + eps)
            f = 2 * math.pi / lam
            assert math.isclose(oracle.llama3_scale(f) / f, target, rel_tol=1e-6)
    # the blended ratio moves monotonically from 1 to 1/8 across the band
    lams = np.linspace(hi_wl * 1.0001, lo_wl * 0.9999, 50)
    ratios = [oracle.llama3_scale(2 * math.pi / l) / (2 * math.pi / l) for l in lams]
    assert all(a >= b for a, b in zip(ratios, ratios[1:]))
    base = oracle.rope_inv_freq(128, 5.0e5)
    same = oracle.rope_inv_freq(128, 5.0e5, dict(factor=1.0, low_freq_factor=1.0,
                                                 high_freq_factor=4.0, original_max_position=8192))
    assert np.allclose(same, base, rtol=1e-15, atol=0)


def test_llama3_blend_interior_values():
    """Inside the band the rule mixes f/factor and f linearly in orig/lambda;
    two interior points whose mixing weight is a simple fraction fix the
    ratio scaled/unscaled exactly (a weight that is monotone and right at
    both edges but not linear, e.g. its square, misses both):
      factor 8, low 1, high 4, orig 8192, lambda 4096: weight 1/3, ratio
        (2/3)(1/8) + 1/3 = 5/12;
      factor 4, low 2, high 8, orig 16384, lambda 16384/5: weight 1/2,
        ratio (1/2)(1/4) + 1/2 = 5/8."""
    for lam, args, ratio in ((4096.0, (8.0, 1.0, 4.0, 8192.0), 5.0 / 12.0),
                             (16384.0 / 5.0, (4.0, 2.0, 8.0, 16384.0), 5.0 / 8.0)):
        f = 2 * math.pi / lam
        assert math.isclose(oracle.llama3_scale(f, *args) / f, ratio, rel_tol=1e-13)


def test_llama3_no_frequency_on_a_band_edge():
    """For D=128, theta=5e5 no wavelength equals 2048 or 8192 exactly, so the
    strict inequalities of the rule need no tie-break."""
    f = oracle.rope_inv_freq(128, 5.0e5)
    lam = 2 * np.pi / f
    assert np.all(np.abs(lam - 2048.0) > 1.0) and np.all(np.abs(lam - 8192.0) > 1.0)
    scaled = oracle.rope_inv_freq(128, 5.0e5, LLAMA3)
    kept, divided = lam < 2048.0, lam > 8192.0
    assert kept.any() and divided.any() and (~kept & ~divided).any()
    assert np.array_equal(scaled[kept], f[kept])
    assert np.allclose(scaled[divided], f[divided] / 8.0, rtol=1e-15, atol=0)


# ------------------------------------------------------------------- RoPE rotation

def _complex_rope(x, pos, inv_freq, style):
    """Independent form: pairs as complex numbers times exp(i * pos * f)."""
    D = x.shape[-1]
    if style == oracle.ROTATE_HALF:
        z = x[..., : D // 2] + 1j * x[..., D // 2:]
    else:
        z = x[..., 0::2] + 1j * x[..., 1::2]
    z = z * np.exp(1j * np.asarray(pos, np.float64)[..., None] * inv_freq)
    y = np.empty_like(x)
    if style == oracle.ROTATE_HALF:
        y[..., : D // 2], y[..., D // 2:] = z.real, z.imag
    else:
        y[..., 0::2], y[..., 1::2] = z.real, z.imag
    return y


def test_rope_closed_form_d4():
    """D=4, theta=100: frequencies (1, 0.1).  The key (1, 0, 0, 1) at position
    3 becomes (cos 3, -sin 0.3, sin 3, cos 0.3) with rotate-half pairs
    (0,2), (1,3), and (cos 3, sin 3, -sin 0.3, cos 0.3) with interleaved pairs
    (0,1), (2,3)."""
    f = oracle.rope_inv_freq(4, 100.0)
    assert np.allclose(f, [1.0, 0.1], rtol=1e-15)
    x = np.array([1.0, 0.0, 0.0, 1.0])
    y = oracle.rope_rows(x[None], [3], f, oracle.ROTATE_HALF)[0]
    assert np.allclose(y, [math.cos(3), -math.sin(0.3), math.sin(3), math.cos(0.3)],
                       rtol=0, atol=1e-15)
    x2 = np.array([1.0, 0.0, 0.0, 1.0])
    y2 = oracle.rope_rows(x2[None], [3], f, oracle.INTERLEAVED)[0]
    assert np.allclose(y2, [math.cos(3), math.sin(3), -math.sin(0.3), math.cos(0.3)],
                       rtol=0, atol=1e-15)


@pytest.mark.parametrize("style", [oracle.ROTATE_HALF, oracle.INTERLEAVED])
@pytest.mark.parametrize("D,theta,scaling", [(64, 1e4, None), (128, 5e5, LLAMA3), (128, 1e6, None)])
def test_rope_matches_complex_multiplication(style, D, theta, scaling):
    rng = np.random.default_rng(3)
    f = oracle.rope_inv_freq(D, theta, scaling)
    x = rng.standard_normal((200, D))
    pos = rng.integers(-5000, 140_000, 200)
    y = oracle.rope_rows(x, pos, f, style)
    assert np.allclose(y, _complex_rope(x, pos, f, style), rtol=0, atol=1e-9)


@pytest.mark.parametrize("style", [oracle.ROTATE_HALF, oracle.INTERLEAVED])
def test_rope_is_a_power_of_the_unit_step(style):
    """R(p) = R(1)^p: the matrix of one step, raised to p by numpy."""
    D = 16
    f = oracle.rope_inv_freq(D, 10.0)
    R1 = oracle.rope_rows(np.eye(D), np.ones(D, np.int64), f, style).T  # columns = R(1) e_j
    rng = np.random.default_rng(4)
    x = rng.standard_normal(D)
    for p in (0, 1, 2, 7, 37):
        want = np.linalg.matrix_power(R1, p) @ x
        got = oracle.rope_rows(x[None], [p], f, style)[0]
        assert np.allclose(got, want, rtol=0, atol=1e-11)


@pytest.mark.parametrize("style", [oracle.ROTATE_HALF, oracle.INTERLEAVED])
def test_rope_non_finite_inputs_follow_ieee_pairwise(style):
    """A NaN or an infinity in a key changes only its own rotation pair, and
    within it follows IEEE arithmetic of x cos - y sin, y cos + x sin: a NaN
    makes both members NaN; an infinity with a finite partner gives
    infinities signed by cos and sin, except that at position 0 the partner
    becomes inf * sin 0 = NaN."""
    D = 16
    f = oracle.rope_inv_freq(D, 1e4)
    pair = (lambda i: (i, i + D // 2)) if style == oracle.ROTATE_HALF else (lambda i: (2 * i, 2 * i + 1))
    rng = np.random.default_rng(9)
    base = rng.standard_normal(D)
    for pos in (0, 3, 1000):
        clean = oracle.rope_rows(base[None], [pos], f, style)[0]
        for i, val in ((2, np.nan), (5, np.inf), (6, -np.inf)):
            a, b = pair(i)
            x = base.copy()
            x[a] = val
            y = oracle.rope_rows(x[None], [pos], f, style)[0]
            others = np.ones(D, bool)
            others[[a, b]] = False
            assert np.array_equal(y[others], clean[others])
            ang = pos * f[i]
            c, s_ = math.cos(ang), math.sin(ang)
            if np.isnan(val):
                assert np.isnan(y[a]) and np.isnan(y[b])
            else:
                assert y[a] == val * np.sign(c)
                if pos == 0:
                    assert np.isnan(y[b])
                else:
                    assert y[b] == val * np.sign(s_)


def test_rope_group_laws_and_norm():
    rng = np.random.default_rng(5)
    for D, theta, sc in ((64, 1e4, None), (128, 5e5, LLAMA3)):
        f = oracle.rope_inv_freq(D, theta, sc)
        x = rng.standard_normal((50, D))
        p = rng.integers(0, 5000, 50)
        q = rng.integers(0, 5000, 50)
        a = oracle.rope_rows(oracle.rope_rows(x, p, f), q, f)
        assert np.allclose(a, oracle.rope_rows(x, p + q, f), rtol=0, atol=1e-10)
        back = oracle.rope_rows(oracle.rope_rows(x, p, f), -p, f)
        assert np.allclose(back, x, rtol=0, atol=1e-12)
        y = oracle.rope_rows(x, p, f)
        h = D // 2
        assert np.allclose(x[:, :h] ** 2 + x[:, h:] ** 2, y[:, :h] ** 2 + y[:, h:] ** 2,
                           rtol=1e-12, atol=1e-12)
        assert np.array_equal(oracle.rope_rows(x, np.zeros(50, np.int64), f), x)


@pytest.mark.parametrize("D,theta,scaling", [(64, 1e4, None), (128, 5e5, LLAMA3), (128, 5e5, None)])
def test_theorem6_scores_depend_only_on_relative_position(D, theta, scaling):
    """Brute force over every placement p_k in [0, 256) with p_q = p_k + delta:
    <R(p_q) q, R(p_k) k> is one number, equal to <q, R(-delta) k>."""
    rng = np.random.default_rng(6)
    f = oracle.rope_inv_freq(D, theta, scaling)
    q, k = rng.standard_normal(D), rng.standard_normal(D)
    for delta in (0, 1, 17, 200):
        pk = np.arange(256)
        qs = oracle.rope_rows(np.broadcast_to(q, (256, D)), pk + delta, f)
        ks = oracle.rope_rows(np.broadcast_to(k, (256, D)), pk, f)
        scores = np.einsum("nd,nd->n", qs, ks)
        ref = q @ oracle.rope_rows(k[None], [-delta], f)[0]
        assert np.allclose(scores, ref, rtol=1e-12, atol=1e-12 * np.abs(q).sum() * np.abs(k).sum())


# ----------------------------------------------------------------- store and inject

def _build_store(wl):
    m = wl.model
    T = int(wl.fact_lens.sum())
    st = oracle.Store(m.num_layers, m.num_kv_heads, m.head_dim, T, len(wl.fact_lens))
    facts = []
    for f, n in enumerate(wl.fact_lens):
        k, v = synth.fact_kv(wl.seed, f, m.num_layers, m.num_kv_heads, int(n), m.head_dim)
        assert st.put(k, v) == f
        facts.append((k, v))
    return st, facts


def _cache(wl, fill_seed=7):
    m, b = wl.model, wl.batch
    shape = (m.num_layers, b.num_blocks, b.block_size, m.num_kv_heads, m.head_dim)
    k = synth.bf16_block(fill_seed, synth.TAG_CACHE | 0, shape)
    v = synth.bf16_block(fill_seed, synth.TAG_CACHE | 1, shape)
    return k, v


def test_store_put_layout():
    wl = synth.tiny(0)
    st, facts = _build_store(wl)
    assert np.array_equal(st.off[:64], np.concatenate([[0], np.cumsum(wl.fact_lens)[:-1]]))
    assert np.array_equal(st.len[:64], wl.fact_lens)
    for f in (0, 13, 63):
        k, v = facts[f]
        o, n = st.off[f], st.len[f]
        assert np.array_equal(st.k[:, :, o:o + n, :], k)
        assert np.array_equal(st.v[:, :, o:o + n, :], v)


def _gather_view(cache, bt_row, B, positions):
    """Read logical positions through a block table (the consumer's view)."""
    return np.stack([cache[:, bt_row[p // B], p % B] for p in positions], axis=1)


@pytest.mark.parametrize("start", [32, 37, 0])
@pytest.mark.parametrize("style", [oracle.ROTATE_HALF, oracle.INTERLEAVED])
def test_inject_gather_view_tiny(start, style):
    """Reading the cache back through the block table at positions
    start .. start+S-1 gives the facts' V rows in retrieval order (bit copy)
    and their K rows rotated to those positions (complex form, one bf16
    rounding); every other slot keeps its previous bits."""
    wl = synth.tiny(0, start_pos=start)
    m, b = wl.model, wl.batch
    st, facts = _build_store(wl)
    f = oracle.rope_inv_freq(m.head_dim, m.rope_theta)
    kc, vc = _cache(wl)
    k0, v0 = kc.copy(), vc.copy()
    kref = np.zeros(kc.shape, np.float64)
    rc, slots = oracle.inject_batch(st, f, b.req_offsets, b.fact_ids, b.start_pos, b.block_tables,
                                    kc, vc, b.block_size, style=style, k_ref=kref)
    assert rc == oracle.OK
    ids = b.fact_ids
    k_seq = np.concatenate([facts[i][0] for i in ids], axis=2)  # [L][H][S][D]
    v_seq = np.concatenate([facts[i][1] for i in ids], axis=2)
    S = k_seq.shape[2]
    pos = np.arange(start, start + S)
    got_v = _gather_view(vc, b.block_tables[0], b.block_size, pos)      # [L][S][H][D]
    assert np.array_equal(got_v, v_seq.transpose(0, 2, 1, 3))
    want_k = _complex_rope(synth.bf16_to_float(k_seq).astype(np.float64),
                           pos[None, None, :], f, style)
    got_kref = _gather_view(kref, b.block_tables[0], b.block_size, pos)
    assert np.allclose(got_kref, want_k.transpose(0, 2, 1, 3), rtol=0, atol=1e-12)
    got_k = _gather_view(kc, b.block_tables[0], b.block_size, pos)
    assert np.array_equal(got_k, oracle.f64_to_bf16(got_kref))
    # slot mapping is the physical slot of each logical position
    assert np.array_equal(slots, b.block_tables[0][pos // 16] * 16 + pos % 16)
    # untouched slots: exactly the slots not in the mapping
    touched = np.zeros(b.num_blocks * b.block_size, bool)
    touched[slots] = True
    kf = kc.reshape(m.num_layers, -1, m.num_kv_heads, m.head_dim)
    k0f = k0.reshape(kf.shape)
    vf, v0f = vc.reshape(kf.shape), v0.reshape(kf.shape)
    assert np.array_equal(kf[:, ~touched], k0f[:, ~touched])
    assert np.array_equal(vf[:, ~touched], v0f[:, ~touched])
    if start == 0:  # position 0 is the identity rotation: K copied bit for bit
        assert np.array_equal(got_k[:, 0], k_seq[:, :, 0, :])


def test_theorem3_single_linear_layer():
    """A tiny random single linear layer: prefill of the fact tokens at their
    serving positions (K = RoPE(bf16(x W_k)), V = bf16(x W_v), written through
    the block table) gives the same cache bytes as storing the pre-RoPE
    bf16(x W_k), bf16(x W_v) once and injecting them.  A single layer has no
    cross-token mixing, so this holds whatever context window encoded them."""
    rng = np.random.default_rng(8)
    L, H, D, dm = 1, 2, 64, 96
    f = oracle.rope_inv_freq(D, 1e4)
    Wk = rng.standard_normal((dm, H * D)) / math.sqrt(dm)
    Wv = rng.standard_normal((dm, H * D)) / math.sqrt(dm)
    lens = [11, 16, 5, 23]
    xs = [rng.standard_normal((n, dm)) for n in lens]
    bf = lambda a: oracle.f64_to_bf16(a)  # noqa: E731 -- bf16 storage of projections
    st = oracle.Store(L, H, D, sum(lens), len(lens))
    for x in xs:
        kp = bf(x @ Wk).reshape(len(x), H, D).transpose(1, 0, 2)[None]
        vp = bf(x @ Wv).reshape(len(x), H, D).transpose(1, 0, 2)[None]
        st.put(kp, vp)
    order = np.array([2, 0, 3, 1], np.int32)
    start, B, NB = 21, 16, 12
    bt = rng.permutation(NB).astype(np.int32)[None]
    shape = (L, NB, B, H, D)
    kc, vc = np.zeros(shape, np.uint16), np.zeros(shape, np.uint16)
    rc, _ = oracle.inject_batch(st, f, [0, 4], order, [start], bt, kc, vc, B)
    assert rc == oracle.OK
    # prefill, written independently: tokens in retrieval order, one position each
    kp_, vp_ = np.zeros(shape, np.uint16), np.zeros(shape, np.uint16)
    p = start
    for j in order:
        for t in range(lens[j]):
            k_tok = bf(xs[j][t] @ Wk).reshape(H, D)
            k_rot = _complex_rope(oracle.bf16_to_f64(k_tok), np.full(H, p), f, oracle.ROTATE_HALF)
            blk, o = bt[0][p // B], p % B
            kp_[0, blk, o] = bf(k_rot)
            vp_[0, blk, o] = bf(xs[j][t] @ Wv).reshape(H, D)
            p += 1
    assert np.array_equal(kc, kp_) and np.array_equal(vc, vp_)


def test_inject_errors_and_isolation():
    """Invalid requests are skipped whole and reported; valid ones still land."""
    wl = synth.tiny(0)
    m, b = wl.model, wl.batch
    st, _ = _build_store(wl)
    f = oracle.rope_inv_freq(m.head_dim, m.rope_theta)
    ids = np.concatenate([b.fact_ids[:2], [999], b.fact_ids[2:4]]).astype(np.int32)
    ro = np.array([0, 2, 3, 5], np.int32)
    sp = np.array([0, 40, 300], np.int32)
    bt = np.stack([np.arange(0, 20), np.arange(20, 40), np.arange(40, 60)]).astype(np.int32)
    kc, vc = _cache(wl)
    k0 = kc.copy()
    rc, slots = oracle.inject_batch(st, f, ro, ids, sp, bt, kc, vc, 16)
    assert rc == oracle.ERR_BAD_FACT_ID
    n0 = int(wl.fact_lens[ids[:2]].sum())
    assert np.all(slots[:n0] >= 0) and np.all(slots[n0:] == -1)  # request 2 overflows
    assert not np.array_equal(kc, k0)
    # position past the block table
    kc2, vc2 = _cache(wl)
    rc, slots = oracle.inject_batch(st, f, [0, 2], ids[:2], [20 * 16 - 5], bt[:1], kc2, vc2, 16)
    assert rc == oracle.ERR_POSITION and np.all(slots == -1)
    # block table entry outside the cache: those slots only are skipped
    kc3, vc3 = _cache(wl)
    bad = bt[:1].copy()
    bad[0, 3] = 64
    rc, slots = oracle.inject_batch(st, f, [0, 2], ids[:2], [40], bad, kc3, vc3, 16)
    assert rc == oracle.ERR_BAD_BLOCK
    pos = 40 + np.arange(len(slots))
    assert np.all((slots == -1) == (pos // 16 == 3))
    # CSR that does not cover the id list: nothing composed, nothing written
    kc4, vc4 = _cache(wl)
    k4 = kc4.copy()
    rc, _ = oracle.inject_batch(st, f, [0, 1], ids[:2], [0], bt[:1], kc4, vc4, 16)
    assert rc == oracle.ERR_INVALID_ARG and np.array_equal(kc4, k4)
    # offsets that decrease (overlapping ranges): the whole batch is rejected
    rc, _ = oracle.inject_batch(st, f, [0, 3, 2, 4], ids[:4], [0, 40, 80], bt, kc4, vc4, 16)
    assert rc == oracle.ERR_INVALID_ARG and np.array_equal(kc4, k4)
    # slot output too small: nothing written
    rc, _ = oracle.inject_batch(st, f, [0, 2], ids[:2], [0], bt[:1], kc4, vc4, 16,
                                slot_capacity=3)
    assert rc == oracle.ERR_CAPACITY and np.array_equal(kc4, k4)


def test_segment_positions_brute_force():
    """Positions of a many-request batch by direct enumeration."""
    rng = np.random.default_rng(9)
    lens = rng.integers(1, 40, 30).astype(np.int32)
    st = oracle.Store(1, 1, 8, int(lens.sum()), 30)
    for n in lens:
        st.put(np.zeros((1, 1, n, 8), np.uint16), np.zeros((1, 1, n, 8), np.uint16))
    reqs = [rng.choice(30, rng.integers(0, 6), replace=True) for _ in range(7)]
    ro = np.concatenate([[0], np.cumsum([len(r) for r in reqs])]).astype(np.int32)
    ids = np.concatenate(reqs).astype(np.int32)
    sp = rng.integers(0, 50, 7).astype(np.int32)
    bt = rng.permutation(7 * 20).astype(np.int32).reshape(7, 20)
    seg, st_ = oracle.segment(st, ro, ids, sp, bt, 16, 140)
    assert st_ == oracle.OK
    off = np.concatenate([[0], np.cumsum(lens)[:-1]])
    want = []
    for r, fl in enumerate(reqs):
        p = sp[r]
        for fid in fl:
            for t in range(lens[fid]):
                want.append((r, off[fid] + t, p, bt[r][p // 16] * 16 + p % 16))
                p += 1
    got = list(zip(seg["request"], seg["src"], seg["pos"], seg["slot"]))
    assert [tuple(map(int, w)) for w in want] == [tuple(map(int, g)) for g in got]


def test_slot_formula_and_table_edges():
    """slot = table[pos / B] * B + pos mod B inside the table; -1 for a
    negative position, a position at or past the table's end, or an entry
    outside the cache.  The row is a view into a longer array whose next
    entry is a valid block, so reading one entry past the row would show."""
    B, nb = 16, 64
    full = np.array([5, 9, 2, 7], np.int32)
    row = full[:3]
    for pos in range(0, 3 * B):
        assert oracle.slot(row, B, nb, pos) == int(row[pos // B]) * B + pos % B
    assert oracle.slot(row, B, nb, 3 * B) == -1
    assert oracle.slot(row, B, nb, 3 * B + 5) == -1
    assert oracle.slot(row, B, nb, -1) == -1
    assert oracle.slot(np.array([5, 64], np.int32), B, nb, B) == -1   # block id == num_blocks
    assert oracle.slot(np.array([5, -1], np.int32), B, nb, B + 3) == -1


def test_golden_tiny_regression():
    """The oracle's result on the tiny workload, frozen by
    tests/golden/make_golden.py (which calls only the oracle and the input
    generator).  A change to the oracle's arithmetic must update this file in
    a commit that names the passage or reading that justifies it."""
    import hashlib
    with open(os.path.join(GOLDEN, "tiny_inject.json")) as fh:
        gold = json.load(fh)
    for case in gold["cases"]:
        wl = synth.tiny(gold["seed"], start_pos=case["start_pos"])
        m, b = wl.model, wl.batch
        st, _ = _build_store(wl)
        f = oracle.rope_inv_freq(m.head_dim, m.rope_theta)
        kc, vc = _cache(wl, gold["cache_fill_seed"])
        rc, slots = oracle.inject_batch(st, f, b.req_offsets, b.fact_ids, b.start_pos,
                                        b.block_tables, kc, vc, b.block_size)
        assert rc == case["status"]
        assert slots.tolist() == case["slot_mapping"]
        assert hashlib.sha256(kc.tobytes()).hexdigest() == case["k_cache_sha256"]
        assert hashlib.sha256(vc.tobytes()).hexdigest() == case["v_cache_sha256"]
