"""The seeded input generator: determinism, independence of streams, the
normal distribution of its bulk values and the shapes of the workloads
(CPU)."""
import numpy as np

import synth


def test_counter_based_and_deterministic():
    a = synth.bf16_bits(0, 5, np.arange(1000))
    b = synth.bf16_bits(0, 5, np.arange(1000))
    assert np.array_equal(a, b)
    # any element can be regenerated alone
    idx = np.array([999, 3, 500])
    assert np.array_equal(synth.bf16_bits(0, 5, idx), a[idx])
    assert not np.array_equal(a, synth.bf16_bits(1, 5, np.arange(1000)))
    assert not np.array_equal(a, synth.bf16_bits(0, 6, np.arange(1000)))


def test_threshold_table_is_the_normal_distribution():
    """Q_c / 2^64 = P(|X| < h_c) for X ~ N(0, 1), h_c the midpoint between
    bf16 codes c and c + 1: checked against scipy's normal distribution (an
    independent implementation) to 1e-15 absolute, and non-decreasing."""
    from scipy.stats import norm
    first, q = synth.normal_table()
    assert np.all(q[1:] >= q[:-1]) and q[0] > 0
    codes = np.arange(first, first + len(q), dtype=np.uint32)
    lo = (codes << 16).view(np.float32).astype(np.float64)
    hi = ((codes + 1) << 16).view(np.float32).astype(np.float64)
    h = 0.5 * (lo + hi)
    want = np.where(h <= 1.0, 2.0 * norm.cdf(h) - 1.0, 1.0 - 2.0 * norm.sf(h))
    assert np.max(np.abs(q.astype(np.float64) / 2.0 ** 64 - want)) < 1e-15
    # the support: from below 2^-64 up to about 9.1
    assert lo[0] < 2.0 ** -64 and 9.0 < hi[-1] < 9.5


def test_standard_normal_samples():
    """Two million samples: symmetric, unit variance, and the counts of |x|
    in bins agree with N(0, 1) rounded to bf16 (chi-square, 11 bins; the
    expected counts from scipy at the bf16 rounding midpoints of the bin
    edges)."""
    from scipy.stats import chi2, norm
    bits = synth.bf16_bits(3, 1, np.arange(2_000_000))
    x = synth.bf16_to_float(bits).astype(np.float64)
    assert abs(x.mean()) < 0.003 and abs(x.std() - 1.0) < 0.003
    assert abs(np.mean(bits >> 15) - 0.5) < 0.002
    assert np.abs(x).max() > 4.5
    edges = np.array([0.0, 0.125, 0.25, 0.5, 0.75, 1.0, 1.5, 2.0, 2.5, 3.0, 4.0, np.inf])
    # a rounded value lands in [e_i, e_(i+1)) exactly when |X| lies in
    # [m(e_i), m(e_(i+1))), m(e) the midpoint between the bf16 value e and
    # the next one below: e - 2^(k-8) for e in (2^k, 2^(k+1)), e - 2^(k-9)
    # for e = 2^k (the spacing halves below a power of two)
    def mid_below(e):
        k = np.floor(np.log2(e))
        return e - 2.0 ** (k - 9 if e == 2.0 ** k else k - 8)

    below = np.array([0.0] + [mid_below(e) for e in edges[1:-1]] + [np.inf])
    p = 2.0 * (norm.cdf(below[1:]) - norm.cdf(below[:-1]))
    n = np.histogram(np.abs(x), bins=edges)[0]
    stat = float(((n - p * len(x)) ** 2 / (p * len(x))).sum())
    assert stat < chi2.ppf(0.9995, len(p) - 1), stat


def test_fact_rows_match_fact_tensor():
    k, v = synth.fact_kv(0, 17, 2, 3, 9, 64)
    rows = synth.fact_rows(0, 17, True, 2, 3, 9, 64, [1, 0], [2, 1], [8, 0])
    assert np.array_equal(rows[0], v[1, 2, 8]) and np.array_equal(rows[1], v[0, 1, 0])


def test_workloads_shapes():
    wl = synth.tiny(0)
    assert wl.fact_lens.min() >= 8 and wl.fact_lens.max() <= 24 and len(wl.fact_lens) == 64
    assert len(set(wl.batch.fact_ids.tolist())) == 5 and wl.batch.start_pos[0] == 32
    assert sorted(wl.batch.block_tables[0].tolist()) == list(range(64))
    big = synth.llama_batch(0)
    b = big.batch
    assert b.num_requests == 100 and b.req_offsets[-1] == 5000 and b.max_blocks == 256
    for r in range(100):
        ids = b.fact_ids[b.req_offsets[r]:b.req_offsets[r + 1]]
        assert len(set(ids.tolist())) == 50
    assert len(set(b.block_tables.ravel().tolist())) == 25600  # disjoint block sets
    assert 190_000 < big.tokens() < 210_000
    sw = synth.sweep(synth.QWEN25_7B, 16, 20)
    assert sw.fact_lens.min() >= 8 and sw.fact_lens.max() <= 96
    assert 28 <= np.median(sw.fact_lens) <= 36
