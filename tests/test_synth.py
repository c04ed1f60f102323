"""The seeded input generator: determinism, independence of streams and the
shape of its distributions (CPU)."""
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


def test_roughly_standard_normal():
    x = synth.bf16_to_float(synth.bf16_bits(3, 1, np.arange(200_000))).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    assert np.abs(x).max() <= 6.0
    # tails close to the normal's: P(|x| > 2) ~ 0.0455
    assert 0.040 < np.mean(np.abs(x) > 2) < 0.050


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
