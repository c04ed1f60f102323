"""The C checker used by the full-size parity tests applies the same rule as
the element-wise check of the other GPU tests (CPU only): random values
around the tolerance boundary, specials and overflowing outputs."""
import numpy as np

import oracle
from kcheck import kcheck
from test_gpu_parity import BF16_OVERFLOW, k_out_of_tolerance


def test_kcheck_agrees_with_the_element_rule():
    rng = np.random.default_rng(17)
    n = 200_000
    ref = rng.standard_normal(n) * 10.0 ** rng.integers(-6, 4, n)
    # outputs: exact rounding, one-ulp and far-off neighbours, specials
    got = oracle.f64_to_bf16(ref)
    k = rng.integers(0, 6, n)
    got = np.where(k == 1, got + 1, got)
    got = np.where(k == 2, got - 3, got)
    got = np.where(k == 3, rng.integers(0, 1 << 16, n), got).astype(np.uint16)
    # refs next to the overflow threshold, specials
    m = 3000
    ref[:m] = np.concatenate([BF16_OVERFLOW * (1 + rng.uniform(-0.02, 0.02, m // 3)),
                              -BF16_OVERFLOW * (1 + rng.uniform(-0.02, 0.02, m // 3)),
                              rng.choice([np.nan, np.inf, -np.inf, 0.0, -0.0, 3e38, 5e-40],
                                         m - 2 * (m // 3))])
    got[:m] = rng.choice(np.array([0x7F80, 0xFF80, 0x7FC0, 0xFFC1, 0x7F7F, 0xFF7F, 0, 0x8000, 1],
                                  np.uint16), m)
    want = k_out_of_tolerance(got, ref)
    assert 100 < want.sum() < n - 100
    bad, first, exact, cmp = kcheck(got, ref, oracle.f64_to_bf16(ref))
    assert bad == int(want.sum()) and first == int(np.argmax(want))
    same = (got == oracle.f64_to_bf16(ref))[~np.isnan(ref)]
    assert exact == int(same.sum()) and cmp == int((~np.isnan(ref)).sum())
