"""The work-unit sizing rule of the inject kernels (unit_size in
kv_cache_injection_gather_b200/csrc/inject_kernels.cuh, transcribed here with
its default knobs) checked for the properties the kernels and their
documentation rely on, over far more shapes than the GPU tests run:

  * the layer ranges of a block's units partition [0, L), none empty;
  * a batch whose one-layer units fit in two waves gets about one wave of
    units (latency): at most the grid plus one unit per block, since layers
    are grouped in equal ranges;
  * a large batch gets units of at least 16 (layer, head) rows and two
    layers whenever the model has them;
  * the unit count fits the kernels' 32-bit counters.
"""
from __future__ import annotations

import itertools

UNITS_PER_CTA, MIN_ROWS, ROWS_LARGE, UNITS_PER_CTA_MIN = 256, 16, 32, 32


def unit_size(total_blocks: int, L: int, H: int, grid: int) -> tuple[int, int]:
    upb = 1
    if total_blocks > 0 and total_blocks * L <= 2 * grid:
        per = (total_blocks * L + grid - 1) // grid
        upb = (L + per - 1) // per
    elif total_blocks > 0:
        h = max(H, 1)
        lmin = min(L, max(2, (MIN_ROWS + h - 1) // h))
        lbig = min(L, max(2, (ROWS_LARGE + h - 1) // h))
        cap_big = max(1, L // lbig)
        cap = cap_big if total_blocks * cap_big >= UNITS_PER_CTA_MIN * grid else max(1, L // lmin)
        want = (grid * UNITS_PER_CTA + total_blocks - 1) // total_blocks
        upb = max(1, min(want, cap))
    lpu = (L + upb - 1) // upb
    upb = (L + lpu - 1) // lpu
    return lpu, upb


def test_unit_sizing_invariants():
    grids = (296, 444, 148)
    layers = (1, 2, 3, 5, 12, 16, 28, 32, 40, 61, 80)
    heads = (1, 2, 3, 4, 8, 16)
    blocks = (1, 2, 5, 9, 10, 37, 100, 147, 148, 296, 297, 592, 1000, 4625, 12_600, 65_536,
              1 << 20)
    for grid, L, H, tb in itertools.product(grids, layers, heads, blocks):
        lpu, upb = unit_size(tb, L, H, grid)
        assert 1 <= lpu <= L and 1 <= upb <= L
        ranges = [(g * lpu, min(L, (g + 1) * lpu)) for g in range(upb)]
        assert all(a < b for a, b in ranges), (grid, L, H, tb, lpu, upb)
        assert ranges[0][0] == 0 and ranges[-1][1] == L
        assert all(ranges[i][1] == ranges[i + 1][0] for i in range(upb - 1))
        if tb * L <= 2 * grid:
            assert tb * upb <= grid + tb, "one-wave batch: about one wave of units"
        else:
            assert lpu >= min(L, 2)
            assert lpu * H >= min(MIN_ROWS, L * H) or lpu == L
        assert tb * upb < 2 ** 31


def test_unit_sizing_at_the_benchmark_shapes():
    # Llama-3.1-8B batch: ~12.6k touched blocks, 32 layers, 8 heads -> units of 6 layers
    assert unit_size(12_633, 32, 8, 296) == (6, 6)
    # Qwen2.5-7B, R=100 k=20: ~4.6k blocks, 4 heads -> 10-layer units (32-row rule)
    assert unit_size(4_625, 28, 4, 296) == (10, 3)
    # one Llama request of 10 blocks: one wave, two layers per unit
    assert unit_size(10, 32, 8, 296) == (2, 16)
