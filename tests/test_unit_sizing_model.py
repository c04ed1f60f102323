"""The work-unit sizing rule of the inject kernels (unit_size in
kv_cache_injection_gather_b200/csrc/inject_kernels.cuh, transcribed here with
its default knobs) checked for the properties the kernels and their
documentation rely on, over far more shapes than the GPU tests run.  A unit
covers (layer, head) rows [g * rpu, min(L * H, (g + 1) * rpu)) of one cache
block, row = layer * H + head:

  * the row ranges of a block's units partition [0, L * H), none empty;
  * without row units (the generic copy loop) every range is whole layers;
  * a batch whose one-layer units fit in two waves gets at most one wave of
    units (latency: no CTA runs a second unit), one unit per block when the
    blocks alone outnumber the grid;
  * a large batch gets units of whole layers, at least 16 rows and two
    layers whenever the model has them, with or without row units;
  * the unit count fits the kernels' 32-bit counters.
"""
from __future__ import annotations

import itertools

UNITS_PER_CTA, MIN_ROWS, ROWS_LARGE, UNITS_PER_CTA_MIN = 256, 16, 32, 32


def unit_size(total_blocks: int, L: int, H: int, grid: int, row_units: bool = False):
    LH = L * H
    upb = 1
    if total_blocks > 0 and total_blocks * L <= 2 * grid:
        fit = max(1, grid // total_blocks)
        if row_units:
            upb = min(LH, fit)
            rpu = (LH + upb - 1) // upb
            return rpu, (LH + rpu - 1) // rpu
        upb = min(L, fit)
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
    return lpu * H, upb


def test_unit_sizing_invariants():
    grids = (296, 444, 148)
    layers = (1, 2, 3, 5, 12, 16, 28, 32, 40, 61, 80)
    heads = (1, 2, 3, 4, 8, 16)
    blocks = (1, 2, 5, 9, 10, 13, 37, 100, 147, 148, 296, 297, 592, 1000, 4625, 12_600, 65_536,
              1 << 20)
    for grid, L, H, tb, rows in itertools.product(grids, layers, heads, blocks, (False, True)):
        LH = L * H
        rpu, upb = unit_size(tb, L, H, grid, rows)
        assert 1 <= rpu <= LH and 1 <= upb <= LH
        ranges = [(g * rpu, min(LH, (g + 1) * rpu)) for g in range(upb)]
        assert all(a < b for a, b in ranges), (grid, L, H, tb, rpu, upb)
        assert ranges[0][0] == 0 and ranges[-1][1] == LH
        assert all(ranges[i][1] == ranges[i + 1][0] for i in range(upb - 1))
        if not rows:
            assert all(a % H == 0 and (b % H == 0) for a, b in ranges), "whole layers"
        if tb * L <= 2 * grid:
            assert tb * upb <= max(grid, tb), "one-wave batch: at most one unit per CTA"
            # and not needlessly large: ranges one row (layer) shorter would
            # overflow the grid, or the units are single rows (layers)
            n, q = (LH, rpu) if rows else (L, rpu // H)
            assert q == 1 or tb * -(-n // (q - 1)) > grid
        else:
            assert rpu % H == 0, "large batches: whole layers"
            assert rpu // H >= min(L, 2)
            assert rpu >= min(MIN_ROWS, LH) or rpu == LH
            assert unit_size(tb, L, H, grid, not rows) == (rpu, upb)
        assert tb * upb < 2 ** 31


def test_unit_sizing_at_the_benchmark_shapes():
    # Llama-3.1-8B batch: ~12.6k touched blocks, 32 layers, 8 heads -> units of 6 layers
    assert unit_size(12_633, 32, 8, 296, True) == (48, 6)
    # Qwen2.5-7B, R=100 k=20: ~4.6k blocks, 4 heads -> 10-layer units (32-row rule)
    assert unit_size(4_625, 28, 4, 296, True) == (40, 3)
    # one Llama request of 10 blocks: one wave; whole layers give 160 units of
    # two layers, row units 290 units of 9 rows
    assert unit_size(10, 32, 8, 296) == (16, 16)
    assert unit_size(10, 32, 8, 296, True) == (9, 29)
    # 15 blocks (a request of ~240 tokens): 285 units of 14 rows, not 300 of
    # 13 (four CTAs would run a second unit)
    assert unit_size(15, 32, 8, 296, True) == (14, 19)
    assert unit_size(13, 28, 4, 296, True) == (6, 19)
