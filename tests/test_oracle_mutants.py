"""The pins must catch plausible mistakes planted in the oracle.

Each case compiles a copy of oracle/inject_oracle.c with one edit (a flipped
sign, a wrong pair index, a dropped factor, positions off by one, without the
start or restarting per fact, a wrong slot, truncation or ties away from zero
instead of round-to-even, V taken from K, K left unrotated, a misplaced
offset, swapped cache strides, a bad id skipped, the wrong llama3 band),
points ORACLE_LIB at it and runs the pin suite in a fresh process, which must
fail.  CPU only; the real oracle is untouched.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "inject_oracle.c")

MUTANTS = {
    "sin_sign": ("out[a] = x[a] * c - x[b] * s;", "out[a] = x[a] * c + x[b] * s;"),
    "pair_index": ("*b = i + D / 2; }", "*b = D - 1 - i; }"),
    "freq_exponent": ("pow(theta, -(2.0 * i) / (double)D)", "pow(theta, -(1.0 * i) / (double)D)"),
    "llama3_blend_swapped": ("(1.0 - smooth) * f / factor + smooth * f",
                             "smooth * f / factor + (1.0 - smooth) * f"),
    "position_off_by_one": ("int64_t pos = (int64_t)start[r] + i;",
                            "int64_t pos = (int64_t)start[r] + i + 1;"),
    "slot_offset": ("return (int64_t)blk * B + pos % B;", "return (int64_t)blk * B + (pos + 1) % B;"),
    "truncating_bf16": ("double n = nearbyint(a / spacing);", "double n = floor(a / spacing);"),
    "v_from_k": ("c->v[dst + d] = s->v[src + d];", "c->v[dst + d] = s->k[src + d];"),
    "store_offset": ("s->off[id] = off;", "s->off[id] = off + 1;"),
    # positions that ignore the request's start, or restart at every fact
    "start_ignored": ("int64_t pos = (int64_t)start[r] + i;", "int64_t pos = i;"),
    "position_restarts_per_fact": ("int64_t pos = (int64_t)start[r] + i;",
                                   "int64_t pos = (int64_t)start[r] + t;"),
    # a bad fact id skipped instead of invalidating its request
    "bad_id_ignored": ("if (f < 0 || f >= s->num_facts) { st = ORC_ERR_BAD_FACT_ID; continue; }",
                       "if (f < 0 || f >= s->num_facts) { continue; }"),
    # the Llama-3.1 rule scaling the high frequencies it must keep
    "llama3_high_band_scaled": ("if (lam < high_wl) return f;", "if (lam < high_wl) return f / factor;"),
    # ties rounded away from zero instead of to even
    "bf16_ties_away": ("double n = nearbyint(a / spacing);", "double n = round(a / spacing);"),
    # the head and token strides of the cache swapped
    "cache_strides_swapped": ("o * c->token_stride +\n                            h * c->head_stride;",
                              "o * c->head_stride +\n                            h * c->token_stride;"),
    # the block-table bound off by one (reads one entry past the row)
    "table_bound_off_by_one": ("if (pos < 0 || pos / B >= max_blocks) return -1;",
                               "if (pos < 0 || pos / B > max_blocks) return -1;"),
    # a blend weight that is monotone and exact at both band edges but not
    # linear in orig / wavelength
    "llama3_blend_squared": ("double smooth = (orig / lam - low) / (high - low);",
                             "double smooth = (orig / lam - low) / (high - low);\n  smooth = smooth * smooth;"),
    # a NaN rounded to an infinity
    "nan_to_inf": ("if (isnan(x)) return 0x7FC0;", "if (isnan(x)) return 0x7F80;"),
    # the rotation pair taken from the interleaved layout under rotate-half
    "pair_style_swapped": ("if (style == 0) { *a = i; *b = i + D / 2; }",
                           "if (style != 0) { *a = i; *b = i + D / 2; }"),
    # K left unrotated
    "k_not_rotated": ("c->k[dst + d] = orc_f64_to_bf16(y[d]);", "c->k[dst + d] = orc_f64_to_bf16(x[d]);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mpath = tmp_path / "mutant.c"
    mpath.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", str(lib), str(mpath), "-lm"],
                   check=True)
    env = dict(os.environ, ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
