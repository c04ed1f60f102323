"""The pins must catch plausible mistakes planted in the oracle.

Each case compiles a copy of oracle/inject_oracle.c with one edit (a flipped
sign, a wrong pair index, a dropped factor, an off-by-one position, a wrong
slot, truncation instead of rounding, V taken from K, a misplaced offset),
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
