"""Writes tests/golden/tiny_inject.json from the CPU oracle alone.

Inputs come from the seeded generator (synth); every expected value is the
oracle's.  Run from the repository root:  python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

SEED, FILL_SEED = 0, 7


def case(start_pos):
    wl = synth.tiny(SEED, start_pos=start_pos)
    m, b = wl.model, wl.batch
    st = oracle.Store(m.num_layers, m.num_kv_heads, m.head_dim, int(wl.fact_lens.sum()),
                      len(wl.fact_lens))
    for f, n in enumerate(wl.fact_lens):
        st.put(*synth.fact_kv(SEED, f, m.num_layers, m.num_kv_heads, int(n), m.head_dim))
    shape = (m.num_layers, b.num_blocks, b.block_size, m.num_kv_heads, m.head_dim)
    kc = synth.bf16_block(FILL_SEED, synth.TAG_CACHE | 0, shape)
    vc = synth.bf16_block(FILL_SEED, synth.TAG_CACHE | 1, shape)
    rc, slots = oracle.inject_batch(st, oracle.rope_inv_freq(m.head_dim, m.rope_theta),
                                    b.req_offsets, b.fact_ids, b.start_pos, b.block_tables,
                                    kc, vc, b.block_size)
    return dict(start_pos=start_pos, status=rc, slot_mapping=[int(s) for s in slots],
                k_cache_sha256=hashlib.sha256(kc.tobytes()).hexdigest(),
                v_cache_sha256=hashlib.sha256(vc.tobytes()).hexdigest())


def main():
    out = dict(description="oracle output on the tiny workload (1 layer, 2 KV heads, D=64, "
                           "theta 1e4, 64 facts of 8-24 tokens, k=5, block size 16, 64 blocks)",
               seed=SEED, cache_fill_seed=FILL_SEED, cases=[case(s) for s in (32, 37, 0)])
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_inject.json")
    cases = out.pop("cases")
    with open(path, "w") as fh:
        body = json.dumps(out, indent=1)[:-2]
        fh.write(body + ',\n "cases": [\n')
        fh.write(",\n".join("  " + json.dumps(c) for c in cases))
        fh.write("\n ]\n}\n")


if __name__ == "__main__":
    main()
