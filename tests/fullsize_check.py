"""Full-size parity checker shared by the full-size GPU tests (oracle and
generator only on the reference side): slot mapping of every token, V of
every row (bit-exact, on the device), K of one whole request plus 20 000
random rows (tolerance, against the oracle's fp64 rotation of the regenerated
stored key), and every untouched cache element (bit-exact against the
regenerated pre-fill)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth
from gpu_common import CACHE_FILL_SEED, batch_tensors, make_cache, to_bits

REL, ABS = 2.0 ** -8, 1e-3


def _lengths_store(wl):
    """Oracle store with the workload's lengths (content unused by segment)."""
    st = oracle.Store(1, 1, 2, int(wl.fact_lens.sum()), len(wl.fact_lens))
    for n in wl.fact_lens:
        z = np.zeros((1, 1, int(n), 2), np.uint16)
        st.put(z, z)
    return st


def check_full_size(wl, store, head_major=False, whole_request=37):
    """Inject wl's batch through store (its facts put in id order) into a
    fresh seeded cache and check the result; K of request whole_request (or
    the last one) is checked in full."""
    m, b = wl.model, wl.batch
    k, v, desc = make_cache(wl, head_major=head_major)
    ro, ids, sp, bt = batch_tensors(b)
    n_tok = wl.tokens()
    slots = torch.empty(n_tok, dtype=torch.int64, device="cuda")
    store.inject(ro, ids, sp, bt, desc, slots)
    assert store.last_error()[0] == 0

    seg, st = oracle.segment(_lengths_store(wl), b.req_offsets, b.fact_ids, b.start_pos,
                             b.block_tables, b.block_size, b.num_blocks)
    assert st == oracle.OK and len(seg["slot"]) == n_tok
    got_slots = slots.cpu().numpy()
    assert np.array_equal(got_slots, seg["slot"])
    for f in (0, 4321, len(wl.fact_lens) - 1):  # same put order, same offsets
        assert store.fact_info(f)[0] == int(np.concatenate([[0], np.cumsum(wl.fact_lens)])[f])

    L, H, D, NB, Bs = m.num_layers, m.num_kv_heads, m.head_dim, b.num_blocks, b.block_size
    shape5 = (L, NB, H, Bs, D) if head_major else (L, NB, Bs, H, D)
    k5, v5 = k.view(shape5), v.view(shape5)

    def slot_rows(t5, blk, o):  # rows of the given slots, all layers and heads: [L][n][H][D]
        return t5[:, blk, :, o].permute(1, 0, 2, 3) if head_major else t5[:, blk, o]

    def layer_by_slot(t4):  # one layer as [NB][Bs][H][D] (a view)
        return t4.permute(0, 2, 1, 3) if head_major else t4

    ka, va = store.arena()
    slot_d = torch.from_numpy(seg["slot"]).cuda()
    src_d = torch.from_numpy(seg["src"]).cuda()
    for a in range(0, n_tok, 8192):
        s_, t_ = slot_d[a:a + 8192], src_d[a:a + 8192]
        got_v = slot_rows(v5, s_ // Bs, s_ % Bs)
        assert torch.equal(got_v, va[:, :, t_].permute(0, 2, 1, 3)), f"V rows at {a}"

    # K: one whole request plus random rows
    f = oracle.rope_inv_freq(D, m.rope_theta, m.scaling())
    tok_fact = np.repeat(b.fact_ids, wl.fact_lens[b.fact_ids])
    tok_t = np.concatenate([np.arange(n) for n in wl.fact_lens[b.fact_ids]])
    rng = np.random.default_rng(1)
    rq = min(whole_request, b.num_requests - 1)
    r0 = int(np.searchsorted(seg["request"], rq))
    r1 = int(np.searchsorted(seg["request"], rq + 1))
    toks = np.concatenate([np.repeat(np.arange(r0, r1), L * H), rng.integers(0, n_tok, 20000)])
    ls = np.concatenate([np.tile(np.repeat(np.arange(L), H), r1 - r0), rng.integers(0, L, 20000)])
    hs = np.concatenate([np.tile(np.tile(np.arange(H), L), r1 - r0), rng.integers(0, H, 20000)])
    sl = slot_d[torch.from_numpy(toks).cuda()]
    l_d, h_d = torch.from_numpy(ls).cuda(), torch.from_numpy(hs).cuda()
    got = to_bits(k5[l_d, sl // Bs, h_d, sl % Bs] if head_major else k5[l_d, sl // Bs, sl % Bs, h_d])
    for fid in np.unique(tok_fact[toks]):
        sel = tok_fact[toks] == fid
        x = synth.fact_rows(wl.seed, int(fid), False, L, H, int(wl.fact_lens[fid]), D,
                            ls[sel], hs[sel], tok_t[toks[sel]])
        ref = oracle.rope_rows(oracle.bf16_to_f64(x), seg["pos"][toks[sel]], f)
        err = np.abs(oracle.bf16_to_f64(got[sel]) - ref)
        assert np.all(err <= REL * np.abs(ref) + ABS), f"K rows of fact {fid}"

    # untouched slots keep the seeded pre-fill
    touched = torch.zeros(NB * Bs, dtype=torch.bool, device="cuda")
    touched[slot_d] = True
    untouched = (~touched).view(NB, Bs)
    per_layer = NB * Bs * H * D
    buf = torch.empty(per_layer, dtype=torch.int16, device="cuda")
    cs = torch.cuda.current_stream().cuda_stream
    for t5, tag in ((k5, 0), (v5, 1)):
        for l in range(L):
            synth.fill_device(buf.data_ptr(), per_layer, CACHE_FILL_SEED, synth.TAG_CACHE | tag,
                              l * per_layer, cs)
            want = layer_by_slot(buf.view(shape5[1:]))[untouched]
            have = layer_by_slot(t5[l].view(torch.int16))[untouched]
            assert torch.equal(have, want), f"untouched slots changed (tensor {tag}, layer {l})"
    del k, v, k5, v5
    torch.cuda.empty_cache()
