"""Theorem 3 on a tiny random multi-layer decoder: when does injecting
precomputed KV equal prefill?

Passages (summaries of "InferScale: GPU-Native KV Injection for Personalized
LLM Serving", technical summary): Contributions, "Retrieve-and-inject
inference" (Theorem 3: injecting precomputed KV is exactly prompt injection
for causal decoders when the memory sits at the intended positions);
Online phase, "Theoretical guarantee" (Theorem 6: re-rotation is exact);
Offline phase, context-window encoding (each fact encoded with w preceding
turns, only the fact's KV kept).

The model (test-only, numpy fp64): L layers of pre-norm attention with GQA
and RoPE (rotations by the oracle) plus an MLP, random weights.  Facts are
encoded offline with pre-RoPE keys captured at every layer, stored, then
injected at serving positions; the query is prefilled alone against
[prefix KV | injected KV].  Findings, asserted below:

  * w = 0 (each fact encoded alone, at any offset): equality (to fp64
    rounding) with a full prefill of [prefix | facts | query] whose fact
    tokens attend only within their own fact;
  * a window covering everything before the fact (encoded at any offset):
    equality with the ordinary causal prefill, i.e. prompt injection;
  * w = 0 against the ordinary causal prefill: layer 0 still agrees exactly
    (its K/V depend only on the token and its position) but deeper layers
    do not, and neither does the query's output.  A window shorter than the
    whole preceding prompt sits between the two: its own tokens are encoded
    without their context, so beyond layer 0 it is an approximation, which
    is what the pages' accuracy results measure.
So Theorem 3's "intended" KV is the KV of the encoding the store was built
with, and re-rotation (Theorem 6) makes the encoding offset irrelevant.
"""
from __future__ import annotations

import math

import numpy as np
import pytest

import oracle


def _rms(x):
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + 1e-6)


class TinyDecoder:
    def __init__(self, seed=0, L=3, dm=64, nq=4, nkv=2, D=32, ff=128, theta=1e4):
        rng = np.random.default_rng(seed)
        n = lambda *s: rng.standard_normal(s) / math.sqrt(s[0])  # noqa: E731
        self.L, self.dm, self.nq, self.nkv, self.D = L, dm, nq, nkv, D
        self.Wq = [n(dm, nq * D) for _ in range(L)]
        self.Wk = [n(dm, nkv * D) for _ in range(L)]
        self.Wv = [n(dm, nkv * D) for _ in range(L)]
        self.Wo = [n(nq * D, dm) for _ in range(L)]
        self.W1 = [n(dm, ff) for _ in range(L)]
        self.W2 = [n(ff, dm) for _ in range(L)]
        self.inv = oracle.rope_inv_freq(D, theta)

    def rope(self, x, pos):  # x [n, heads, D]
        return oracle.rope_rows(x, np.broadcast_to(np.asarray(pos)[:, None], x.shape[:2]), self.inv)

    def run(self, x, pos, allowed, past=None):
        """New tokens x [n, dm] at positions pos attend to [past | new] where
        allowed [n, m + n] is True.  past: per layer (K_rot, V) [m, nkv, D].
        Returns final states and, per layer, (pre-RoPE K, V, rotated K)."""
        h = x.copy()
        n = len(x)
        g = self.nq // self.nkv
        caps = []
        for l in range(self.L):
            hn = _rms(h)
            q = (hn @ self.Wq[l]).reshape(n, self.nq, self.D)
            k = (hn @ self.Wk[l]).reshape(n, self.nkv, self.D)
            v = (hn @ self.Wv[l]).reshape(n, self.nkv, self.D)
            qr, kr = self.rope(q, pos), self.rope(k, pos)
            K = kr if past is None else np.concatenate([past[l][0], kr])
            V = v if past is None else np.concatenate([past[l][1], v])
            out = np.zeros((n, self.nq, self.D))
            for hq in range(self.nq):
                s = qr[:, hq] @ K[:, hq // g].T / math.sqrt(self.D)
                s = np.where(allowed, s, -np.inf)
                p = np.exp(s - s.max(axis=1, keepdims=True))
                out[:, hq] = (p / p.sum(axis=1, keepdims=True)) @ V[:, hq // g]
            h = h + out.reshape(n, -1) @ self.Wo[l]
            h = h + np.tanh(_rms(h) @ self.W1[l]) @ self.W2[l]
            caps.append((k, v, kr))
        return h, caps


def _setup(seed=1, P=5, lens=(4, 7, 3), Q=3, dm=64):
    rng = np.random.default_rng(seed)
    prefix = rng.standard_normal((P, dm))
    facts = [rng.standard_normal((n, dm)) for n in lens]
    query = rng.standard_normal((Q, dm))
    return prefix, facts, query


def _mask(P, lens, Q, fact_scope):
    """[prefix | facts | query] mask.  fact_scope: 'local' (own fact),
    ('window', w) (own fact + the w tokens just before it), 'causal'."""
    T = P + sum(lens) + Q
    m = np.tril(np.ones((T, T), bool))
    start = P
    for n in lens:
        for i in range(start, start + n):
            if fact_scope == "causal":
                continue
            lo = start if fact_scope == "local" else max(0, start - fact_scope[1])
            m[i, :lo] = False
        start += n
    return m


def _inject_path(model, prefix, facts, query, context=None, offset=0):
    """Offline: encode each fact (after its window context[j], if given) at
    positions offset, offset+1, ..., keep the fact's pre-RoPE K and V per
    layer.  Online: prefix prefill, rotate the stored keys to the serving
    positions, query-only prefill."""
    P, Q = len(prefix), len(query)
    _, pre_caps = model.run(prefix, np.arange(P), np.tril(np.ones((P, P), bool)))
    past = [(c[2], c[1]) for c in pre_caps]
    pos = P
    for j, f in enumerate(facts):
        win = context[j] if context is not None else np.zeros((0, prefix.shape[1]))
        enc = np.concatenate([win, f])
        n = len(enc)
        _, caps = model.run(enc, offset + np.arange(n), np.tril(np.ones((n, n), bool)))
        for l in range(model.L):
            k_pre, v = caps[l][0][len(win):], caps[l][1][len(win):]
            k_rot = model.rope(k_pre, np.arange(pos, pos + len(f)))  # re-rotation
            past[l] = (np.concatenate([past[l][0], k_rot]), np.concatenate([past[l][1], v]))
        pos += len(f)
    m = pos
    allowed = np.concatenate([np.ones((Q, m), bool), np.tril(np.ones((Q, Q), bool))], axis=1)
    out, _ = model.run(query, np.arange(m, m + Q), allowed, past=past)
    return out, past


def _prefill(model, prefix, facts, query, scope):
    x = np.concatenate([prefix] + facts + [query])
    T = len(x)
    out, caps = model.run(x, np.arange(T), _mask(len(prefix), [len(f) for f in facts],
                                                 len(query), scope))
    return out[-len(query):], caps


@pytest.mark.parametrize("offset", [0, 123])
def test_injection_equals_fact_local_prefill(offset):
    model = TinyDecoder()
    prefix, facts, query = _setup()
    got, _ = _inject_path(model, prefix, facts, query, offset=offset)
    want, _ = _prefill(model, prefix, facts, query, "local")
    assert np.allclose(got, want, rtol=0, atol=1e-10 * np.abs(want).max())


@pytest.mark.parametrize("offset", [0, 57])
def test_full_window_encoding_equals_prompt_injection(offset):
    """Each fact encoded after everything that precedes it in the prompt:
    the injected cache and the query output equal the causal prefill."""
    model = TinyDecoder(seed=2)
    prefix, facts, query = _setup(seed=3, lens=(4, 5, 6))
    seq = [prefix] + facts
    context = [np.concatenate(seq[: j + 1]) for j in range(len(facts))]
    got, past = _inject_path(model, prefix, facts, query, context=context, offset=offset)
    want, caps = _prefill(model, prefix, facts, query, "causal")
    assert np.allclose(got, want, rtol=0, atol=1e-10 * np.abs(want).max())
    for l in range(model.L):
        assert np.allclose(past[l][0], caps[l][2][: len(past[l][0])], atol=1e-10)


def test_causal_prompt_injection_differs_beyond_layer_zero():
    model = TinyDecoder(seed=4)
    prefix, facts, query = _setup(seed=5)
    got, past = _inject_path(model, prefix, facts, query)
    want, caps = _prefill(model, prefix, facts, query, "causal")
    P, S = len(prefix), sum(len(f) for f in facts)
    # layer 0: identical K (rotated) and V for the fact tokens
    assert np.allclose(past[0][0][P:P + S], caps[0][2][P:P + S], atol=1e-12)
    assert np.allclose(past[0][1][P:P + S], caps[0][1][P:P + S], atol=1e-12)
    # deeper layers and the query output: not equal
    for l in range(1, model.L):
        assert np.abs(past[l][1][P:P + S] - caps[l][1][P:P + S]).max() > 1e-3
    assert np.abs(got - want).max() > 1e-3 * np.abs(want).max()


@pytest.mark.gpu
def test_gpu_injected_cache_serves_the_query():
    """The same check through the CUDA path: facts' pre-RoPE K/V (bf16) go
    into a FactStore, the GPU injects them into a paged cache, and the query
    is prefilled against that cache.  Agreement with the fact-local fp64
    prefill is at bf16 level, far closer than the causal prompt injection."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_injection_gather_b200 import FactStore, RopeConfig, cache_desc

    model = TinyDecoder(seed=6)
    prefix, facts, query = _setup(seed=7)
    P, Q, L, H, D = len(prefix), len(query), model.L, model.nkv, model.D
    lens = [len(f) for f in facts]
    store = FactStore(L, H, D, RopeConfig(theta=1e4), sum(lens), len(facts))
    to_bf = lambda a: torch.from_numpy(oracle.f64_to_bf16(a).view(np.int16)).view(torch.bfloat16)  # noqa: E731
    for f in facts:
        _, caps = model.run(f, np.arange(len(f)), np.tril(np.ones((len(f), len(f)), bool)))
        k = np.stack([c[0] for c in caps]).transpose(0, 2, 1, 3)  # [L][H][len][D]
        v = np.stack([c[1] for c in caps]).transpose(0, 2, 1, 3)
        store.put_fact(to_bf(np.ascontiguousarray(k)), to_bf(np.ascontiguousarray(v)))
    B, NB = 16, 8
    bt = torch.tensor([[3, 0, 6, 1, 7, 2, 5, 4]], dtype=torch.int32, device="cuda")
    kc = torch.zeros((L, NB, B, H, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    ro = torch.tensor([0, len(facts)], dtype=torch.int32, device="cuda")
    ids = torch.arange(len(facts), dtype=torch.int32, device="cuda")
    sp = torch.tensor([P], dtype=torch.int32, device="cuda")
    store.inject(ro, ids, sp, bt, cache_desc(kc, vc))
    assert store.last_error()[0] == 0
    store.close()
    # read the injected positions back through the block table
    S = sum(lens)
    pos = np.arange(P, P + S)
    slot = bt[0].cpu().numpy()[pos // B] * B + pos % B
    to64 = lambda t: oracle.bf16_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))  # noqa: E731
    kinj = to64(kc.view(L, NB * B, H, D)[:, torch.from_numpy(slot).cuda()])
    vinj = to64(vc.view(L, NB * B, H, D)[:, torch.from_numpy(slot).cuda()])
    _, pre_caps = model.run(prefix, np.arange(P), np.tril(np.ones((P, P), bool)))
    past = [(np.concatenate([pre_caps[l][2], kinj[l]]), np.concatenate([pre_caps[l][1], vinj[l]]))
            for l in range(L)]
    allowed = np.concatenate([np.ones((Q, P + S), bool), np.tril(np.ones((Q, Q), bool))], axis=1)
    got, _ = model.run(query, np.arange(P + S, P + S + Q), allowed, past=past)
    want, _ = _prefill(model, prefix, facts, query, "local")
    causal, _ = _prefill(model, prefix, facts, query, "causal")
    err = np.abs(got - want).max()
    assert err < 3e-2 * np.abs(want).max()
    assert err < 0.1 * np.abs(causal - want).max()


@pytest.mark.gpu
def test_gpu_window_encoding_through_the_store_equals_prompt_injection():
    """Context-window encoding end to end on the CUDA path: each fact is
    encoded after everything before it (at an arbitrary offset), the encoder's
    K/V of [window | fact] go to is_store_put_fact_window (window dropped), the
    GPU injects, the query is prefilled against the cache.  The output equals
    the ordinary causal prefill at bf16 level."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_injection_gather_b200 import FactStore, RopeConfig, cache_desc

    model = TinyDecoder(seed=8)
    prefix, facts, query = _setup(seed=9, lens=(5, 3, 6))
    P, Q, L, H, D = len(prefix), len(query), model.L, model.nkv, model.D
    lens = [len(f) for f in facts]
    seq = [prefix] + facts
    store = FactStore(L, H, D, RopeConfig(theta=1e4), sum(lens), len(facts))
    to_bf = lambda a: torch.from_numpy(oracle.f64_to_bf16(a).view(np.int16)).view(torch.bfloat16)  # noqa: E731
    for j, f in enumerate(facts):
        enc = np.concatenate(seq[: j + 1] + [f])
        n = len(enc)
        _, caps = model.run(enc, 31 + np.arange(n), np.tril(np.ones((n, n), bool)))
        k = np.ascontiguousarray(np.stack([c[0] for c in caps]).transpose(0, 2, 1, 3))
        v = np.ascontiguousarray(np.stack([c[1] for c in caps]).transpose(0, 2, 1, 3))
        kt, vt = to_bf(k), to_bf(v)
        fid = store.put_fact_window(kt.cuda() if j % 2 else kt, vt.cuda() if j % 2 else vt, n - len(f))
        kr, vr = store.read_fact(fid)  # only the fact's rows were kept
        assert torch.equal(kr.cpu(), kt[:, :, n - len(f):]) and torch.equal(vr.cpu(), vt[:, :, n - len(f):])
    B, NB = 16, 4
    bt = torch.tensor([[2, 0, 3, 1]], dtype=torch.int32, device="cuda")
    kc = torch.zeros((L, NB, B, H, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    store.inject(torch.tensor([0, 3], dtype=torch.int32, device="cuda"),
                 torch.arange(3, dtype=torch.int32, device="cuda"),
                 torch.tensor([P], dtype=torch.int32, device="cuda"), bt, cache_desc(kc, vc))
    assert store.last_error()[0] == 0
    store.close()
    S = sum(lens)
    pos = np.arange(P, P + S)
    slot = torch.from_numpy(bt[0].cpu().numpy()[pos // B] * B + pos % B).cuda()
    to64 = lambda t: oracle.bf16_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))  # noqa: E731
    kinj = to64(kc.view(L, NB * B, H, D)[:, slot])
    vinj = to64(vc.view(L, NB * B, H, D)[:, slot])
    _, pre_caps = model.run(prefix, np.arange(P), np.tril(np.ones((P, P), bool)))
    past = [(np.concatenate([pre_caps[l][2], kinj[l]]), np.concatenate([pre_caps[l][1], vinj[l]]))
            for l in range(L)]
    allowed = np.concatenate([np.ones((Q, P + S), bool), np.tril(np.ones((Q, Q), bool))], axis=1)
    got, _ = model.run(query, np.arange(P + S, P + S + Q), allowed, past=past)
    want, _ = _prefill(model, prefix, facts, query, "causal")
    local, _ = _prefill(model, prefix, facts, query, "local")
    err = np.abs(got - want).max()
    assert err < 3e-2 * np.abs(want).max()
    assert err < 0.1 * np.abs(local - want).max()
