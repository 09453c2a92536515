"""Pins of the oracle's per-layer operations against brute force, closed forms
and invariants (no GPU)."""
import math

import numpy as np
import pytest

from oracle import layers as L
from oracle.model import Oracle
from synth import ModelConfig, make_weights

from . import bruteforce as bf
from .helpers import oracle_weights

TOY = ModelConfig(n_layers=1, d_model=8, n_q_heads=2, n_kv_heads=1, head_dim=4, n_experts=4,
                  top_k=2, ffn_expert=6, ffn_shared=5, vocab=16, canvas=7)


def _rng(s=0):
    return np.random.default_rng(s)


# ---- RMSNorm -------------------------------------------------------------------------
def test_rms_norm_unit_rms_and_gain():
    x = _rng().normal(size=(5, 16)) * 3.0
    y = L.rms_norm(x, np.ones(16), 0.0)
    np.testing.assert_allclose(np.sqrt((y ** 2).mean(-1)), 1.0, rtol=1e-12)
    g = _rng(1).normal(size=16)
    np.testing.assert_allclose(L.rms_norm(x, g, 0.0), y * g, rtol=1e-12)
    # eps enters under the root
    x1 = np.full((1, 4), 1e-3)
    np.testing.assert_allclose(L.rms_norm(x1, np.ones(4), 1e-6), x1 / math.sqrt(1e-6 + 1e-6))


# ---- RoPE ----------------------------------------------------------------------------
def test_rope_identity_at_zero_and_norm_preserving():
    x = _rng().normal(size=(6, 3, 8))
    np.testing.assert_allclose(L.rope(x, np.zeros(6), 1e4), x, atol=0)
    y = L.rope(x, np.arange(6) * 37, 1e4)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)


def test_rope_is_complex_rotation():
    """Pair (i, i+D/2) as a complex number is multiplied by exp(1j * pos * theta^(-2i/D))."""
    D = 8
    x = _rng(2).normal(size=(4, 1, D))
    pos = np.array([0, 1, 5, 1000])
    y = L.rope(x, pos, 1e4)
    for t in range(4):
        for i in range(D // 2):
            z = complex(x[t, 0, i], x[t, 0, i + D // 2]) * np.exp(1j * pos[t] * 1e4 ** (-2 * i / D))
            assert abs(y[t, 0, i] - z.real) < 1e-12 and abs(y[t, 0, i + D // 2] - z.imag) < 1e-12


def test_rope_relative_position():
    q = _rng(3).normal(size=(1, 1, 16))
    k = _rng(4).normal(size=(1, 1, 16))
    base = (L.rope(q, np.array([7]), 1e4) * L.rope(k, np.array([3]), 1e4)).sum()
    shifted = (L.rope(q, np.array([7 + 1234]), 1e4) * L.rope(k, np.array([3 + 1234]), 1e4)).sum()
    assert abs(base - shifted) < 1e-9


# ---- attention -----------------------------------------------------------------------
def test_attention_matches_loops():
    rng = _rng(5)
    T, Hq, Hkv, D, S = 7, 4, 2, 8, 12
    q = rng.normal(size=(T, Hq, D))
    K = rng.normal(size=(Hkv, S, D))
    V = rng.normal(size=(Hkv, S, D))
    got = L.attention(q, K, V)
    for t in range(T):
        for h in range(Hq):
            g = h * Hkv // Hq
            sc = [sum(q[t, h, d] * K[g, s, d] for d in range(D)) / math.sqrt(D) for s in range(S)]
            m = max(sc)
            e = [math.exp(v - m) for v in sc]
            Z = sum(e)
            for d in range(D):
                ref = sum(e[s] / Z * V[g, s, d] for s in range(S))
                assert abs(got[t, h, d] - ref) < 1e-12


def test_attention_closed_forms():
    rng = _rng(6)
    D, S = 8, 9
    q = rng.normal(size=(3, 2, D))
    Kc = np.tile(rng.normal(size=(1, 1, D)), (1, S, 1))          # all keys equal
    V = rng.normal(size=(1, S, D))
    out = L.attention(q, Kc, V)
    np.testing.assert_allclose(out, np.broadcast_to(V[0].mean(0), out.shape), rtol=1e-12)
    # one key with an overwhelming score returns its value row
    K = rng.normal(size=(1, S, D)) * 0.01
    K[0, 4] = q[0, 0] * 1e4
    out = L.attention(q[:1, :1], K, V)
    np.testing.assert_allclose(out[0, 0], V[0, 4], rtol=1e-9)


# ---- router and experts --------------------------------------------------------------
def test_route_ties_and_renormalisation():
    r = np.array([[1.0, 3.0, 3.0, 0.5, 3.0]])
    idx, w = L.route(r, 2)
    assert idx.tolist() == [[1, 2]]                       # three-way tie -> lowest ids
    np.testing.assert_allclose(w, [[0.5, 0.5]])
    r = _rng(7).normal(size=(20, 16))
    idx, w = L.route(r, 4)
    np.testing.assert_allclose(w.sum(-1), 1.0)
    p = np.exp(r) / np.exp(r).sum(-1, keepdims=True)
    for t in range(20):
        top = sorted(range(16), key=lambda e: -p[t, e])[:4]
        assert idx[t].tolist() == top
        np.testing.assert_allclose(w[t], p[t, top] / p[t, top].sum(), rtol=1e-12)


def _expert_weights(rng, E, f, d):
    return rng.normal(size=(E, f, d)) * 0.3, rng.normal(size=(E, f, d)) * 0.3, rng.normal(size=(E, d, f)) * 0.3


def test_routed_experts_bruteforce():
    rng = _rng(8)
    T, d, E, f, k = 9, 6, 5, 7, 2
    u = rng.normal(size=(T, d))
    Wg, Wu, Wd = _expert_weights(rng, E, f, d)
    r = rng.normal(size=(T, E))
    idx, w = L.route(r, k)
    got = L.routed_experts(u, idx, w, Wg, Wu, Wd)
    # every expert on every token, then keep the top-k by probability
    allout = np.stack([L.swiglu(u, Wg[e], Wu[e], Wd[e]) for e in range(E)], 1)   # [T, E, d]
    p = np.exp(r) / np.exp(r).sum(-1, keepdims=True)
    for t in range(T):
        top = np.argsort(-p[t])[:k]
        ref = (p[t, top, None] * allout[t, top]).sum(0) / p[t, top].sum()
        np.testing.assert_allclose(got[t], ref, rtol=1e-11, atol=1e-12)


def test_identical_experts_equal_dense_ffn():
    rng = _rng(9)
    T, d, E, f, k = 11, 6, 8, 5, 3
    u = rng.normal(size=(T, d))
    wg, wu, wd = rng.normal(size=(f, d)), rng.normal(size=(f, d)), rng.normal(size=(d, f))
    Wg, Wu, Wd = np.stack([wg] * E), np.stack([wu] * E), np.stack([wd] * E)
    idx, w = L.route(rng.normal(size=(T, E)), k)
    np.testing.assert_allclose(L.routed_experts(u, idx, w, Wg, Wu, Wd), L.swiglu(u, wg, wu, wd),
                               rtol=1e-11, atol=1e-12)


def test_all_experts_is_softmax_mixture():
    rng = _rng(10)
    T, d, E, f = 5, 4, 6, 3
    u = rng.normal(size=(T, d))
    Wg, Wu, Wd = _expert_weights(rng, E, f, d)
    r = rng.normal(size=(T, E))
    idx, w = L.route(r, E)
    p = np.exp(r) / np.exp(r).sum(-1, keepdims=True)
    ref = sum(p[:, e:e + 1] * L.swiglu(u, Wg[e], Wu[e], Wd[e]) for e in range(E))
    np.testing.assert_allclose(L.routed_experts(u, idx, w, Wg, Wu, Wd), ref, rtol=1e-11, atol=1e-12)


def test_histogram_permutation():
    idx = np.array([[2, 0], [0, 1], [2, 1], [3, 2]])
    counts, offsets, perm, inv = L.histogram_and_permutation(idx, 5)
    assert counts.tolist() == [2, 2, 3, 1, 0]
    assert offsets.tolist() == [0, 2, 4, 7, 8, 8]
    # expert 0: (t0,j1),(t1,j0); expert 1: (t1,j1),(t2,j1); expert 2: (t0,j0),(t2,j0),(t3,j1); expert 3: (t3,j0)
    assert perm.tolist() == [1, 2, 3, 5, 0, 4, 7, 6]
    for t in range(4):
        for j in range(2):
            assert perm[inv[t, j]] == t * 2 + j


# ---- LM-head statistics --------------------------------------------------------------
def test_lm_stats_uniform_and_one_hot():
    V, d = 64, 4
    E = np.zeros((V, d))
    st = L.lm_head_stats(np.ones((2, d)), E)
    np.testing.assert_allclose(st["entropy"], math.log(V), rtol=1e-14)
    np.testing.assert_allclose(st["logconf"], -math.log(V), rtol=1e-14)
    assert st["argmax"].tolist() == [0, 0]                 # all tied -> lowest id
    E[37, 0] = 50.0
    st = L.lm_head_stats(np.array([[1.0, 0, 0, 0]]), E)
    assert st["argmax"][0] == 37
    # 63 rivals at margin 50: H ~ 63 * 51 * e^-50 ~ 6e-19, logconf ~ -63 e^-50
    assert 0.0 <= st["entropy"][0] < 1e-17
    assert -1e-18 < st["logconf"][0] <= 0.0


def test_lm_stats_bruteforce():
    rng = _rng(11)
    xn = rng.normal(size=(3, 5))
    E = rng.normal(size=(40, 5))
    st = L.lm_head_stats(xn, E)
    for t in range(3):
        ref = bf.lm_stats(xn[t].tolist(), E.tolist())
        assert st["argmax"][t] == ref["argmax"]
        for key in ("max", "logZ", "entropy", "logconf"):
            assert abs(st[key][t] - ref[key]) < 1e-12


def test_online_merge_of_partials_equals_direct():
    """The per-chunk (max, argmax, sum e^(z-m), sum e^(z-m)(z-m)) merge, in fp64,
    reproduces the direct statistics: the algebra a split LM head relies on."""
    rng = _rng(12)
    z = rng.normal(size=(4, 1000)) * 3.0
    z[2, 123] = z[2, 877] = 40.0                     # exact tie across chunks
    chunks = [z[:, i:i + 96] for i in range(0, 1000, 96)]
    m = np.full(4, -np.inf)
    s = np.zeros(4)
    t = np.zeros(4)
    a = np.zeros(4, dtype=np.int64)
    base = 0
    for ch in chunks:
        mc = ch.max(-1)
        ac = ch.argmax(-1) + base
        sc = np.exp(ch - mc[:, None]).sum(-1)
        tc = (np.exp(ch - mc[:, None]) * (ch - mc[:, None])).sum(-1)
        mn = np.maximum(m, mc)
        f0 = np.where(np.isfinite(m), np.exp(m - mn), 0.0)
        f1 = np.exp(mc - mn)
        t = f0 * (t + np.where(np.isfinite(m), m - mn, 0.0) * s) + f1 * (tc + (mc - mn) * sc)
        s = f0 * s + f1 * sc
        a = np.where(mc > m, ac, a)
        m = mn
        base += ch.shape[1]
    st = L.lm_head_stats(np.eye(4), np.ascontiguousarray(z.T))
    np.testing.assert_allclose(m + np.log(s), st["logZ"], rtol=1e-13)
    np.testing.assert_allclose(np.log(s) - t / s, st["entropy"], rtol=1e-11)
    np.testing.assert_allclose(-np.log(s), st["logconf"], rtol=1e-11, atol=1e-13)
    assert a.tolist() == st["argmax"].tolist() and a[2] == 123


# ---- one full layer against the scalar brute force -------------------------------------
@pytest.mark.parametrize("use_rope", [True, False])
def test_layer_bruteforce(use_rope):
    cfg = TOY
    w = oracle_weights(make_weights(cfg, seed=3, std=0.3, gain_std=0.2))
    ora = Oracle(cfg, w)
    ora.use_rope = use_rope
    rng = _rng(13)
    Lc, T = 3, 5
    cache = ora.new_cache(Lc + T)
    Kc = rng.normal(size=(cfg.n_kv_heads, Lc, cfg.head_dim))
    Vc = rng.normal(size=(cfg.n_kv_heads, Lc, cfg.head_dim))
    cache.K[0][:, :Lc] = Kc
    cache.V[0][:, :Lc] = Vc
    cache.length = Lc
    toks = rng.integers(0, cfg.vocab, size=T)
    from oracle.model import Trace
    tr = Trace()
    st = ora.forward(toks, cache, trace=tr)
    xs = [w["embed"][t].tolist() for t in toks]
    out, k_rows, v_rows = bf.layer(xs, [Lc + i for i in range(T)], Kc.tolist(), Vc.tolist(),
                                   {k: v.tolist() for k, v in w["layers"][0].items()}, cfg, use_rope)
    np.testing.assert_allclose(tr.layers[0]["x_out"], np.array(out), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(cache.K[0][:, Lc:Lc + T].transpose(1, 0, 2), np.array(k_rows), atol=1e-12)
    np.testing.assert_allclose(cache.V[0][:, Lc:Lc + T].transpose(1, 0, 2), np.array(v_rows), atol=1e-12)
    xn = L.rms_norm(np.array(out), w["final_norm"], cfg.norm_eps)
    for t in range(T):
        ref = bf.lm_stats(xn[t].tolist(), w["embed"].tolist())
        assert st["argmax"][t] == ref["argmax"]
        assert abs(st["entropy"][t] - ref["entropy"]) < 1e-10
        assert abs(st["logconf"][t] - ref["logconf"]) < 1e-10


# ---- self-conditioning -----------------------------------------------------------------------

def test_topk_probs_bruteforce_with_ties():
    rng = _rng(30)
    for _ in range(200):
        z = rng.choice([-1.0, 0.0, 0.5, 2.0, 2.0, 3.0], size=(1, 12))
        k = int(rng.integers(1, 9))
        p, ids = L.topk_probs(z, k)
        ref = sorted(range(12), key=lambda i: (-z[0, i], i))[:k]      # value descending, lower id first
        assert ids[0].tolist() == ref
        full = np.exp(z[0]) / np.exp(z[0]).sum()
        np.testing.assert_allclose(p[0], full[ref], rtol=1e-14)


def test_soft_embedding_closed_forms():
    rng = _rng(31)
    V, d = 10, 6
    E = rng.normal(size=(V, d))
    z = rng.normal(size=(3, V))
    # k = V: the full expectation of the embedding under softmax(z)
    p, ids = L.topk_probs(z, V)
    sm = np.exp(z) / np.exp(z).sum(axis=1, keepdims=True)
    np.testing.assert_allclose(L.soft_embedding(p, ids, E), sm @ E, rtol=1e-12)
    # a dominant logit: the embedding of that id
    zd = np.zeros((1, V))
    zd[0, 7] = 60.0
    p, ids = L.topk_probs(zd, 3)
    np.testing.assert_allclose(L.soft_embedding(p, ids, E)[0], E[7], atol=1e-20)
    # two equal dominant logits: half of each (k = 2), half of the lower id alone (k = 1)
    zt = np.zeros((1, V))
    zt[0, [2, 5]] = 60.0
    p, ids = L.topk_probs(zt, 2)
    np.testing.assert_allclose(L.soft_embedding(p, ids, E)[0], 0.5 * (E[2] + E[5]), rtol=1e-12)
    p, ids = L.topk_probs(zt, 1)
    np.testing.assert_allclose(L.soft_embedding(p, ids, E)[0], 0.5 * E[2], rtol=1e-12)


def test_self_condition_invariances():
    rng = _rng(32)
    V, d, f, k = 16, 8, 12, 4
    E = rng.normal(size=(V, d))
    wg, wu, wd = rng.normal(size=(f, d)), rng.normal(size=(f, d)), rng.normal(size=(d, f))
    z = rng.normal(size=(5, V))
    out = L.self_condition(z, E, wg, wu, wd, k)
    # a constant added to a row's logits changes nothing (softmax shift invariance)
    np.testing.assert_allclose(L.self_condition(z + 3.7, E, wg, wu, wd, k), out, rtol=1e-10)
    # relabelling the vocabulary (logits and embedding rows together) changes nothing
    perm = rng.permutation(V)
    np.testing.assert_allclose(L.self_condition(z[:, perm], E[perm], wg, wu, wd, k), out, rtol=1e-10)
    # with a dominant logit the term is the gated MLP of that token's embedding
    zd = np.full((1, V), -50.0)
    zd[0, 11] = 50.0
    np.testing.assert_allclose(L.self_condition(zd, E, wg, wu, wd, k)[0], L.swiglu(E[11:12], wg, wu, wd)[0],
                               rtol=1e-12)
    # a zero-mass input gives a zero term (no biases)
    np.testing.assert_array_equal(L.swiglu(np.zeros((1, d)), wg, wu, wd), np.zeros((1, d)))


def test_self_conditioning_enters_only_after_the_first_step():
    cfg = TOY.with_(ffn_selfcond=8, selfcond_topk=3)
    w = oracle_weights(make_weights(cfg, seed=3))
    ora = Oracle(cfg, w)
    toks = np.arange(cfg.canvas) % cfg.vocab
    c1 = ora.new_cache(32)
    c2 = ora.new_cache(32)
    st_plain = ora.forward(toks, c1)
    st_none = ora.forward(toks, c2, sc=ora.self_condition(None))
    np.testing.assert_array_equal(st_plain["logits"], st_none["logits"])
    sc = ora.self_condition(st_plain["logits"])
    assert sc.shape == (cfg.canvas, cfg.d_model) and np.abs(sc).max() > 0
    from oracle.model import Trace
    tr = Trace()
    st_sc = ora.forward(toks, ora.new_cache(32), sc=sc, trace=tr)
    # the term is added to the token embeddings at the first layer's input
    np.testing.assert_array_equal(tr.layers[0]["x_in"], w["embed"][toks] + sc)
    assert np.abs(st_sc["logits"] - st_plain["logits"]).max() > 1e-12
