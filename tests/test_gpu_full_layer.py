"""GPU vs oracle at the full synthetic shape: one decoder layer (d 2816, 16/8
heads of 256, 128 experts top-8 + shared 2112, vocab 262144) over a 256-token
canvas with a 4096-token synthetic KV prefix, in the same launch configuration
as the benchmark (1 request, 256 canvas tokens)."""
import numpy as np
import pytest
import torch

from oracle import layers as OL
from oracle.model import Oracle, Trace
from oracle import sampler as OS
from synth import LAYER, make_kv_prefix, make_weights, to_f64

from .gpu_common import (LOGIT_MAX_ABS, MAX_EXCLUDED_DIVERGED, REL_L2, argmax_agreement, assert_excluded_fraction,
                         np64, rel_l2, routing_divergence)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

CFG = LAYER
L_PREFIX = 4096


@pytest.fixture(scope="module")
def setup():
    import block_diffusion_moe_denoise_b200 as dgm
    w = make_weights(CFG, seed=0, device="cuda")
    k, v = make_kv_prefix(CFG, L_PREFIX, seed=1, device="cuda")
    h = dgm.DG(CFG, w, max_requests=1, kv_capacity=L_PREFIX + CFG.canvas)
    h.set_kv(0, 0, 0, k, v)
    h.set_kv_len(0, L_PREFIX)
    h.open_canvas(0, 2, 0)
    tok, _, _, _ = h.get_canvas(0)
    h.debug_forward(0, tok, 1)                 # the whole 1-layer pass incl. LM head
    h.sync()
    ow = {"embed": to_f64(w["embed"]), "final_norm": to_f64(w["final_norm"]),
          "layers": [{n: to_f64(t) for n, t in w["layers"][0].items()}]}
    ora = Oracle(CFG, ow)
    cache = ora.new_cache(L_PREFIX + CFG.canvas)
    cache.K[0][:, :L_PREFIX] = to_f64(k)
    cache.V[0][:, :L_PREFIX] = to_f64(v)
    cache.length = L_PREFIX
    tr = Trace()
    ora.forward(tok.cpu().numpy().astype(np.int64), cache, want_stats=False, trace=tr)
    yield dict(h=h, w=w, ora=ora, tr=tr.layers[0], tok=tok, cache=cache)
    h.close()


def test_canvas_init_is_philox(setup):
    ref, _ = OS.init_canvas(CFG.canvas, seed=2, block=0, vocab=CFG.vocab)
    np.testing.assert_array_equal(setup["tok"].cpu().numpy(), ref)


def test_attention_path(setup):
    h, rec = setup["h"], setup["tr"]
    T, d, Hq, D = CFG.canvas, CFG.d_model, CFG.n_q_heads, CFG.head_dim
    Tcap = h.token_capacity()
    q = np64(h.debug_buffer("q", torch.bfloat16, (Hq, Tcap, D))[:, :T]).transpose(1, 0, 2)
    assert rel_l2(q, rec["q"]) < REL_L2
    kk, vv = h.get_kv(0, 0, L_PREFIX, T)
    assert rel_l2(np64(kk).transpose(1, 0, 2), rec["k"]) < REL_L2
    assert rel_l2(np64(vv).transpose(1, 0, 2), rec["v"]) < REL_L2
    o = np64(h.debug_buffer("o", torch.bfloat16, (T, Hq * D)))
    eo = rel_l2(o, rec["o"].reshape(T, Hq * D))
    print(f"full layer: rel-L2 of attention output {eo:.2e}")
    assert eo < REL_L2
    assert rel_l2(np64(h.debug_buffer("u", torch.bfloat16, (T, d))), rec["u"]) < REL_L2


def test_moe_path(setup):
    h, rec, ora = setup["h"], setup["tr"], setup["ora"]
    T, d, k = CFG.canvas, CFG.d_model, CFG.top_k
    idx = h.debug_buffer("idx", torch.int32, (T, k)).cpu().numpy()
    # every token whose GPU routing differs from the oracle's must be a near-tie
    same = routing_divergence([idx], [rec["router_logits"]], [rec["idx"]], k) == 1
    assert_excluded_fraction(~same, MAX_EXCLUDED_DIVERGED, "full layer, routed differently at a near-tie")
    counts = h.debug_buffer("counts", torch.int32, (CFG.n_experts,)).cpu().numpy()
    assert counts.sum() == T * k and (counts == np.bincount(idx.ravel(), minlength=CFG.n_experts)).all()
    pair_row = h.debug_buffer("pair_row", torch.int32, (T * k,)).cpu().numpy()
    yp = np64(h.debug_buffer("yp", torch.bfloat16, (T * k, d)))
    W = ora.layer(0)
    rng = np.random.default_rng(0)
    got, ref = [], []
    for t in rng.choice(np.nonzero(same)[0], 24, replace=False):
        for j in range(k):
            e = idx[t, j]
            jj = list(rec["idx"][t]).index(e)
            hid = OL.silu(rec["u"][t] @ W["w_gate"][e].T) * (rec["u"][t] @ W["w_up"][e].T)
            got.append(yp[pair_row[t * k + j]])
            ref.append(rec["w"][t, jj] * (hid @ W["w_down"][e].T))
    assert rel_l2(got, ref) < REL_L2
    hs = np64(h.debug_buffer("hs", torch.bfloat16, (256, CFG.ffn_shared)))
    assert rel_l2(hs, OL.silu(rec["u"] @ W["ws_gate"].T) * (rec["u"] @ W["ws_up"].T)) < REL_L2
    x = np64(h.debug_buffer("x", torch.float32, (256, d)))
    ex = rel_l2(x[same], rec["x_out"][same])
    print(f"full layer: rel-L2 of the layer output {ex:.2e}, of expert outputs {rel_l2(got, ref):.2e}")
    assert ex < REL_L2


def test_router_epilogue(setup):
    """The shared-expert GEMM's router tile: its fp32 logits against the
    oracle's, and the top-k its epilogue picked against the oracle's routing
    rule applied to those same logits (exact experts, ties to the lower id;
    renormalised softmax weights to fp32 rounding)."""
    h, rec = setup["h"], setup["tr"]
    T, k, E = CFG.canvas, CFG.top_k, CFG.n_experts
    gl = h.debug_buffer("router_logits", torch.float32, (256, E))[:T].cpu().numpy().astype(np.float64)
    assert rel_l2(gl, rec["router_logits"]) < REL_L2
    idx = h.debug_buffer("idx", torch.int32, (T, k)).cpu().numpy()
    wts = h.debug_buffer("w", torch.float32, (T, k)).cpu().numpy()
    ridx, rw = OL.route(gl, k)
    np.testing.assert_array_equal(idx, ridx)
    np.testing.assert_allclose(wts, rw, rtol=2e-6, atol=1e-7)


def test_lm_head_sampled_rows(setup):
    h, rec, ora = setup["h"], setup["tr"], setup["ora"]
    stats = h.debug_buffer("stats", torch.float32, (256, 4)).cpu().numpy().astype(np.float64)
    am = h.debug_buffer("argmax", torch.int32, (256,)).cpu().numpy()
    idx = h.debug_buffer("idx", torch.int32, (256, CFG.top_k)).cpu().numpy()
    same = routing_divergence([idx], [rec["router_logits"]], [rec["idx"]], CFG.top_k) == 1
    assert_excluded_fraction(~same, MAX_EXCLUDED_DIVERGED, "full layer LM head, routed differently at a near-tie")
    rows = np.random.default_rng(1).choice(np.nonzero(same)[0], 32, replace=False)
    xn = OL.rms_norm(rec["x_out"][rows], ora.final_norm, CFG.norm_eps)
    ref = OL.lm_head_stats(xn, ora.embed)
    assert np.max(np.abs(stats[rows, 2] - ref["max"])) < LOGIT_MAX_ABS
    assert np.max(np.abs(stats[rows, 3] - ref["logZ"])) < LOGIT_MAX_ABS
    assert rel_l2(stats[rows, 0], ref["entropy"]) < REL_L2
    n, bad, rate = argmax_agreement(am[rows], ref["logits"], min_rate=0.95)
    print(f"full layer argmax: {n} rows with margin > 1e-2, {bad} differ ({rate:.3f})")


def test_public_step_matches_debug_pass(setup):
    """dg_denoise_step on the same canvas reproduces the pass bit for bit and
    applies the rule to its statistics: the 22 most confident positions are
    frozen to their argmax, every other position is re-drawn."""
    h = setup["h"]
    before = h.debug_buffer("stats", torch.float32, (256, 4)).clone()
    h.denoise_step([0])
    tok, mask, stats, am = h.get_canvas(0)
    h.sync()
    assert torch.equal(stats, before)
    assert h.read_remaining(0) == 256 - 22
    lc = stats[:, 1].cpu().numpy()
    m = mask.cpu().numpy().astype(bool)
    assert m.sum() == 22 and (stats[:, 0].cpu().numpy() > 1.0).all()
    order = sorted(range(256), key=lambda i: (-lc[i], i))
    assert set(np.nonzero(m)[0]) == set(order[:22])
    np.testing.assert_array_equal(tok.cpu().numpy()[m], am.cpu().numpy()[m])
    t = tok.cpu().numpy()
    assert t.min() >= 0 and t.max() < CFG.vocab


def test_lm_sample_full_vocab_sampled_rows(setup):
    """The candidate draw at the full LM-head shape (vocab 262144 = 1024 tiles,
    the benchmark's grid) on exact-logit inputs: sampled rows equal the
    oracle's draw wherever the targets lie more than 3e-5 from an interval edge."""
    import block_diffusion_moe_denoise_b200 as dgm
    from .test_gpu_ops import _assert_argmax_lowest_tied, _exact_lm_inputs, _oracle_draw
    E, x = _exact_lm_inputs(CFG.vocab, CFG.d_model, CFG.canvas, 32, seed=43)
    w = dict(setup["w"])
    w["embed"] = E
    h = dgm.DG(CFG, w, max_requests=1, kv_capacity=CFG.canvas)
    tau, seed, block, step = 0.7, 1234, 1, 4
    _, am, cand = h.op_lm_sample(x, tau, seed, block, step, 0)
    h.sync()
    rows = list(range(0, CFG.canvas, 8)) + [CFG.canvas - 1]
    (c_o, margin), z = _oracle_draw(E, x, rows, CFG.norm_eps, tau, seed, block, step, 0)
    sel = margin > 3e-5
    assert sel.sum() >= 0.75 * len(rows), sel.sum()
    np.testing.assert_array_equal(cand.cpu().numpy()[rows][sel], c_o[sel])
    _assert_argmax_lowest_tied(am.cpu().numpy()[rows], z)
    h.close()


def test_selfcond_op_full_vocab_sampled_rows(setup):
    """The self-conditioning term at the full LM-head shape (vocab 262144, the
    benchmark's grid; MLP width 1024) on exact-logit inputs, sampled rows."""
    import block_diffusion_moe_denoise_b200 as dgm
    from synth import make_selfcond
    from .gpu_common import REL_L2, rel_l2
    from .test_gpu_ops import _exact_lm_inputs, _exact_z, _oracle_selfcond
    cfg = CFG.with_(ffn_selfcond=1024, selfcond_topk=8)
    E, x = _exact_lm_inputs(cfg.vocab, cfg.d_model, cfg.canvas, 32, seed=53)
    w = dict(setup["w"])
    w["embed"] = E
    w.update(make_selfcond(cfg, seed=5, device="cuda"))
    h = dgm.DG(cfg, w, max_requests=1, kv_capacity=cfg.canvas)
    sc, p, ids = h.op_selfcond(0, x)
    h.sync()
    rows = list(range(0, cfg.canvas, 16)) + [cfg.canvas - 1]
    z = _exact_z(E, x, rows, cfg.norm_eps)
    p_o, ids_o, sc_o = _oracle_selfcond(z, E, w, cfg.selfcond_topk)
    np.testing.assert_array_equal(ids.cpu().numpy()[rows], ids_o)
    np.testing.assert_allclose(p.cpu().numpy()[rows], p_o, rtol=1e-4)
    assert rel_l2(sc.cpu().double().numpy()[rows], sc_o) < REL_L2
    h.close()
