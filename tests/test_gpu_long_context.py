"""GPU vs oracle for the long-context batched step at full shape: four
requests, each with a 65,536-token synthetic committed KV prefix and its own
256-token canvas, denoised together in one step (1,024 canvas tokens routed
together).  One decoder layer at full width plus the LM head over the full
vocabulary.  The oracle cannot run the whole step in fp64 on the host, so it
checks sampled outputs it computes one by one: attention rows of sampled
(request, query head, token) triples over all 65,792 keys, and the LM-head
statistics of sampled tokens (each token's layer output depends only on its
own attention output)."""
import numpy as np
import pytest
import torch

from oracle import layers as OL
from synth import LAYER, make_kv_prefix, make_weights, to_f64

from .gpu_common import (LOGIT_MAX_ABS, MAX_EXCLUDED_NEAR_TIES, REL_L2, argmax_agreement, assert_excluded_fraction,
                         np64, rel_l2, routing_divergence)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

CFG = LAYER
L_PREFIX = 65536
N_REQ = 4


@pytest.fixture(scope="module")
def setup():
    import block_diffusion_moe_denoise_b200 as dgm
    w = make_weights(CFG, seed=0, device="cuda")
    h = dgm.DG(CFG, w, max_requests=N_REQ, kv_capacity=L_PREFIX + CFG.canvas)
    kvs = []
    for r in range(N_REQ):
        k, v = make_kv_prefix(CFG, L_PREFIX, seed=10 + r, device="cuda")
        h.set_kv(r, 0, 0, k, v)
        h.set_kv_len(r, L_PREFIX)
        h.open_canvas(r, 100 + r, 0)
        kvs.append((k, v))
    canv = [h.get_canvas(r)[0].cpu().numpy().astype(np.int64) for r in range(N_REQ)]
    h.denoise_step(list(range(N_REQ)))
    h.sync()
    T = N_REQ * CFG.canvas
    Tcap = T
    out = dict(h=h, w=w, kvs=kvs, canv=canv,
               o=np64(h.debug_buffer("o", torch.bfloat16, (Tcap, CFG.n_q_heads * CFG.head_dim))),
               stats=h.debug_buffer("stats", torch.float32, (Tcap, 4)).cpu().numpy().astype(np.float64),
               argmax=h.debug_buffer("argmax", torch.int32, (Tcap,)).cpu().numpy(),
               idx=h.debug_buffer("idx", torch.int32, (Tcap, CFG.top_k)).cpu().numpy(),
               remaining=[h.read_remaining(r) for r in range(N_REQ)])
    yield out
    h.close()


def _oracle_canvas_qkv(lw, embed, canvas, pos0):
    """q, k, v of every canvas token of one request (RoPE at pos0 + i)."""
    c = CFG
    x = to_f64(embed[torch.from_numpy(canvas).to(embed.device)])
    hn = OL.rms_norm(x, to_f64(lw["attn_norm"]), c.norm_eps)
    qkv = hn @ to_f64(lw["w_qkv"]).T
    Hq, Hkv, D = c.n_q_heads, c.n_kv_heads, c.head_dim
    T = canvas.shape[0]
    q = qkv[:, :Hq * D].reshape(T, Hq, D)
    k = qkv[:, Hq * D:(Hq + Hkv) * D].reshape(T, Hkv, D)
    v = qkv[:, (Hq + Hkv) * D:].reshape(T, Hkv, D)
    pos = pos0 + np.arange(T)
    return x, OL.rope(q, pos, c.rope_theta), OL.rope(k, pos, c.rope_theta), v


def test_all_requests_took_one_step(setup):
    assert setup["remaining"] == [CFG.canvas - CFG.min_accept] * N_REQ


def test_sampled_attention_rows_over_65k_keys(setup):
    c = CFG
    lw, embed = setup["w"]["layers"][0], setup["w"]["embed"]
    rng = np.random.default_rng(0)
    got, ref = [], []
    for r in range(N_REQ):
        x, q, k, v = _oracle_canvas_qkv(lw, embed, setup["canv"][r], L_PREFIX)
        kp, vp = setup["kvs"][r]
        for _ in range(3):
            t = int(rng.integers(0, c.canvas))
            hq = int(rng.integers(0, c.n_q_heads))
            g = hq * c.n_kv_heads // c.n_q_heads
            K = np.concatenate([to_f64(kp[g]), k[:, g]], 0)
            V = np.concatenate([to_f64(vp[g]), v[:, g]], 0)
            o = OL.attention(q[t:t + 1, hq:hq + 1], K[None], V[None])[0, 0]
            ref.append(o)
            got.append(setup["o"][r * c.canvas + t, hq * c.head_dim:(hq + 1) * c.head_dim])
    e = rel_l2(got, ref)
    print(f"long context: attention rows rel-L2 {e:.2e}")
    assert e < REL_L2


def test_sampled_lm_head_statistics(setup):
    """Whole layer + LM head for 32 sampled tokens (8 per request): the attention
    of each sampled token over its request's 65,792 keys, then its MoE and the
    full-vocabulary statistics.  A sampled token whose GPU routing differs from
    the oracle's must be a near-tie and is left out (counted; at most 20% of
    so small a sample, against ~5% expected);
    on the rest, max logit within the logit bound and argmax equal where the
    oracle's margin exceeds twice it, at a rate >= 95% where it exceeds 1e-2."""
    c = CFG
    lw = {n: to_f64(t) for n, t in setup["w"]["layers"][0].items()}
    embed = setup["w"]["embed"]
    rng = np.random.default_rng(1)
    rows, xns, rls, oidx = [], [], [], []
    for r in range(N_REQ):
        x, q, k, v = _oracle_canvas_qkv(setup["w"]["layers"][0], embed, setup["canv"][r], L_PREFIX)
        kp, vp = setup["kvs"][r]
        Kall = [np.concatenate([to_f64(kp[g]), k[:, g]], 0) for g in range(c.n_kv_heads)]
        Vall = [np.concatenate([to_f64(vp[g]), v[:, g]], 0) for g in range(c.n_kv_heads)]
        for t in rng.choice(c.canvas, 8, replace=False):
            o = OL.attention(q[t:t + 1], np.stack(Kall), np.stack(Vall))[0]
            xa = x[t] + o.reshape(-1) @ lw["w_o"].T
            u = OL.rms_norm(xa[None], lw["ffn_norm"], c.norm_eps)
            rl = u @ lw["w_router"].T
            idx, wts = OL.route(rl, c.top_k)
            y = OL.routed_experts(u, idx, wts, lw["w_gate"], lw["w_up"], lw["w_down"])
            xo = xa + y[0] + OL.swiglu(u, lw["ws_gate"], lw["ws_up"], lw["ws_down"])[0]
            xns.append(OL.rms_norm(xo[None], to_f64(setup["w"]["final_norm"]), c.norm_eps)[0])
            rls.append(rl[0])
            oidx.append(idx[0])
            rows.append(r * c.canvas + t)
    rows = np.array(rows)
    same = routing_divergence([setup["idx"][rows]], [np.stack(rls)], [np.stack(oidx)], c.top_k) == 1
    assert_excluded_fraction(~same, MAX_EXCLUDED_NEAR_TIES, "long context, sampled tokens routed differently")
    assert same.sum() >= 16
    XN = np.stack(xns)[same]
    rows = rows[same]
    ref_logits = np.concatenate([XN @ to_f64(embed[i:i + 32768]).T for i in range(0, c.vocab, 32768)], axis=1)
    ref_max = ref_logits.max(axis=1)
    st, am = setup["stats"], setup["argmax"]
    assert np.max(np.abs(st[rows, 2] - ref_max)) < LOGIT_MAX_ABS
    n, bad, rate = argmax_agreement(am[rows], ref_logits, min_rate=0.95)
    print(f"long context: {len(rows)} sampled tokens, argmax {n - bad}/{n} at margin > 1e-2")
