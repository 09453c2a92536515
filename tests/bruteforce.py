"""Scalar brute-force restatement of one decoder layer and the LM-head statistics.

Independent of oracle/: plain python floats and loops, no NumPy linear
algebra, written straight from the definitions (RMSNorm, rotate-half RoPE as a
complex rotation, unmasked softmax attention with grouped KV heads, a router
that scores every expert and keeps the k largest, SwiGLU experts, one shared
expert).  Only usable at toy sizes.
"""
from __future__ import annotations

import cmath
import math


def _mv(W, x):                       # W: list of rows (out x in)
    return [sum(wi * xi for wi, xi in zip(row, x)) for row in W]


def _rms(x, g, eps):
    s = math.sqrt(sum(v * v for v in x) / len(x) + eps)
    return [v / s * gi for v, gi in zip(x, g)]


def _rope_complex(vec, pos, theta):
    """Rotate pair (i, i+D/2) as the complex number vec[i] + 1j*vec[i+D/2] by pos*freq_i."""
    D = len(vec)
    h = D // 2
    out = [0.0] * D
    for i in range(h):
        z = complex(vec[i], vec[i + h]) * cmath.exp(1j * pos * theta ** (-2.0 * i / D))
        out[i], out[i + h] = z.real, z.imag
    return out


def _silu(v):
    return v / (1.0 + math.exp(-v))


def _swiglu(u, Wg, Wu, Wd):
    g = _mv(Wg, u)
    up = _mv(Wu, u)
    hid = [_silu(a) * b for a, b in zip(g, up)]
    return _mv(Wd, hid)


def layer(x_rows, pos, Kc, Vc, w, cfg, use_rope=True):
    """x_rows: list of T vectors; pos: T positions; Kc, Vc: committed cache as
    [Hkv][L][D] nested lists (not modified).  Returns (x_out rows, k rows, v rows)."""
    Hq, Hkv, D = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    T = len(x_rows)
    q_all, k_all, v_all = [], [], []
    for t in range(T):
        h = _rms(x_rows[t], w["attn_norm"], cfg.norm_eps)
        qkv = _mv(w["w_qkv"], h)
        q = [qkv[hh * D:(hh + 1) * D] for hh in range(Hq)]
        k = [qkv[(Hq + g) * D:(Hq + g + 1) * D] for g in range(Hkv)]
        v = [qkv[(Hq + Hkv + g) * D:(Hq + Hkv + g + 1) * D] for g in range(Hkv)]
        if use_rope:
            q = [_rope_complex(vec, pos[t], cfg.rope_theta) for vec in q]
            k = [_rope_complex(vec, pos[t], cfg.rope_theta) for vec in k]
        q_all.append(q)
        k_all.append(k)
        v_all.append(v)
    out = []
    for t in range(T):
        o = []
        for hh in range(Hq):
            g = hh * Hkv // Hq
            keys = list(Kc[g]) + [k_all[s][g] for s in range(T)]
            vals = list(Vc[g]) + [v_all[s][g] for s in range(T)]
            sc = [sum(a * b for a, b in zip(q_all[t][hh], kk)) / math.sqrt(D) for kk in keys]
            mx = max(sc)
            e = [math.exp(s - mx) for s in sc]
            Z = sum(e)
            o.extend(sum(e[j] / Z * vals[j][dd] for j in range(len(keys))) for dd in range(D))
        x1 = [a + b for a, b in zip(x_rows[t], _mv(w["w_o"], o))]
        u = _rms(x1, w["ffn_norm"], cfg.norm_eps)
        # router: every expert scored, k best kept (ties to the lower id), renormalised
        r = _mv(w["w_router"], u)
        best = sorted(range(len(r)), key=lambda e_: (-r[e_], e_))[: cfg.top_k]
        mx = max(r)
        p = [math.exp(v - mx) for v in r]
        Z = sum(p[e_] for e_ in best)
        y = [0.0] * len(u)
        for e_ in best:
            ye = _swiglu(u, w["w_gate"][e_], w["w_up"][e_], w["w_down"][e_])
            y = [a + p[e_] / Z * b for a, b in zip(y, ye)]
        ys = _swiglu(u, w["ws_gate"], w["ws_up"], w["ws_down"])
        out.append([a + b + c for a, b, c in zip(x1, y, ys)])
    return out, k_all, v_all


def lm_stats(xn_row, E_rows):
    z = [sum(a * b for a, b in zip(xn_row, e)) for e in E_rows]
    m = max(z)
    a = z.index(m)
    Z = sum(math.exp(v - m) for v in z)
    logZ = m + math.log(Z)
    H = 0.0
    for v in z:
        p = math.exp(v - logZ)
        if p > 0.0:
            H -= p * (v - logZ)
    return dict(argmax=a, max=m, logZ=logZ, entropy=H, logconf=m - logZ)
