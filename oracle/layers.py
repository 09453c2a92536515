"""The per-layer operations of the denoising pass, in float64 NumPy.

Every function is the plain definition of its operation.  Page tags are
defined in the package docstring.

The pages fix the structure (bidirectional attention over the committed
context and the whole canvas [P1] §"26B MoE Architecture"; [P2] §"What
DiffusionGemma is"; 128 experts, top-8 plus one shared expert [P3] §"The speed
numbers and the hardware they require") but not the Gemma internals.  The
readings taken where they are silent:
  * pre-norm RMSNorm with a learned gain, eps 1e-6;
  * rotate-half RoPE (pairs i, i + D/2), theta 1e4, angle = pos * theta^(-2i/D);
  * score scale 1/sqrt(D); no mask over prefix + canvas; q-head h reads
    kv-head floor(h * Hkv / Hq);
  * router softmax over all experts, top-k by logit with ties to the lower
    expert id, the k probabilities renormalised to sum to 1;
  * SwiGLU experts silu(u Wg^T) * (u Wu^T) then Wd; the shared expert has the
    same form and is added with weight 1;
  * tied LM head z = RMSNorm(x) E^T with per-row argmax (lowest id on ties),
    log-partition, entropy in nats and log-confidence log max p.
"""
from __future__ import annotations

import numpy as np


def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * g over the last axis."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * g


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE.  x: [T, H, D]; pos: [T] absolute positions."""
    D = x.shape[-1]
    half = D // 2
    i = np.arange(half, dtype=np.float64)
    freq = theta ** (-2.0 * i / D)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * freq[None, :]
    cos = np.cos(ang)[:, None, :]
    sin = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """Unmasked softmax attention with grouped KV heads.

    q: [T, Hq, D]; K, V: [Hkv, S, D] (all S keys visible to every query).
    Returns [T, Hq, D]."""
    T, Hq, D = q.shape
    Hkv = K.shape[0]
    out = np.empty_like(q)
    for h in range(Hq):
        g = h * Hkv // Hq
        s = q[:, h, :] @ K[g].T / np.sqrt(D)
        s = s - s.max(axis=-1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=-1, keepdims=True)
        out[:, h, :] = p @ V[g]
    return out


def silu(v: np.ndarray) -> np.ndarray:
    return v / (1.0 + np.exp(-v))


def swiglu(u: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray) -> np.ndarray:
    """silu(u wg^T) * (u wu^T), then wd.  wg, wu: [f, d]; wd: [d, f]."""
    return (silu(u @ wg.T) * (u @ wu.T)) @ wd.T


def route(r: np.ndarray, k: int):
    """Router: softmax over experts, top-k (ties to the lower expert id), renormalised.

    r: [T, E] router logits.  Returns idx int64 [T, k] (in selection order, i.e.
    descending logit, ties by id) and w float64 [T, k] summing to 1 per row."""
    T, E = r.shape
    p = np.exp(r - r.max(axis=-1, keepdims=True))
    p = p / p.sum(axis=-1, keepdims=True)
    # stable sort of -r keeps equal logits in ascending expert order
    idx = np.argsort(-r, axis=-1, kind="stable")[:, :k]
    sel = np.take_along_axis(p, idx, axis=-1)
    w = sel / sel.sum(axis=-1, keepdims=True)
    return idx, w


def routed_experts(u: np.ndarray, idx: np.ndarray, w: np.ndarray, Wg, Wu, Wd) -> np.ndarray:
    """sum_j w[t,j] * expert_{idx[t,j]}(u_t), looping over experts with gathered rows.

    Wg, Wu: [E, f, d]; Wd: [E, d, f]."""
    T = u.shape[0]
    E = Wg.shape[0]
    y = np.zeros((T, Wd.shape[1]), dtype=np.float64)
    for e in range(E):
        rows, slots = np.nonzero(idx == e)
        if rows.size == 0:
            continue
        ye = swiglu(u[rows], Wg[e], Wu[e], Wd[e])
        y[rows] += w[rows, slots][:, None] * ye
    return y


def routed_experts_fp8(u: np.ndarray, idx: np.ndarray, w: np.ndarray, Wg, Wu, Wd) -> np.ndarray:
    """routed_experts with FP8 expert GEMMs (oracle/quant.py): the weights are the
    dequantised E4M3 weights; each token's row is quantised per row before
    gate|up, and each SwiGLU row before down."""
    from .quant import fake_quant_rows
    T, d = u.shape
    out = np.zeros((T, d))
    xq = fake_quant_rows(u)
    for t in range(T):
        for j in range(idx.shape[1]):
            e = idx[t, j]
            h = silu(xq[t] @ Wg[e].T) * (xq[t] @ Wu[e].T)
            out[t] += w[t, j] * (fake_quant_rows(h[None, :])[0] @ Wd[e].T)
    return out


def histogram_and_permutation(idx: np.ndarray, n_experts: int):
    """Counts per expert, exclusive-scan offsets and the (token, slot) pairs
    grouped by expert, ordered by token inside each expert.

    Returns counts int64 [E], offsets int64 [E+1], perm int64 [T*k] holding
    t*k + j, and inv int64 [T, k]: the row of pair (t, j) in the grouped order."""
    T, k = idx.shape
    counts = np.array([(idx == e).sum() for e in range(n_experts)], dtype=np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    perm = np.empty(T * k, dtype=np.int64)
    inv = np.empty((T, k), dtype=np.int64)
    fill = offsets[:-1].copy()
    for t in range(T):                       # ascending token order inside each expert
        for j in range(k):
            e = idx[t, j]
            perm[fill[e]] = t * k + j
            inv[t, j] = fill[e]
            fill[e] += 1
    return counts, offsets, perm, inv


def lm_head_stats(xn: np.ndarray, E_tok: np.ndarray):
    """Full logits z = xn E^T and, per row: argmax (lowest id on ties), max logit,
    log-partition logZ, entropy H = -sum p ln p (nats) and logconf = ln max p.

    xn: [T, d] (already normalised); E_tok: [V, d]."""
    z = xn @ E_tok.T
    a = np.argmax(z, axis=-1)                      # first occurrence = lowest id
    m = z.max(axis=-1)
    logZ = m + np.log(np.exp(z - m[:, None]).sum(axis=-1))
    logp = z - logZ[:, None]
    p = np.exp(logp)
    H = -(p * logp).sum(axis=-1)
    logconf = m - logZ
    return dict(argmax=a.astype(np.int64), max=m, logZ=logZ, entropy=H, logconf=logconf, logits=z)


def topk_probs(z: np.ndarray, k: int):
    """Per row, the k largest entries of softmax(z) (ties to the lower id) and their ids.
    Returns (p [T, k], ids [T, k]) in descending probability order."""
    z = np.asarray(z, dtype=np.float64)
    m = z.max(axis=-1, keepdims=True)
    e = np.exp(z - m)
    p = e / e.sum(axis=-1, keepdims=True)
    order = np.argsort(-z, axis=-1, kind="stable")[:, :k]     # stable: equal logits keep id order
    return np.take_along_axis(p, order, axis=-1), order.astype(np.int64)


def soft_embedding(p: np.ndarray, ids: np.ndarray, E_tok: np.ndarray) -> np.ndarray:
    """sum_k p[t, k] E[ids[t, k]] per row: the embedding expected under the given
    (truncated) distribution."""
    return np.einsum("tk,tkd->td", p, E_tok[ids])


def self_condition(z_prev: np.ndarray, E_tok: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray,
                   k: int) -> np.ndarray:
    """Self-conditioning term added to the canvas embeddings ([P2] "How the sampler
    actually works": the previous step's softmax goes back through a small gated
    MLP).  Reading (the pages give no shape): the previous step's softmax at each
    position, truncated to its k largest entries (not renormalised), is turned
    into the expected embedding under it, and a gated MLP of the shared expert's
    form maps that to the residual stream."""
    p, ids = topk_probs(z_prev, k)
    return swiglu(soft_embedding(p, ids, E_tok), wg, wu, wd)

