"""The decoder pass, the denoising step, commit, prefill and generation loop.

Block-autoregressive decoding ([P2] §"What DiffusionGemma is"; [P3] §"How
diffusion text generation changes the bottleneck"): output is produced in
fixed 256-token canvases.  A canvas starts as random tokens; each step runs a
bidirectional decoder pass over all canvas positions, which attend to the
committed KV cache and to the whole canvas; confident positions are accepted
and the rest re-randomised; a finished canvas is committed to the KV cache and
the next canvas is conditioned on it.  The pass itself is a stack of MoE
decoder layers (128 routed experts, top-8 plus one shared) with a tied LM head
([P1] §"26B MoE Architecture, but Only 3.8B Activated"; [P3] §"The speed
numbers and the hardware they require").

Readings where the pages are silent:
  * a canvas step writes its own K/V into the cache slots [L, L+T) and attends
    to keys [0, L+T) with no mask; L is not advanced;
  * commit re-runs the pass over the final canvas tokens at [L, L+T) and
    advances L (tokens accepted in the last step were not inputs to it, so the
    last step's K/V cannot be reused exactly);
  * prefill is the same segment pass over 256-token segments counted from the
    first prompt token (the last one may be shorter): each segment attends to
    everything before it and bidirectionally to itself, so commit(C) and
    prefill(C) produce identical caches;
  * embedding rows are used unscaled; the LM head is tied to the embedding;
  * self-conditioning (when the model has it) adds a term computed from the
    previous denoising step's logits of the same canvas to the canvas token
    embeddings (see layers.self_condition); a canvas's first step has none,
    and prefill and commit passes never have it.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import layers as L_
from .sampler import DRAW_TILE, candidate_uniforms, draw_candidates, init_canvas, sample_step


@dataclass
class Cache:
    K: list            # per layer [Hkv, capacity, D] float64
    V: list
    length: int = 0    # committed positions


@dataclass
class Trace:
    """Optional per-layer intermediates of one pass (for per-operation parity)."""
    layers: list = field(default_factory=list)
    final: dict = field(default_factory=dict)


class Oracle:
    def __init__(self, cfg, weights):
        """weights: dict with float64 arrays `embed` [V, d], `final_norm` [d] and
        `layers`: a list of per-layer dicts, or a callable l -> dict (names as in
        synth.weights)."""
        self.cfg = cfg
        self._weights = weights
        self.embed = weights["embed"]
        self.final_norm = weights["final_norm"]
        self._layers = weights["layers"]
        self.use_rope = True

    def layer(self, l: int) -> dict:
        return self._layers(l) if callable(self._layers) else self._layers[l]

    def new_cache(self, capacity: int) -> Cache:
        c = self.cfg
        shape = (c.n_kv_heads, capacity, c.head_dim)
        return Cache([np.zeros(shape) for _ in range(c.n_layers)],
                     [np.zeros(shape) for _ in range(c.n_layers)], 0)

    # ---- one pass over a segment -------------------------------------------------
    def forward(self, tokens, cache: Cache, want_stats: bool = True, trace: Trace | None = None,
                n_layers: int | None = None, sc=None):
        """Run the decoder over `tokens` at positions [L, L+T), writing their K/V to
        the cache slots [L, L+T).  `sc` ([T, d]) is added to the token embeddings
        (self-conditioning).  Returns LM-head statistics (or None)."""
        c = self.cfg
        tokens = np.asarray(tokens, dtype=np.int64)
        T = tokens.shape[0]
        L = cache.length
        Hq, Hkv, D = c.n_q_heads, c.n_kv_heads, c.head_dim
        pos = L + np.arange(T)
        x = self.embed[tokens].astype(np.float64)
        if sc is not None:
            x = x + sc
        for l in range(c.n_layers if n_layers is None else n_layers):
            w = self.layer(l)
            rec = {"x_in": x.copy()} if trace is not None else None
            h = L_.rms_norm(x, w["attn_norm"], c.norm_eps)
            qkv = h @ w["w_qkv"].T
            q = qkv[:, : Hq * D].reshape(T, Hq, D)
            k = qkv[:, Hq * D: (Hq + Hkv) * D].reshape(T, Hkv, D)
            v = qkv[:, (Hq + Hkv) * D:].reshape(T, Hkv, D)
            if self.use_rope:
                q = L_.rope(q, pos, c.rope_theta)
                k = L_.rope(k, pos, c.rope_theta)
            cache.K[l][:, L:L + T] = k.transpose(1, 0, 2)
            cache.V[l][:, L:L + T] = v.transpose(1, 0, 2)
            o = L_.attention(q, cache.K[l][:, : L + T], cache.V[l][:, : L + T])
            x = x + o.reshape(T, Hq * D) @ w["w_o"].T
            u = L_.rms_norm(x, w["ffn_norm"], c.norm_eps)
            r = u @ w["w_router"].T
            idx, wts = L_.route(r, c.top_k)
            experts = L_.routed_experts_fp8 if getattr(c, "expert_fp8", 0) else L_.routed_experts
            y = experts(u, idx, wts, w["w_gate"], w["w_up"], w["w_down"])
            ys = L_.swiglu(u, w["ws_gate"], w["ws_up"], w["ws_down"])
            if rec is not None:
                rec.update(h=h, q=q, k=k, v=v, o=o, x_attn=x.copy(), u=u, router_logits=r,
                           idx=idx, w=wts, y_routed=y, y_shared=ys)
            x = x + y + ys
            if rec is not None:
                rec["x_out"] = x.copy()
                trace.layers.append(rec)
        if not want_stats:
            return None
        xn = L_.rms_norm(x, self.final_norm, c.norm_eps)
        st = L_.lm_head_stats(xn, self.embed)
        if trace is not None:
            trace.final = dict(x=x, xn=xn, **st)
        return st

    # ---- the loop pieces -------------------------------------------------------------
    def prefill(self, cache: Cache, tokens) -> None:
        tokens = np.asarray(tokens, dtype=np.int64)
        seg = self.cfg.canvas
        for s0 in range(0, tokens.shape[0], seg):
            part = tokens[s0: s0 + seg]
            self.forward(part, cache, want_stats=False)
            cache.length += part.shape[0]

    def commit(self, cache: Cache, canvas) -> None:
        canvas = np.asarray(canvas, dtype=np.int64)
        self.forward(canvas, cache, want_stats=False)
        cache.length += canvas.shape[0]

    def self_condition(self, prev_logits):
        """Self-conditioning term from the previous step's logits (None at a canvas's
        first step, or when the model has none)."""
        c = self.cfg
        if prev_logits is None or getattr(c, "ffn_selfcond", 0) <= 0:
            return None
        w = self._weights
        return L_.self_condition(prev_logits, self.embed, w["sc_gate"], w["sc_up"], w["sc_down"], c.selfcond_topk)

    def denoise_step(self, cache: Cache, canvas, accepted, *, seed: int, block: int, step: int,
                     request: int = 0, stats=None, prev_argmax=None, prev_logits=None):
        """One step: pass over the canvas (unless `stats` is given), then the sampler
        (the configuration's rule; `prev_argmax` = the previous step's argmax, for
        the entropy-budget rule; `prev_logits` = the previous step's logits, for
        self-conditioning).  Returns (canvas, accepted, remaining, stats)."""
        c = self.cfg
        if stats is None:
            stats = self.forward(canvas, cache, want_stats=True, sc=self.self_condition(prev_logits))
        cand = None
        tau = getattr(c, "temperature", 0.0)
        if tau > 0:
            n = stats["logits"].shape[0]
            u_row, u_tile = candidate_uniforms(seed, block, step, np.arange(n), c.vocab // DRAW_TILE, request)
            cand, _ = draw_candidates(stats["logits"], tau, u_row, u_tile)
        canvas, accepted, remaining = sample_step(
            canvas, accepted, stats["argmax"], stats["entropy"], stats["logconf"], seed=seed,
            block=block, step=step, vocab=c.vocab, entropy_thresh=c.entropy_thresh,
            min_accept=c.min_accept, max_steps=c.max_steps, request=request,
            rule="budget" if getattr(c, "sampler", 0) == 1 else "threshold",
            entropy_budget=getattr(c, "entropy_budget", 0.1), stop_entropy=getattr(c, "stop_entropy", 0.005),
            prev_argmax=prev_argmax, candidates=cand)
        return canvas, accepted, remaining, stats

    def open_canvas(self, *, seed: int, block: int, request: int = 0):
        return init_canvas(self.cfg.canvas, seed=seed, block=block, vocab=self.cfg.vocab,
                           request=request)

    def generate(self, prompt, n_out: int, seed: int, request: int = 0, capacity: int | None = None):
        """Prefill `prompt`, then produce n_out tokens as consecutive canvases.
        Returns (tokens int64 [n_out], steps per canvas)."""
        c = self.cfg
        prompt = np.asarray(prompt, dtype=np.int64)
        cap = capacity or (prompt.shape[0] + n_out)
        cache = self.new_cache(cap)
        self.prefill(cache, prompt)
        out, steps = [], []
        for b in range(n_out // c.canvas):
            canvas, accepted = self.open_canvas(seed=seed, block=b, request=request)
            s = 0
            prev = prev_logits = None
            while True:
                s += 1
                canvas, accepted, rem, st = self.denoise_step(cache, canvas, accepted, seed=seed, block=b,
                                                              step=s, request=request, prev_argmax=prev,
                                                              prev_logits=prev_logits)
                prev = st["argmax"]
                prev_logits = st["logits"]
                if rem == 0:
                    break
            steps.append(s)
            self.commit(cache, canvas)
            out.append(canvas)
        return np.concatenate(out), steps
