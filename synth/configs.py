"""Model shapes and workloads of the synthetic block-diffusion MoE decoder.

This module holds dimensions only: no arithmetic of the method lives here.

The full shape follows the DiffusionGemma pages: 128 routed experts with
top-8 plus one shared expert, 25.2B total / 3.8B active parameters and a
256-token canvas (carussignal.com, "The speed numbers and the hardware they
require"; saify.me, "What DiffusionGemma is").  The exact dims (d_model 2816,
16 query / 8 KV heads of width 256, expert width 704, shared width 2112,
vocab 262144, 30 layers) are synthetic choices sized to reproduce those two
parameter counts.
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class ModelConfig:
    n_layers: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n_experts: int
    top_k: int
    ffn_expert: int
    ffn_shared: int
    vocab: int
    canvas: int = 256
    max_steps: int = 12
    min_accept: int = 22
    entropy_thresh: float = 1.0
    rope_theta: float = 10000.0
    norm_eps: float = 1e-6
    sampler: int = 0               # 0: entropy threshold + min_accept; 1: the pages' entropy budget
    entropy_budget: float = 0.1
    stop_entropy: float = 0.005
    temperature: float = 0.0       # 0: argmax candidates; > 0: candidates drawn from softmax(z / temperature)
    ffn_selfcond: int = 0          # self-conditioning gated-MLP width (0: off)
    selfcond_topk: int = 8         # softmax entries of the previous step fed back per position
    expert_fp8: int = 0            # 1: routed-expert weights E4M3 with per-row scales, W8A8 GEMMs

    @property
    def qkv_rows(self) -> int:
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim

    def with_(self, **kw) -> "ModelConfig":
        return replace(self, **kw)

    # parameter counts (weights only; norm gains excluded)
    def params_per_layer(self) -> int:
        d, D = self.d_model, self.head_dim
        attn = self.qkv_rows * d + d * self.n_q_heads * D
        experts = self.n_experts * 3 * self.ffn_expert * d
        shared = 3 * self.ffn_shared * d
        router = self.n_experts * d
        return attn + experts + shared + router

    def total_params(self) -> int:
        return self.n_layers * self.params_per_layer() + self.vocab * self.d_model

    def active_params_per_token(self) -> int:
        d, D = self.d_model, self.head_dim
        attn = self.qkv_rows * d + d * self.n_q_heads * D
        per_layer = attn + self.top_k * 3 * self.ffn_expert * d + 3 * self.ffn_shared * d + self.n_experts * d
        return self.n_layers * per_layer + self.vocab * self.d_model


# Tiny full loop: 2 layers, d 256, 4/2 heads of 64, 16 experts top-2 + shared,
# SwiGLU width 512 (experts and shared), vocab 2048.
TINY = ModelConfig(n_layers=2, d_model=256, n_q_heads=4, n_kv_heads=2, head_dim=64,
                   n_experts=16, top_k=2, ffn_expert=512, ffn_shared=512, vocab=2048)

# Full synthetic stack: 30 layers at the shape above.
FULL = ModelConfig(n_layers=30, d_model=2816, n_q_heads=16, n_kv_heads=8, head_dim=256,
                   n_experts=128, top_k=8, ffn_expert=704, ffn_shared=2112, vocab=262144)

# One decoder layer at full shape (plus the tied LM head over the full vocab).
LAYER = FULL.with_(n_layers=1)


@dataclass(frozen=True)
class Workload:
    name: str
    model: ModelConfig
    n_requests: int
    kv_prefix: int          # committed KV length per request before the step
    synthetic_kv: bool      # prefix K/V drawn N(0,1) instead of prefilled
    n_out: int = 256        # output tokens per request (multiple of canvas)
    seed: int = 0


WORKLOADS = {
    # tiny full loop: 128-token prompt prefilled, one canvas, then commit
    "tiny": Workload("tiny", TINY, 1, 128, False, 256, 0),
    # one layer, one step, 4096-token synthetic prefix
    "layer": Workload("layer", LAYER, 1, 4096, True, 256, 0),
    # full stack, one step, 4096-token prefix
    "full_step": Workload("full_step", FULL, 1, 4096, True, 256, 0),
    # end-to-end generation: 4096-token prompt, 1024 output tokens, Philox seed 1234
    "generate": Workload("generate", FULL, 1, 4096, False, 1024, 1234),
    # four requests with 65536-token prefixes denoised together
    "long": Workload("long", FULL, 4, 65536, True, 256, 0),
}
