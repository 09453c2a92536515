"""Seeded synthetic weights and inputs, shared by the oracle tests and the GPU path.

Nothing here computes any step of the method: it only draws random numbers.
Every tensor has its own seed, derived from (base seed, layer, tensor name),
so one layer can be regenerated alone.  Weights are drawn N(0, 0.02) in fp32
and rounded to bf16, the storage type both sides consume; the oracle upcasts
those bf16 values to fp64 exactly.

Weight layout (row-major, "out x in" like a linear layer):
  embed       [V, d]            tied token embedding / LM head
  final_norm  [d]               fp32 gain
  per layer:
    attn_norm [d]               fp32 gain
    w_qkv     [(Hq+2Hkv)*D, d]  rows: q heads, then k heads, then v heads
    w_o       [d, Hq*D]
    ffn_norm  [d]               fp32 gain
    w_router  [E, d]
    w_gate    [E, f_e, d]
    w_up      [E, f_e, d]
    w_down    [E, d, f_e]
    ws_gate   [f_s, d]
    ws_up     [f_s, d]
    ws_down   [d, f_s]
  FP8 checkpoint form (when expert_fp8): w_gate, w_up, w_down hold E4M3 codes
    (uint8) of the bf16 draws divided by one float32 scale per output row
    (largest magnitude -> 448), with w_gate_scale [E, f_e], w_up_scale [E, f_e],
    w_down_scale [E, d]; the checkpoint is an input, like the bf16 weights.
  self-conditioning (when ffn_selfcond > 0):
    sc_gate   [f_sc, d]
    sc_up     [f_sc, d]
    sc_down   [d, f_sc]
"""
from __future__ import annotations

import torch

from .configs import ModelConfig

_TENSOR_IDS = {
    "embed": 1, "final_norm": 2, "attn_norm": 3, "w_qkv": 4, "w_o": 5, "ffn_norm": 6,
    "w_router": 7, "w_gate": 8, "w_up": 9, "w_down": 10, "ws_gate": 11, "ws_up": 12,
    "ws_down": 13, "kv_k": 14, "kv_v": 15, "prompt": 16, "canvas": 17,
    "sc_gate": 18, "sc_up": 19, "sc_down": 20,
}

LAYER_TENSORS = ("attn_norm", "w_qkv", "w_o", "ffn_norm", "w_router", "w_gate", "w_up",
                 "w_down", "ws_gate", "ws_up", "ws_down")


def tensor_seed(base: int, layer: int, name: str) -> int:
    return (base * 1_000_003 + (layer + 1) * 10_007 + _TENSOR_IDS[name] * 101) & ((1 << 62) - 1)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def layer_shapes(cfg: ModelConfig) -> dict:
    d, D, E, fe, fs = cfg.d_model, cfg.head_dim, cfg.n_experts, cfg.ffn_expert, cfg.ffn_shared
    return {
        "attn_norm": (d,), "w_qkv": (cfg.qkv_rows, d), "w_o": (d, cfg.n_q_heads * D),
        "ffn_norm": (d,), "w_router": (E, d), "w_gate": (E, fe, d), "w_up": (E, fe, d),
        "w_down": (E, d, fe), "ws_gate": (fs, d), "ws_up": (fs, d), "ws_down": (d, fs),
    }


def _normal_bf16(shape, seed, device, std, chunk_rows=None):
    g = _gen(device, seed)
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(shape[0], -1)
    step = chunk_rows or max(1, (1 << 26) // max(1, flat.shape[1]))
    for r0 in range(0, flat.shape[0], step):
        r1 = min(flat.shape[0], r0 + step)
        t = torch.randn((r1 - r0, flat.shape[1]), generator=g, device=device, dtype=torch.float32)
        flat[r0:r1] = (t * std).to(torch.bfloat16)
    return out


def _gain(shape, seed, device, gain_std):
    if gain_std == 0.0:
        return torch.ones(shape, dtype=torch.float32, device=device)
    g = _gen(device, seed)
    return 1.0 + gain_std * torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def make_layer(cfg: ModelConfig, layer: int, seed: int = 0, device="cpu", std=0.02,
               gain_std=0.0) -> dict:
    shapes = layer_shapes(cfg)
    w = {}
    for name in LAYER_TENSORS:
        s = tensor_seed(seed, layer, name)
        if name.endswith("norm"):
            w[name] = _gain(shapes[name], s, device, gain_std)
        else:
            w[name] = _normal_bf16(shapes[name], s, device, std)
    if getattr(cfg, "expert_fp8", 0):
        for name in ("w_gate", "w_up", "w_down"):
            w[name], w[name + "_scale"] = _to_e4m3_rows(w[name])
    return w


def _to_e4m3_rows(t):
    """E4M3 codes (uint8) and float32 per-row scales of a bf16 tensor (rows = last dim)."""
    out = torch.empty(t.shape, dtype=torch.uint8, device=t.device)
    scale = torch.empty(t.shape[:-1], dtype=torch.float32, device=t.device)
    step = 1024
    for e in range(t.shape[0]):
        for r0 in range(0, t.shape[1], step):
            x = t[e, r0:r0 + step].float()
            amax = x.abs().amax(dim=-1)
            sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
            q = (x / sc[:, None]).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
            out[e, r0:r0 + step] = q.view(torch.uint8)
            scale[e, r0:r0 + step] = torch.where(amax > 0, sc, torch.zeros_like(sc))
    return out, scale


def make_weights(cfg: ModelConfig, seed: int = 0, device="cpu", std=0.02, gain_std=0.0) -> dict:
    """All weights of the model as bf16 tensors (fp32 norm gains) on `device`."""
    w = {
        "embed": _normal_bf16((cfg.vocab, cfg.d_model), tensor_seed(seed, -1, "embed"), device, std),
        "final_norm": _gain((cfg.d_model,), tensor_seed(seed, -1, "final_norm"), device, gain_std),
        "layers": [make_layer(cfg, l, seed, device, std, gain_std) for l in range(cfg.n_layers)],
    }
    if getattr(cfg, "ffn_selfcond", 0) > 0:
        w.update(make_selfcond(cfg, seed, device, std))
    return w


def make_selfcond(cfg: ModelConfig, seed: int = 0, device="cpu", std=0.02) -> dict:
    """The self-conditioning MLP's weights (sc_gate, sc_up, sc_down) as bf16 tensors."""
    f, d = cfg.ffn_selfcond, cfg.d_model
    return {name: _normal_bf16(shape, tensor_seed(seed, -1, name), device, std)
            for name, shape in (("sc_gate", (f, d)), ("sc_up", (f, d)), ("sc_down", (d, f)))}


def make_kv_prefix(cfg: ModelConfig, n_pos: int, seed: int = 1, device="cpu", layer: int = 0):
    """Synthetic committed K and V for one layer: N(0,1) bf16, shape [Hkv, n_pos, D] each.
    The values are taken as post-RoPE keys and as values at positions 0..n_pos-1."""
    shape = (cfg.n_kv_heads, n_pos, cfg.head_dim)
    k = _normal_bf16(shape, tensor_seed(seed, layer, "kv_k"), device, 1.0)
    v = _normal_bf16(shape, tensor_seed(seed, layer, "kv_v"), device, 1.0)
    return k, v


def make_tokens(cfg: ModelConfig, n: int, seed: int, name: str = "prompt", device="cpu"):
    """Uniform random token ids in [0, vocab), int32."""
    g = _gen(device, tensor_seed(seed, -1, name))
    return torch.randint(0, cfg.vocab, (n,), generator=g, device=device, dtype=torch.int64).to(torch.int32)


def to_f64(t: torch.Tensor):
    """Exact upcast of a (bf16/fp32) tensor to a float64 numpy array."""
    return t.detach().to("cpu", torch.float32).double().numpy()
