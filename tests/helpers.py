"""Shared test helpers: converting synthetic weights for the oracle, tolerances."""
from __future__ import annotations

import numpy as np

from synth import to_f64


def oracle_weights(w: dict) -> dict:
    """float64 copies of a synth weight dict (exact upcast of bf16/fp32 values)."""
    out = {
        "embed": to_f64(w["embed"]),
        "final_norm": to_f64(w["final_norm"]),
        "layers": [_layer_f64(lw) for lw in w["layers"]],
    }
    for name in ("sc_gate", "sc_up", "sc_down"):
        if name in w:
            out[name] = to_f64(w[name])
    return out


def _layer_f64(lw: dict) -> dict:
    """float64 layer weights; FP8 expert weights (codes + per-row scales) dequantised exactly."""
    from oracle.quant import e4m3_decode
    out = {}
    for k, v in lw.items():
        if k.endswith("_scale"):
            continue
        if k + "_scale" in lw:
            out[k] = e4m3_decode(v.cpu().numpy()) * to_f64(lw[k + "_scale"])[..., None]
        else:
            out[k] = to_f64(v)
    return out


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64))))
