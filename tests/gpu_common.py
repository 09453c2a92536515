"""Shared pieces of the GPU parity tests: device weights, tolerances, comparisons.

Tolerances.  The GPU path stores weights and every GEMM input in bf16 and
accumulates in fp32; the oracle runs the same bf16 weights in fp64 on
unrounded activations.  Rounding an activation to bf16 has relative error at
most 2^-9 (RMS about 1.1e-3), so each stage carries a relative L2 error of a
few 1e-3.  The bound used everywhere for bf16 forward values is relative L2
<= 1e-2 and, for logits, max-abs <= 5e-2 (the workload's stated tolerance).
Integer results (routing from identical logits, accept masks, re-noised
tokens, Philox draws) must match bit for bit.
"""
from __future__ import annotations

import numpy as np
import torch

REL_L2 = 1e-2
LOGIT_MAX_ABS = 5e-2


def to_device(w: dict, device="cuda") -> dict:
    return {
        "embed": w["embed"].to(device),
        "final_norm": w["final_norm"].to(device),
        "layers": [{k: v.to(device).contiguous() for k, v in lw.items()} for lw in w["layers"]],
    }


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float32).double().numpy()


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def routing_match(gpu_idx: np.ndarray, ora_idx: np.ndarray) -> np.ndarray:
    """Tokens whose selected experts agree (same set; order may differ only on exact ties)."""
    return np.array([set(a.tolist()) == set(b.tolist()) for a, b in zip(gpu_idx, ora_idx)])
