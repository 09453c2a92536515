"""FP8 (E4M3) expert weights and activations.

The pages name FP8 and NVFP4 checkpoints of the model ([P2] "Serve it with
vLLM") and a quantised model that fits 18 GB ([P1] "26B MoE Architecture, but
Only 3.8B Activated"; [P4] "What's new") without giving the scheme.
Reading taken (the common W8A8 form): expert weights are stored as E4M3 codes
with one float32 scale per output row (W = decode(q) * scale); the expert
inputs -- the normalised token rows entering gate|up and the SwiGLU rows
entering down -- are quantised per row on the fly:
  amax  = max_i |x_i|                      (float32)
  s_inv = 448 / amax                       (float32 division)
  q_i   = E4M3(x_i * s_inv)                (float32 product, round to nearest
                                            even, saturating at +-448)
  scale = amax / 448                       (float32 division)
and a row of zeros gives zero codes and scale 0.  The GEMM then sums
decode(q_w) decode(q_x) exactly and applies both scales.

E4M3 (the OCP 8-bit floating-point "E4M3" format): sign, 4 exponent bits with
bias 7, 3 mantissa bits; exponent field 0 holds the subnormals m * 2^-9;
S.1111.111 is NaN; no infinities; largest finite value 448.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """Values (float64) of E4M3 codes (uint8)."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 0xF) & ((c & 0x7) == 0x7), np.nan, val)
    return sign * val


def e4m3_encode(y) -> np.ndarray:
    """E4M3 codes of float values: round to nearest, ties to even mantissa,
    saturating to +-448; NaN gives the NaN code 0x7F."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    f, E = np.frexp(np.where(a > 0, a, 1.0))          # a = f 2^E, f in [0.5, 1): exact
    e = np.maximum(E - 1, -6)                          # exponent of the leading bit, normals >= 2^-6
    quantum = np.exp2(e - 3.0)                         # 3 mantissa bits (2^-9 for subnormals)
    q = np.rint(a / quantum) * quantum                 # exact: a / quantum < 16; rint ties to even
    q = np.minimum(q, E4M3_MAX)
    q = np.where(a > 0, q, 0.0)
    # code of the representable value q
    fq, Eq = np.frexp(np.where(q > 0, q, 1.0))
    eq = Eq - 1
    normal = q >= 2.0 ** -6
    exp_field = np.where(normal, eq + 7, 0)
    mant = np.where(normal, np.rint((q / np.exp2(eq) - 1.0) * 8.0), np.rint(q / 2.0 ** -9))
    code = (exp_field << 3) | mant.astype(np.int64)
    code = np.where(q > 0, code, 0) | np.where(np.signbit(y) & (q > 0), 0x80, 0)
    code = np.where(np.isnan(y), 0x7F, code)
    return code.astype(np.uint8)


def quantize_rows(x):
    """Per-row E4M3 quantisation in float32 (see the module docstring).
    x: [R, n].  Returns (codes uint8 [R, n], scale float32 [R])."""
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    amax = np.abs(x32).max(axis=-1)
    safe = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
    s_inv = (np.float32(E4M3_MAX) / safe).astype(np.float32)
    y = (x32 * s_inv[:, None]).astype(np.float32)
    codes = e4m3_encode(y)
    codes = np.where(amax[:, None] > 0, codes, 0).astype(np.uint8)
    scale = np.where(amax > 0, (amax / np.float32(E4M3_MAX)).astype(np.float32), np.float32(0.0))
    return codes, scale.astype(np.float32)


def dequantize_rows(codes, scale) -> np.ndarray:
    """decode(codes) * scale per row, float64 (exact)."""
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[..., None]


def fake_quant_rows(x) -> np.ndarray:
    """The values a row carries into an FP8 GEMM: dequantize(quantize(x))."""
    return dequantize_rows(*quantize_rows(x))
