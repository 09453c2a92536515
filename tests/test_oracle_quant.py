"""Pins of the oracle's FP8 (E4M3) codec, per-row quantisation and FP8 expert
path (no GPU).  The codec is checked against PyTorch's float8_e4m3fn type (an
independent library implementation of the same format) on every code and on
random and tie values; saturation follows the format's largest finite value."""
import numpy as np
import torch

from oracle import layers as L
from oracle import quant as Q


def test_decode_matches_library_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = Q.e4m3_decode(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    assert Q.e4m3_decode(np.uint8(0x7E)) == 448.0 and Q.e4m3_decode(np.uint8(0x01)) == 2.0 ** -9


def test_encode_matches_library_round_to_nearest_even():
    rng = np.random.default_rng(0)
    vals = np.concatenate([rng.normal(0, 30, 20000), rng.normal(0, 0.01, 5000),
                           rng.uniform(-464, 464, 5000)]).astype(np.float32)
    # exact midpoints between neighbouring codes (ties to the even mantissa)
    rep = np.unique(np.abs(Q.e4m3_decode(np.arange(0x7E + 1, dtype=np.uint8))))
    mids = ((rep[1:] + rep[:-1]) / 2).astype(np.float32)
    vals = np.concatenate([vals, mids, -mids])
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = Q.e4m3_encode(vals)
    # +0 / -0: the library keeps the sign of zero results, the value is the same
    same = (got == ref) | ((Q.e4m3_decode(got) == 0) & (Q.e4m3_decode(ref) == 0))
    assert same.all(), vals[~same][:10]


def test_encode_saturates_and_keeps_nan():
    got = Q.e4m3_encode(np.array([464.0, 480.0, 1e9, -1e9, np.nan]))
    np.testing.assert_array_equal(got, [0x7E, 0x7E, 0x7E, 0xFE, 0x7F])


def test_quantize_rows_properties():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(64, 300)) * np.exp(rng.normal(size=(64, 1)))
    codes, scale = Q.quantize_rows(x)
    # the largest magnitude of each row lands on +-448
    i = np.abs(x).argmax(axis=1)
    np.testing.assert_array_equal(np.abs(Q.e4m3_decode(codes[np.arange(64), i])), 448.0)
    # round to nearest with 3 mantissa bits: relative error <= 2^-4 above the subnormal range
    xd = Q.dequantize_rows(codes, scale)
    normal = np.abs(x) >= 2.0 ** -6 * scale[:, None] * (1 + 1e-6)
    assert np.all(np.abs(xd - x)[normal] <= 2.0 ** -4 * np.abs(x)[normal] * (1 + 1e-6))
    # scaling a row by a power of two keeps the codes and scales the scale
    c2, s2 = Q.quantize_rows(x * 8.0)
    np.testing.assert_array_equal(c2, codes)
    np.testing.assert_array_equal(s2, scale * 8)
    # a zero row
    c0, s0 = Q.quantize_rows(np.zeros((1, 10)))
    assert not c0.any() and s0[0] == 0


def test_fp8_experts_reduce_to_exact_path_on_representable_rows():
    """Rows whose entries are E4M3 values times 2^j with max 448 * 2^j quantise
    exactly; with one hidden unit per expert the SwiGLU row has a single entry
    that quantises to +-448 times its own scale.  The FP8 path then equals the
    plain routed experts up to the float32 rounding of that scale."""
    rng = np.random.default_rng(2)
    T, d, E, k = 6, 16, 4, 2
    codes = rng.integers(0, 0x7E, size=(T, d)).astype(np.uint8)
    codes[:, 0] = 0x7E                                     # 448 in every row
    u = Q.e4m3_decode(codes) * np.exp2(rng.integers(-8, 3, size=(T, 1)))
    Wg, Wu, Wd = rng.normal(size=(E, 1, d)), rng.normal(size=(E, 1, d)), rng.normal(size=(E, d, 1))
    idx = np.array([rng.choice(E, k, replace=False) for _ in range(T)])
    w = rng.uniform(0.2, 1, size=(T, k))
    np.testing.assert_allclose(L.routed_experts_fp8(u, idx, w, Wg, Wu, Wd),
                               L.routed_experts(u, idx, w, Wg, Wu, Wd), rtol=1e-6, atol=1e-12)
