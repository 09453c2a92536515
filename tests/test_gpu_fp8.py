"""FP8 (E4M3) routed experts on the GPU.

The per-row quantisation of the expert inputs is checked bit for bit against
the oracle's quantisation (oracle.quant, itself pinned against PyTorch's
float8_e4m3fn on every code and midpoint) of the kernel's own rows (the codes
are an integer decision: both sides take it in float32 from the same bf16 row).  The
two tcgen05 kind::f8f6f4 GEMMs are checked against float64 products of their own
input codes and scales.  The routed-expert output is compared with the oracle's
FP8 path: the GPU's activations carry the ~3e-3 relative error of bf16 GEMM
inputs, which moves some values across an E4M3 rounding boundary (a step of
6-12%); simulating that rounding in the oracle alone moves the tiny model's
routed output by 3.3% rel-L2, so the bound is 6e-2."""
import numpy as np
import pytest
import torch

from oracle.model import Oracle, Trace
from oracle.quant import e4m3_decode, quantize_rows
from synth import LAYER, TINY, make_tokens, make_weights

from .gpu_common import MAX_EXCLUDED_NEAR_TIES, ambiguous_tokens, assert_excluded_fraction, np64, rel_l2, to_device
from .helpers import oracle_weights

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

FP8_REL_L2 = 6e-2
BF16_U = 2.0 ** -8  # unit roundoff of bf16 (8 significand bits, round to nearest)


def _decode(codes: torch.Tensor) -> np.ndarray:
    return e4m3_decode(codes.contiguous().cpu().numpy())


def _run_layer(cfg, w, T, device_weights=True):
    import block_diffusion_moe_denoise_b200 as dgm
    wd = to_device(w) if device_weights else w
    h = dgm.DG(cfg, wd, max_requests=1, kv_capacity=512)
    toks = make_tokens(cfg, T, seed=2, name="canvas")
    h.debug_forward(0, toks.cuda(), 1)
    h.sync()
    return h, toks


def _buffers(h, cfg, T):
    d, fe, k = cfg.d_model, cfg.ffn_expert, cfg.top_k
    P = T * k
    B = lambda n, dt, shape: h.debug_buffer(n, dt, shape)
    return dict(
        u=B("u", torch.bfloat16, (h.token_capacity(), d))[:T],
        xq=B("xq", torch.uint8, (P, d)), xs=B("xs", torch.float32, (P,)),
        hp=B("hp", torch.bfloat16, (P, fe)), hq=B("hq", torch.uint8, (P, fe)), hs=B("hsq", torch.float32, (P,)),
        yp=B("yp", torch.bfloat16, (P, d)), row_token=B("row_token", torch.int32, (P,)),
        row_weight=B("row_weight", torch.float32, (P,)), pair_row=B("pair_row", torch.int32, (P,)),
        offsets=B("offsets", torch.int32, (cfg.n_experts + 1,)))


def _check_quant(rows: torch.Tensor, codes: torch.Tensor, scale: torch.Tensor):
    """Codes and scales equal the oracle's per-row E4M3 quantisation
    (oracle.quant.quantize_rows, float32 like the kernel: the scaled values often
    sit exactly on an E4M3 midpoint, so both sides must divide the same way) of
    the kernel's own bf16 rows; a value that rounds to zero may carry either
    sign (the kernel's conversion may drop it), so zeros compare by value."""
    x = rows.float().cpu().numpy()
    ref, ref_scale = quantize_rows(x)
    codes = codes.cpu().numpy()
    same = (codes == ref) | (((codes & 0x7F) == 0) & ((ref & 0x7F) == 0))
    if not bool(same.all()):
        bad = np.argwhere(~same)[:8]
        info = [(int(r), int(c), float(x[r, c]), int(codes[r, c]), int(ref[r, c])) for r, c in bad]
        raise AssertionError(f"{int((~same).sum())} codes differ, e.g. (row, col, value, kernel, oracle): {info}")
    np.testing.assert_array_equal(scale.cpu().numpy(), ref_scale)


def _check_gemms(cfg, lw, b, rows):
    """hp and yp of the sampled grouped rows against float64 products of the
    GEMMs' own codes and scales."""
    off = b["offsets"].cpu().numpy()
    cache = {}

    def weights(e):
        if e not in cache:
            cache[e] = [_decode(lw[n][e]) * lw[n + "_scale"][e].double().cpu().numpy()[:, None]
                        for n in ("w_gate", "w_up", "w_down")]
        return cache[e]

    for r in rows:
        e = int(np.searchsorted(off, r, side="right") - 1)
        Wg, Wu, Wd = weights(e)
        x = _decode(b["xq"][r]) * float(b["xs"][r])
        g, u = Wg @ x, Wu @ x
        hp_ref = g / (1 + np.exp(-g)) * u
        assert rel_l2(np64(b["hp"][r]), hp_ref) < 1e-2, r
        hrow = _decode(b["hq"][r]) * float(b["hs"][r])
        y_ref = float(b["row_weight"][r]) * (Wd @ hrow)
        # the weighted output is stored in bf16: each element within one unit
        # roundoff (2^-8) of the fp32 product, so the row within 2^-8 in L2
        assert rel_l2(np64(b["yp"][r]), y_ref) < BF16_U + 1e-4, r


def test_fp8_tiny_layer():
    cfg = TINY.with_(expert_fp8=1)
    w = make_weights(cfg, seed=0, gain_std=0.1)
    T = 256
    h, toks = _run_layer(cfg, w, T)
    b = _buffers(h, cfg, T)
    P = T * cfg.top_k
    # quantised rows: every grouped row holds its token's codes
    tok = b["row_token"].long()
    _check_quant(b["u"][tok], b["xq"], b["xs"])
    _check_quant(b["hp"], b["hq"], b["hs"])
    # the two FP8 GEMMs
    lw = {k: v.cuda() for k, v in w["layers"][0].items()}
    _check_gemms(cfg, lw, b, range(0, P, 7))
    # routed output against the oracle's FP8 path
    ora = Oracle(cfg, oracle_weights(w))
    tr = Trace()
    ora.forward(toks.numpy(), ora.new_cache(512), want_stats=False, trace=tr, n_layers=1)
    rec = tr.layers[0]
    yp = np64(b["yp"])
    pr = b["pair_row"].cpu().numpy().reshape(T, cfg.top_k)
    y_gpu = np.stack([yp[pr[t]].sum(axis=0) for t in range(T)])
    keep = ~ambiguous_tokens(tr.layers, cfg.top_k)
    assert_excluded_fraction(~keep, MAX_EXCLUDED_NEAR_TIES, "FP8 layer, routing near a tie")
    err = rel_l2(y_gpu[keep], rec["y_routed"][keep])
    assert err < FP8_REL_L2, err
    print(f"FP8 routed output rel-L2 vs oracle: {err:.3e}")
    h.close()


def test_fp8_full_shape_gemms():
    """The full expert shape (d 2816: 22 k-blocks of 128; width 704: 5.5
    k-blocks, the last half read past the row end as zeros) on sampled rows."""
    cfg = LAYER.with_(expert_fp8=1)
    w = make_weights(cfg, seed=0, device="cuda")
    T = 256
    h, _ = _run_layer(cfg, w, T, device_weights=False)
    b = _buffers(h, cfg, T)
    tok = b["row_token"].long()
    sample = torch.arange(0, T * cfg.top_k, 37, device="cuda")
    _check_quant(b["u"][tok[sample]], b["xq"][sample], b["xs"][sample])
    _check_quant(b["hp"][sample], b["hq"][sample], b["hs"][sample])
    _check_gemms(cfg, w["layers"][0], b, sample.tolist())
    h.close()
