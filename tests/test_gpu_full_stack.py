"""GPU vs oracle over the whole 30-layer synthetic stack at the benchmark's
shape: d 2816, 16/8 heads of 256, 128 experts top-8 + shared 2112, vocab
262144, a 4096-token committed KV prefix (synthetic N(0, 1) bf16 keys and
values per layer) and one 256-token canvas, in the launch configuration the
benchmark times (one request, 256 canvas tokens).  Sizes: "DiffusionGemma Hits
1,000 Tokens per Second", section "The speed numbers and the hardware they
require" (128 experts, eight active plus one shared, 25.2B total / 3.8B active
parameters); the 256-token canvas and the 4096-token input: "DiffusionGemma
hits ~1,500 TPS on one H100", section "The specs that matter for serving".

The oracle (fp64) takes the same bf16 weights one layer at a time from the
device tensors and runs the canvas through all 30 layers and the LM head.

Routing over 30 layers.  Top-k routing is discontinuous and 21% of the tokens
of a full-shape layer have their 8th and 9th router logits within 1.5% of the
logits' RMS, so over 30 layers nearly every token passes some near-tie, and
the GPU (bf16 GEMM inputs) takes the other side of some of them.  Excluding
every near-tie token would leave nothing to compare.  Instead the test reads
the GPU's routing at every layer (a debug pass stopped after layer l leaves
layer l's routing and residual stream in the workspace) and requires that the
GPU leaves the oracle's routing only at near-ties (tests/gpu_common.py,
routing_divergence); every other difference fails.  Values are compared on
the tokens that have not diverged up to the compared layer, and the number
that have is bounded from below and printed (the exclusions counted)."""
import numpy as np
import pytest
import torch

from oracle import sampler as OS
from oracle.model import Oracle, Trace
from synth import FULL, make_kv_prefix, make_weights, to_f64

from .gpu_common import (LOGIT_MAX_ABS, PAGE_MARGIN, REL_L2, STRICT_MARGIN, np64, rel_l2,
                         routing_divergence)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

CFG = FULL
L_PREFIX = 4096
SEED, BLOCK = 2, 0
# Lower bounds on the tokens still on the oracle's routing: measured 30-layer
# survival is about a fifth of the canvas (per-layer divergence ~5%); these
# floors leave room for seed-to-seed spread while keeping the comparisons
# meaningful (at least 32 rows for the end-to-end statistics).
MIN_ON_TRACK_FINAL = 32


class _SlimLayers(list):
    """Per-layer trace records reduced to what the test compares (the full
    trace of 30 layers would hold ~2 GB)."""
    KEEP = ("router_logits", "idx", "x_out")

    def append(self, rec):
        super().append({k: rec[k] for k in self.KEEP})


@pytest.fixture(scope="module")
def run():
    import block_diffusion_moe_denoise_b200 as dgm
    w = make_weights(CFG, seed=0, device="cuda")
    T, d, k = CFG.canvas, CFG.d_model, CFG.top_k
    h = dgm.DG(CFG, w, max_requests=1, kv_capacity=L_PREFIX + T)
    kvs = []
    for l in range(CFG.n_layers):
        kk, vv = make_kv_prefix(CFG, L_PREFIX, seed=1, device="cuda", layer=l)
        h.set_kv(0, l, 0, kk, vv)
        kvs.append((kk, vv))
    h.set_kv_len(0, L_PREFIX)
    h.open_canvas(0, SEED, BLOCK)
    tok = h.get_canvas(0)[0].clone()
    # the GPU's routing and residual stream after every layer: a pass stopped
    # after layer l folds that layer's expert outputs into "x"
    g_idx, g_x = [], []
    for n in range(1, CFG.n_layers + 1):
        h.debug_forward(0, tok, n)
        g_idx.append(h.debug_buffer("idx", torch.int32, (T, k)).cpu().numpy().copy())
        g_x.append(h.debug_buffer("x", torch.float32, (T, d)).cpu().numpy().astype(np.float64))
    # the last pass is the full one (LM head included)
    dbg_stats = h.debug_buffer("stats", torch.float32, (T, 4)).clone()
    dbg_am = h.debug_buffer("argmax", torch.int32, (T,)).cpu().numpy().copy()
    x_final = h.debug_buffer("x", torch.float32, (T, d)).clone()
    # the public denoising step on the same canvas
    h.denoise_step([0])
    tok1, mask1, stats1, am1 = h.get_canvas(0)
    h.sync()
    step = dict(tok=tok1.cpu().numpy().astype(np.int64), mask=mask1.cpu().numpy().astype(bool),
                stats=stats1.cpu().numpy().astype(np.float64), argmax=am1.cpu().numpy(),
                same_as_debug=bool(torch.equal(stats1, dbg_stats)), remaining=h.read_remaining(0))
    # GPU logits of its own final hidden rows (same LM-head kernels, logits written)
    _, _, g_logits = h.op_lm_head(x_final, want_logits=True)
    h.sync()
    h.close()

    ora_w = {"embed": to_f64(w["embed"]), "final_norm": to_f64(w["final_norm"]),
             "layers": lambda l: {n: to_f64(t) for n, t in w["layers"][l].items()}}
    ora = Oracle(CFG, ora_w)
    cache = ora.new_cache(L_PREFIX + T)
    for l, (kk, vv) in enumerate(kvs):
        cache.K[l][:, :L_PREFIX] = to_f64(kk)
        cache.V[l][:, :L_PREFIX] = to_f64(vv)
    cache.length = L_PREFIX
    tr = Trace()
    tr.layers = _SlimLayers()
    canvas = tok.cpu().numpy().astype(np.int64)
    st = ora.forward(canvas, cache, want_stats=True, trace=tr)
    first = routing_divergence(g_idx, [r["router_logits"] for r in tr.layers], [r["idx"] for r in tr.layers], k)
    out = dict(canvas=canvas, g_idx=g_idx, g_x=g_x, dbg_stats=dbg_stats.cpu().numpy().astype(np.float64),
               dbg_am=dbg_am, step=step, g_logits=g_logits, ora=st, tr=tr.layers, first=first)
    yield out
    del w


def test_routing_leaves_the_oracle_only_at_near_ties(run):
    """routing_divergence (in the fixture) already failed on any divergence that
    is not a near-tie; here the survival over depth is bounded and printed."""
    first = run["first"]
    T = first.shape[0]
    alive = [int((first > l).sum()) for l in range(CFG.n_layers)]
    print(f"30 layers: tokens on the oracle's routing after layers 1, 5, 10, 20, 30: "
          f"{alive[0]}, {alive[4]}, {alive[9]}, {alive[19]}, {alive[29]} of {T}")
    per_layer = [(int((first == l).sum()) / max(1, int((first >= l).sum()))) for l in range(CFG.n_layers)]
    print("per-layer divergence rate: " + " ".join(f"{p:.3f}" for p in per_layer))
    assert max(per_layer) <= 0.15, per_layer
    assert alive[-1] >= MIN_ON_TRACK_FINAL, alive


def test_residual_stream_every_layer(run):
    """After every layer, the residual stream of the tokens still on the
    oracle's routing within the bf16 bound (relative L2 1e-2)."""
    errs = []
    for l in range(CFG.n_layers):
        keep = run["first"] > l
        errs.append(rel_l2(run["g_x"][l][keep], run["tr"][l]["x_out"][keep]))
    print("30 layers: residual-stream rel-L2 after each layer: " + " ".join(f"{e:.2e}" for e in errs))
    assert max(errs) < REL_L2, errs


def test_lm_statistics_after_30_layers(run):
    """LM-head statistics of the full pass (logits never written) on every token
    that stayed on the oracle's routing: max logit and log-partition within the
    logit bound, entropy within the relative bound; argmax equal wherever the
    oracle's top-1 margin exceeds twice the logit bound, and at a rate >= 95%
    where it exceeds 1e-2."""
    keep = run["first"] == CFG.n_layers
    g, o = run["dbg_stats"], run["ora"]
    e_max = np.max(np.abs(g[keep, 2] - o["max"][keep]))
    e_lz = np.max(np.abs(g[keep, 3] - o["logZ"][keep]))
    e_h = rel_l2(g[keep, 0], o["entropy"][keep])
    z = o["logits"]
    srt = np.partition(z, -2, axis=1)[:, -2:]
    margin = srt[:, 1] - srt[:, 0]
    strict = keep & (margin > STRICT_MARGIN)
    counted = keep & (margin > PAGE_MARGIN)
    agree = run["dbg_am"] == o["argmax"]
    print(f"30 layers: {int(keep.sum())} tokens on track; max-logit err {e_max:.2e}, logZ err {e_lz:.2e}, "
          f"entropy rel-L2 {e_h:.2e}; argmax {int(agree[counted].sum())}/{int(counted.sum())} at margin > 1e-2")
    assert e_max < LOGIT_MAX_ABS and e_lz < LOGIT_MAX_ABS and e_h < REL_L2
    np.testing.assert_array_equal(run["dbg_am"][strict], o["argmax"][strict])
    assert agree[counted].mean() >= 0.95


def test_logits_after_30_layers_sampled_rows(run):
    """The full logits (262,144 per row) of 32 sampled on-track tokens: max-abs
    error <= 5e-2 and relative L2 <= 1e-2 against the oracle's."""
    keep = np.nonzero(run["first"] == CFG.n_layers)[0]
    rows = np.random.default_rng(0).choice(keep, min(32, keep.size), replace=False)
    got = run["g_logits"][torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
    ref = run["ora"]["logits"][rows]
    ea, er = float(np.max(np.abs(got - ref))), rel_l2(got, ref)
    print(f"30 layers: logits of {rows.size} rows: max-abs {ea:.2e}, rel-L2 {er:.2e}")
    assert ea < LOGIT_MAX_ABS and er < REL_L2


def test_public_step_and_accept_decisions(run):
    """dg_denoise_step reproduces the debug pass bit for bit and applies the rule;
    its accept decisions equal the oracle's (the oracle's rule on the oracle's
    statistics) on every position whose decision is not within 1e-2 of a
    boundary (top-1 margin, the rank-22 confidence cut, the entropy threshold)
    and whose routing stayed on the oracle's; over all such positions
    including diverged ones the agreement rate is reported and bounded.
    Positions rejected on both sides carry the same Philox re-noise token."""
    s, o = run["step"], run["ora"]
    assert s["same_as_debug"] and s["remaining"] == CFG.canvas - CFG.min_accept
    acc0 = np.zeros(CFG.canvas, dtype=bool)
    c_o, a_o, rem_o = OS.sample_step(run["canvas"], acc0, o["argmax"], o["entropy"], o["logconf"], seed=SEED,
                                     block=BLOCK, step=1, vocab=CFG.vocab, entropy_thresh=CFG.entropy_thresh,
                                     min_accept=CFG.min_accept, max_steps=CFG.max_steps)
    assert rem_o == s["remaining"]
    lc = o["logconf"]
    cut = np.sort(lc)[::-1][CFG.min_accept - 1]
    z = o["logits"]
    srt = np.partition(z, -2, axis=1)[:, -2:]
    margin = srt[:, 1] - srt[:, 0]
    counted = (margin > PAGE_MARGIN) & (np.abs(lc - cut) > PAGE_MARGIN) & (np.abs(o["entropy"] - 1.0) > PAGE_MARGIN)
    on_track = run["first"] == CFG.n_layers
    strict = counted & on_track
    np.testing.assert_array_equal(s["mask"][strict], a_o[strict])
    both = s["mask"] & a_o & strict
    np.testing.assert_array_equal(s["tok"][both], c_o[both])
    rej = ~s["mask"] & ~a_o
    np.testing.assert_array_equal(s["tok"][rej], c_o[rej])
    rate = float((s["mask"] == a_o)[counted].mean())
    print(f"30 layers, step 1: {int(counted.sum())} counted decisions ({int(strict.sum())} on track), "
          f"{CFG.canvas - int(counted.sum())} excluded near a boundary; agreement {rate:.3f}")
    assert rate >= 0.95
