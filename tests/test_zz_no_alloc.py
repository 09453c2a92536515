"""dg_op_lm_head_noalloc, the LM-head entry point for callers that cannot
allocate device memory (their allocator already owns the free HBM, or a
cudaMalloc's implicit synchronisation is not acceptable), agrees with the
workspace-based dg_op_lm_head on two calls in a row.

Collected last on purpose: the entry point keeps scratch in a library-wide
array, so this file runs after every other test has used the library, and it
also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

from oracle import layers as OL
from synth import TINY, make_weights

from .gpu_common import LOGIT_MAX_ABS, REL_L2, argmax_agreement, rel_l2, to_device

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_noalloc_lm_head_matches_workspace_entry_point():
    import block_diffusion_moe_denoise_b200 as dgm
    cfg = TINY
    w = to_device(make_weights(cfg, seed=0, gain_std=0.1))
    h = dgm.DG(cfg, w, max_requests=1, kv_capacity=512)
    rng = np.random.default_rng(0)
    # two calls in a row with different sizes: the second must not see the first's scratch
    for T in (200, 77):
        x = torch.from_numpy(rng.normal(size=(T, cfg.d_model)).astype(np.float32)).cuda()
        ref_stats, ref_am, _ = h.op_lm_head(x)
        stats = torch.empty((T, 4), dtype=torch.float32, device="cuda")
        am = torch.empty(T, dtype=torch.int32, device="cuda")
        err = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        dgm.lm_head_noalloc(x, w["final_norm"], w["embed"], cfg.norm_eps, stats, am, err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        np.testing.assert_allclose(stats.cpu().numpy(), ref_stats.cpu().numpy(), rtol=1e-6, atol=1e-6)
        np.testing.assert_array_equal(am.cpu().numpy(), ref_am.cpu().numpy())
    h.sync()
    h.close()


def test_noalloc_rejects_sizes_beyond_its_limit():
    import block_diffusion_moe_denoise_b200 as dgm
    from block_diffusion_moe_denoise_b200._ffi import DGError
    cfg = TINY
    x = torch.zeros((257, cfg.d_model), dtype=torch.float32, device="cuda")
    g = torch.ones(cfg.d_model, dtype=torch.float32, device="cuda")
    e = torch.zeros((cfg.vocab, cfg.d_model), dtype=torch.bfloat16, device="cuda")
    stats = torch.empty((257, 4), dtype=torch.float32, device="cuda")
    am = torch.empty(257, dtype=torch.int32, device="cuda")
    with pytest.raises(DGError) as ei:
        dgm.lm_head_noalloc(x, g, e, cfg.norm_eps, stats, am)
    assert ei.value.code == -1


def test_noalloc_at_its_limits_matches_oracle():
    """The documented limits themselves: T = 256 tokens of width d_model = 4096
    fill the array's row region exactly (the padded token count equals the
    maximum).  Two calls in a row (the second on other rows) agree with the
    fp64 oracle's LM-head statistics within the bf16 bounds, and the first is
    reproduced bit for bit when repeated after the second."""
    import block_diffusion_moe_denoise_b200 as dgm
    T, d, V = 256, 4096, 4096
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    embed = (0.02 * torch.randn((V, d), generator=g, device="cuda")).to(torch.bfloat16)
    gain = 1.0 + 0.1 * torch.randn(d, generator=g, device="cuda")
    xs = [torch.randn((T, d), generator=g, device="cuda") for _ in range(2)]
    E64, g64 = embed.double().cpu().numpy(), gain.double().cpu().numpy()
    outs = []
    for x in xs + xs[:1]:
        stats = torch.empty((T, 4), dtype=torch.float32, device="cuda")
        am = torch.empty(T, dtype=torch.int32, device="cuda")
        err = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        dgm.lm_head_noalloc(x, gain, embed, 1e-6, stats, am, err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        outs.append((stats.clone(), am.clone()))
    for x, (stats, am) in zip(xs, outs):
        ref = OL.lm_head_stats(OL.rms_norm(x.double().cpu().numpy(), g64, 1e-6), E64)
        st = stats.cpu().numpy().astype(np.float64)
        assert np.max(np.abs(st[:, 2] - ref["max"])) < LOGIT_MAX_ABS
        assert np.max(np.abs(st[:, 3] - ref["logZ"])) < LOGIT_MAX_ABS
        assert rel_l2(st[:, 0], ref["entropy"]) < REL_L2
        argmax_agreement(am.cpu().numpy(), ref["logits"])
    assert torch.equal(outs[0][0], outs[2][0]) and torch.equal(outs[0][1], outs[2][1])


@pytest.mark.parametrize("d", [4160, 4032 + 32, 200])
def test_noalloc_rejects_widths_beyond_its_limit(d):
    """A row width above DG_NOALLOC_MAX_DMODEL or not a multiple of 64 returns
    DG_E_ARG before any work is enqueued."""
    import block_diffusion_moe_denoise_b200 as dgm
    from block_diffusion_moe_denoise_b200._ffi import DGError
    T, V = 8, 1024
    x = torch.zeros((T, d), dtype=torch.float32, device="cuda")
    g = torch.ones(d, dtype=torch.float32, device="cuda")
    e = torch.zeros((V, d), dtype=torch.bfloat16, device="cuda")
    stats = torch.empty((T, 4), dtype=torch.float32, device="cuda")
    am = torch.empty(T, dtype=torch.int32, device="cuda")
    with pytest.raises(DGError) as ei:
        dgm.lm_head_noalloc(x, g, e, 1e-6, stats, am)
    assert ei.value.code == -1
