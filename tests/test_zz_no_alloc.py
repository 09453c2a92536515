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

from synth import TINY, make_weights

from .gpu_common import to_device

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
