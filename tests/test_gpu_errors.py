"""Failure detection on the GPU without a fault: host-made bad inputs that the
kernels already handle in bounds (an out-of-range token id is clamped, a NaN
row propagates to non-finite statistics) set the device error word, dg_sync
reports DG_E_DEVICE once and clears it, and the same handle then computes
clean results bit-identical to a handle that never saw the bad input."""
import numpy as np
import pytest
import torch

from synth import TINY, make_tokens, make_weights

from .gpu_common import to_device

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

CFG = TINY
DG_E_DEVICE = -5


@pytest.fixture(scope="module")
def wd():
    return to_device(make_weights(CFG, seed=0, gain_std=0.1))


def _clean_step(h, prompt):
    h.prefill(0, prompt)
    h.open_canvas(0, 11, 0)
    h.denoise_step([0])
    tok, mask, stats, am = h.get_canvas(0)
    h.sync()
    return tok.clone(), mask.clone(), stats.clone(), am.clone()


def test_bad_prompt_id_sets_error_word_and_handle_recovers(wd):
    import block_diffusion_moe_denoise_b200 as dgm
    from block_diffusion_moe_denoise_b200._ffi import DGError
    prompt = make_tokens(CFG, 128, seed=3).cuda()
    ref = dgm.DG(CFG, wd, max_requests=1, kv_capacity=512)
    want = _clean_step(ref, prompt)
    ref.close()

    h = dgm.DG(CFG, wd, max_requests=1, kv_capacity=512)
    bad = prompt.clone()
    bad[17] = CFG.vocab            # one past the last id: clamped in the kernel, flagged
    bad[90] = -1
    h.prefill(0, bad)
    with pytest.raises(DGError) as ei:
        h.sync()
    assert ei.value.code == DG_E_DEVICE
    h.sync()                       # the word was cleared by the failing sync
    h.set_kv_len(0, 0)             # drop the poisoned prefix; same handle, same workspace
    got = _clean_step(h, prompt)
    for a, b in zip(got, want):
        assert torch.equal(a, b)
    h.close()


def test_nan_hidden_row_sets_error_word_and_handle_recovers(wd):
    import block_diffusion_moe_denoise_b200 as dgm
    from block_diffusion_moe_denoise_b200._ffi import DGError
    h = dgm.DG(CFG, wd, max_requests=1, kv_capacity=512)
    rng = np.random.default_rng(0)
    x = torch.from_numpy(rng.normal(size=(64, CFG.d_model)).astype(np.float32)).cuda()
    st0, am0, _ = h.op_lm_head(x)
    h.sync()
    st0, am0 = st0.clone(), am0.clone()
    xn = x.clone()
    xn[5, 7] = float("nan")
    st1, am1, _ = h.op_lm_head(xn)
    with pytest.raises(DGError) as ei:
        h.sync()
    assert ei.value.code == DG_E_DEVICE
    assert not torch.isfinite(st1[5]).all()
    others = torch.ones(64, dtype=torch.bool, device="cuda")
    others[5] = False
    assert torch.equal(st1[others], st0[others]) and torch.equal(am1[others], am0[others])
    st2, am2, _ = h.op_lm_head(x)
    h.sync()                       # clean again
    assert torch.equal(st2, st0) and torch.equal(am2, am0)
    h.close()
