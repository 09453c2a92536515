"""Bit-exact parity of the integer / selection kernels against the oracle, on
identical fp32 inputs: Philox re-noise draws, router top-k, expert grouping,
canvas initialisation and the accept / re-noise rule."""
import numpy as np
import pytest
import torch

from oracle import layers as OL
from oracle import philox as OP
from oracle import sampler as OS
from synth import TINY, make_weights

from .gpu_common import to_device

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def dgmod():
    import block_diffusion_moe_denoise_b200 as dgm
    return dgm


@pytest.fixture(scope="module")
def tiny_handle(dgmod):
    w = to_device(make_weights(TINY, seed=0))
    h = dgmod.DG(TINY, w, max_requests=4, kv_capacity=1024)
    yield h
    h.close()


@pytest.mark.parametrize("seed,block,step,req_id,vocab", [
    (0, 0, 0, 0, 2048), (1234, 3, 12, 0, 262144), (2**40 + 7, 1, 5, 3, 262144), (99, 2, 1, 1, 1000)])
def test_philox_tokens_bitwise(dgmod, seed, block, step, req_id, vocab):
    n = 1_000_000 if vocab == 262144 and seed == 1234 else 65536
    out = torch.empty(n, dtype=torch.int32, device="cuda")
    dgmod.philox_tokens(seed, block, step, req_id, 0, n, vocab, out)
    torch.cuda.synchronize()
    ref = OP.renoise_tokens(seed, block, step, np.arange(n), vocab, req_id)
    np.testing.assert_array_equal(out.cpu().numpy(), ref)


def test_route_topk_bitwise(dgmod):
    rng = np.random.default_rng(0)
    for T, E, k in ((256, 128, 8), (1024, 128, 8), (37, 16, 2), (5, 256, 8)):
        logits = rng.normal(size=(T, E)).astype(np.float32)
        logits[: T // 4, : E // 2] = np.round(logits[: T // 4, : E // 2], 1)   # many exact ties
        logits[0, :] = 0.5                                                    # all tied
        d = torch.from_numpy(logits).cuda()
        idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, k), dtype=torch.float32, device="cuda")
        dgmod.route_topk(d, k, idx, w)
        torch.cuda.synchronize()
        ridx, rw = OL.route(logits.astype(np.float64), k)
        np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
        np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=2e-6, atol=1e-7)


def test_route_group_bitwise(tiny_handle):
    rng = np.random.default_rng(1)
    E, k = TINY.n_experts, TINY.top_k
    for T in (256, 1024, 1, 77):
        logits = rng.normal(size=(T, E))
        if T == 77:
            logits[:, 3] += 10.0                     # one expert takes every token
        idx, w = OL.route(logits, k)
        counts, offsets, perm = tiny_handle.op_route_group(
            torch.from_numpy(idx.astype(np.int32)).cuda(), torch.from_numpy(w.astype(np.float32)).cuda())
        torch.cuda.synchronize()
        rc, ro, rp, _ = OL.histogram_and_permutation(idx, E)
        np.testing.assert_array_equal(counts.cpu().numpy(), rc)
        np.testing.assert_array_equal(offsets.cpu().numpy(), ro)
        np.testing.assert_array_equal(perm.cpu().numpy(), rp)
        tiny_handle.sync()


def test_open_canvas_bitwise(tiny_handle):
    tiny_handle.open_canvas(2, 1234, 3)
    tok, mask, _, _ = tiny_handle.get_canvas(2)
    torch.cuda.synchronize()
    ref, racc = OS.init_canvas(TINY.canvas, seed=1234, block=3, vocab=TINY.vocab, request=2)
    np.testing.assert_array_equal(tok.cpu().numpy(), ref)
    assert not mask.cpu().numpy().any() and not racc.any()


def _rand_stats(rng, n, vocab, low_entropy=0):
    H = rng.uniform(2.0, 8.0, size=n).astype(np.float32)
    if low_entropy:
        H[rng.choice(n, low_entropy, replace=False)] = rng.uniform(0.0, 1.0, size=low_entropy)
        H[0] = np.float32(1.0)                                    # exactly at the threshold
    lc = np.round(rng.normal(-5.0, 0.3, size=n), 2).astype(np.float32)   # ties in logconf
    am = rng.integers(0, vocab, size=n).astype(np.int32)
    return H, lc, am


@pytest.mark.parametrize("low_entropy", [0, 30])
def test_sampler_bitwise_full_canvas(tiny_handle, low_entropy):
    """Twelve steps of the rule from identical fp32 statistics: canvas, mask and
    remaining match the oracle exactly, and the canvas converges."""
    C, V = TINY.canvas, TINY.vocab
    req, seed = 1, 77 + low_entropy
    tiny_handle.open_canvas(req, seed, 0)
    canvas, acc = OS.init_canvas(C, seed=seed, block=0, vocab=V, request=req)
    rng = np.random.default_rng(2 + low_entropy)
    for step in range(1, TINY.max_steps + 1):
        H, lc, am = _rand_stats(rng, C, V, low_entropy if step == 1 else 0)
        tiny_handle.op_sample(req, torch.from_numpy(H).cuda(), torch.from_numpy(lc).cuda(),
                              torch.from_numpy(am).cuda(), step)
        canvas, acc, rem = OS.sample_step(canvas, acc, am, H.astype(np.float64), lc.astype(np.float64), seed=seed,
                                          block=0, step=step, vocab=V, entropy_thresh=TINY.entropy_thresh,
                                          min_accept=TINY.min_accept, max_steps=TINY.max_steps, request=req)
        tok, mask, _, _ = tiny_handle.get_canvas(req)
        np.testing.assert_array_equal(tok.cpu().numpy(), canvas)
        np.testing.assert_array_equal(mask.cpu().numpy().astype(bool), acc)
        assert tiny_handle.read_remaining(req) == rem
        if rem == 0:
            break
    assert rem == 0
    tiny_handle.sync()


def test_sampler_step_cap_forces_acceptance(tiny_handle):
    C, V = TINY.canvas, TINY.vocab
    req = 3
    tiny_handle.open_canvas(req, 5, 1)
    rng = np.random.default_rng(9)
    H, lc, am = _rand_stats(rng, C, V)
    tiny_handle.op_sample(req, torch.from_numpy(H).cuda(), torch.from_numpy(lc).cuda(), torch.from_numpy(am).cuda(),
                          TINY.max_steps)
    tok, mask, _, _ = tiny_handle.get_canvas(req)
    assert mask.cpu().numpy().all() and tiny_handle.read_remaining(req) == 0
    np.testing.assert_array_equal(tok.cpu().numpy(), am)


@pytest.fixture(scope="module")
def budget_handle(dgmod):
    w = to_device(make_weights(TINY, seed=0))
    h = dgmod.DG(TINY.with_(sampler=1), w, max_requests=2, kv_capacity=1024)
    yield h
    h.close()


@pytest.mark.parametrize("case", ["budget", "converge"])
def test_entropy_budget_sampler_bitwise(budget_handle, case):
    """The pages' entropy-budget rule from identical fp32 statistics: canvas,
    mask and remaining match the oracle exactly at every step.  "budget": small
    entropies spread so the running sum crosses 0.1 mid-canvas; "converge": the
    argmax repeats with tiny entropies from step 3, so the canvas converges."""
    C, V = TINY.canvas, TINY.vocab
    req, seed = 1, 5 if case == "budget" else 6
    budget_handle.open_canvas(req, seed, 0)
    canvas, acc = OS.init_canvas(C, seed=seed, block=0, vocab=V, request=req)
    rng = np.random.default_rng(17 if case == "budget" else 18)
    am_fixed = rng.integers(0, V, size=C).astype(np.int32)
    prev = None
    for step in range(1, TINY.max_steps + 1):
        if case == "budget":
            H = rng.choice([0.0, 0.004, 0.01, 0.03, 2.0], size=C).astype(np.float32)
            am = rng.integers(0, V, size=C).astype(np.int32)
        else:
            H = np.full(C, 1e-4 if step >= 3 else 0.5, dtype=np.float32)
            am = am_fixed
        lc = np.round(rng.normal(-5.0, 0.3, size=C), 2).astype(np.float32)
        budget_handle.op_sample(req, torch.from_numpy(H).cuda(), torch.from_numpy(lc).cuda(),
                                torch.from_numpy(am).cuda(), step)
        canvas, acc, rem = OS.sample_step(canvas, acc, am, H.astype(np.float64), lc.astype(np.float64), seed=seed,
                                          block=0, step=step, vocab=V, entropy_thresh=TINY.entropy_thresh,
                                          min_accept=TINY.min_accept, max_steps=TINY.max_steps, request=req,
                                          rule="budget", entropy_budget=0.1, stop_entropy=0.005, prev_argmax=prev)
        prev = am
        tok, mask, _, _ = budget_handle.get_canvas(req)
        np.testing.assert_array_equal(tok.cpu().numpy(), canvas)
        np.testing.assert_array_equal(mask.cpu().numpy().astype(bool), acc)
        assert budget_handle.read_remaining(req) == rem
        if rem == 0:
            break
    if case == "converge":
        assert step == 3 and rem == 0
    budget_handle.sync()


# ---- candidate draw at a temperature (LM-head epilogue + combine) ---------------------------

def _exact_lm_inputs(V, d, T, nz_inv, seed):
    """Inputs whose logits every summation order computes exactly: embedding rows
    with entries in {-1/4, 0, 1/4} (nonzero with probability 1/nz_inv) and hidden
    rows of +-1 (the final RMSNorm with unit gain maps them to +-1 after bf16
    rounding), so z = sum of +-1/4 terms is exact in fp32 and fp64 alike."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    sign = torch.randint(0, 2, (V, d), generator=g, device="cuda", dtype=torch.int8) * 2 - 1
    keep = torch.randint(0, nz_inv, (V, d), generator=g, device="cuda", dtype=torch.int16) == 0
    E = (sign * keep).to(torch.bfloat16) * 0.25
    x = (torch.randint(0, 2, (T, d), generator=g, device="cuda", dtype=torch.int8) * 2 - 1).to(torch.float32)
    return E, x


def _oracle_draw(E, x, rows, eps, tau, seed, block, step, request):
    """Oracle logits (fp64, in vocabulary chunks) and the oracle's candidate draw for `rows`."""
    xn = OL.rms_norm(x[rows].cpu().double().numpy(), np.ones(x.shape[1]), eps)
    V = E.shape[0]
    z = np.empty((len(rows), V))
    for v0 in range(0, V, 32768):
        z[:, v0:v0 + 32768] = xn @ E[v0:v0 + 32768].to(torch.float32).cpu().double().numpy().T
    u_row, u_tile = OS.candidate_uniforms(seed, block, step, np.asarray(rows), V // OS.DRAW_TILE, request)
    return OS.draw_candidates(z, tau, u_row, u_tile), z


def _assert_argmax_lowest_tied(am, z):
    """The logits here take few distinct values (multiples of 1/4), so the maximum
    is often shared; the kernel takes the lowest id among the ids within 1e-6 of
    it (fp64 rounding of the oracle's sums only separates exact ties)."""
    for r in range(z.shape[0]):
        tied = np.nonzero(z[r] >= z[r].max() - 1e-6)[0]
        assert am[r] == tied.min(), (r, am[r], tied[:8])


def test_lm_sample_bitwise_on_exact_logits(dgmod):
    """Drawn candidates equal the oracle's draw for every row whose targets lie
    more than 3e-5 (relative) from an interval edge: the logits are exact on
    both sides, so only float32 sums of the draw itself differ from fp64.  The
    statistics and argmax equal those of the plain LM-head entry point."""
    cfg = TINY.with_(n_layers=1, d_model=512, vocab=32768)
    w = to_device(make_weights(cfg, seed=0))
    E, x = _exact_lm_inputs(cfg.vocab, cfg.d_model, cfg.canvas, 8, seed=41)
    w["embed"] = E
    h = dgmod.DG(cfg, w, max_requests=2, kv_capacity=1024)
    tau, seed, block, step, req = 0.7, 2**33 + 17, 2, 3, 1
    stats, am, cand = h.op_lm_sample(x, tau, seed, block, step, req)
    stats0, am0, _ = h.op_lm_head(x)
    h.sync()
    assert torch.equal(stats, stats0) and torch.equal(am, am0)
    rows = list(range(cfg.canvas))
    (c_o, margin), z = _oracle_draw(E, x, rows, cfg.norm_eps, tau, seed, block, step, req)
    sel = margin > 3e-5
    assert sel.sum() >= 0.85 * len(rows), sel.sum()
    np.testing.assert_array_equal(cand.cpu().numpy()[sel], c_o[sel])
    assert (cand.cpu().numpy() != am.cpu().numpy()).sum() > 20      # the draw is not the argmax
    _assert_argmax_lowest_tied(am.cpu().numpy(), z)
    h.close()


# ---- self-conditioning term -------------------------------------------------------------------

def _exact_z(E, x, rows, eps):
    """Oracle logits of the exact-logit inputs with their ties intact: the normed
    rows are +-m (one magnitude m), so z = m/4 * (signs @ 4E^T), an integer
    matrix product that fp64 computes exactly in any summation order."""
    xn = OL.rms_norm(x[rows].cpu().double().numpy(), np.ones(x.shape[1]), eps)
    m = np.abs(xn[0, 0])
    assert np.all(np.abs(xn) == m)
    V = E.shape[0]
    z = np.empty((len(rows), V))
    for v0 in range(0, V, 32768):
        E4 = (E[v0:v0 + 32768].to(torch.float32) * 4).cpu().double().numpy()
        z[:, v0:v0 + 32768] = np.sign(xn) @ E4.T
    return z * (m / 4)


def _oracle_selfcond(z, E, w, k):
    """The oracle's self-conditioning term of logits z, reading only the embedding
    rows the top-k entries name."""
    p, ids = OL.topk_probs(z, k)
    uniq = np.unique(ids)
    E_sub = E[torch.from_numpy(uniq).to(E.device)].to(torch.float32).cpu().double().numpy()
    e = OL.soft_embedding(p, np.searchsorted(uniq, ids), E_sub)
    f64 = lambda t: t.to(torch.float32).cpu().double().numpy()
    return p, ids, OL.swiglu(e, f64(w["sc_gate"]), f64(w["sc_up"]), f64(w["sc_down"]))


def test_selfcond_op_on_exact_logits(dgmod):
    """The self-conditioning term from hidden rows: the top-8 ids equal the
    oracle's exactly (exact logits, ties to the lower id), their probabilities to
    float32 rounding, and the term itself within the bf16 tolerance (the soft
    embedding and the MLP's hidden rows are bf16 GEMM inputs)."""
    from .gpu_common import REL_L2, rel_l2
    cfg = TINY.with_(n_layers=1, d_model=512, vocab=32768, ffn_selfcond=256, selfcond_topk=8)
    w = to_device(make_weights(cfg, seed=0))
    E, x = _exact_lm_inputs(cfg.vocab, cfg.d_model, cfg.canvas, 8, seed=47)
    w["embed"] = E
    h = dgmod.DG(cfg, w, max_requests=2, kv_capacity=1024)
    sc, p, ids = h.op_selfcond(1, x)
    h.sync()
    rows = list(range(cfg.canvas))
    z = _exact_z(E, x, rows, cfg.norm_eps)
    p_o, ids_o, sc_o = _oracle_selfcond(z, E, w, cfg.selfcond_topk)
    np.testing.assert_array_equal(ids.cpu().numpy(), ids_o)
    np.testing.assert_allclose(p.cpu().numpy(), p_o, rtol=1e-4)
    assert rel_l2(sc.cpu().double().numpy(), sc_o) < REL_L2
    # the state of request 1 now holds these entries
    top = h.debug_buffer("sc_top", torch.float32, (2, cfg.canvas, 8, 2))[1]
    assert torch.equal(top[..., 0], p)
    h.close()
