"""Pins of the oracle's decoder pass and generation loop by invariants (no GPU)."""
import json
import os

import numpy as np
import pytest

from oracle.model import Oracle
from synth import FULL, TINY, ModelConfig, make_tokens, make_weights

from .helpers import oracle_weights

SMALL = ModelConfig(n_layers=2, d_model=64, n_q_heads=4, n_kv_heads=2, head_dim=16, n_experts=8,
                    top_k=2, ffn_expert=32, ffn_shared=48, vocab=256, canvas=32, min_accept=3,
                    max_steps=12)


@pytest.fixture(scope="module")
def small():
    return Oracle(SMALL, oracle_weights(make_weights(SMALL, seed=1, std=0.15, gain_std=0.1)))


def test_synthetic_dims_reproduce_page_parameter_counts():
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))
    assert FULL.n_experts == g["experts"] and FULL.top_k == g["top_k"] and FULL.canvas == g["canvas"]
    assert abs(FULL.total_params() / 1e9 - g["total_params_b"]) < 0.05
    assert abs(FULL.active_params_per_token() / 1e9 - g["active_params_b"]) < 0.06
    # the pages' own serving numbers are self-consistent: tok/s = canvas / (steps * ms/step)
    steps = g["output_tokens"] / g["h100_tok_s"] / (g["h100_ms_per_step"] * 1e-3)
    assert abs(steps / (g["output_tokens"] / g["canvas"]) - 12.7) < 0.1
    assert abs(g["canvas"] / (steps / (g["output_tokens"] / g["canvas"])) - g["tokens_per_pass"]) < 0.3


def test_canvas_permutation_equivariance_without_rope(small):
    """With RoPE off every canvas position is treated alike: permuting the canvas
    permutes every per-position statistic (bidirectional, unmasked pass)."""
    small.use_rope = False
    try:
        rng = np.random.default_rng(0)
        prompt = rng.integers(0, SMALL.vocab, 40)
        cache = small.new_cache(40 + SMALL.canvas)
        small.prefill(cache, prompt)
        c = rng.integers(0, SMALL.vocab, SMALL.canvas)
        perm = rng.permutation(SMALL.canvas)
        a = small.forward(c, cache)
        b = small.forward(c[perm], cache)
        for key in ("entropy", "logconf", "max", "logZ"):
            np.testing.assert_allclose(b[key], a[key][perm], rtol=1e-11, atol=1e-12)
        np.testing.assert_array_equal(b["argmax"], a["argmax"][perm])
    finally:
        small.use_rope = True


def test_commit_equals_prefill(small):
    rng = np.random.default_rng(1)
    prompt = rng.integers(0, SMALL.vocab, 50)
    block = rng.integers(0, SMALL.vocab, SMALL.canvas)
    c1 = small.new_cache(200)
    small.prefill(c1, prompt)
    c2 = small.new_cache(200)
    small.prefill(c2, prompt)
    small.forward(rng.integers(0, SMALL.vocab, SMALL.canvas), c1)   # a step scribbles the slot
    small.commit(c1, block)
    small.prefill(c2, block)
    assert c1.length == c2.length == 50 + SMALL.canvas
    for l in range(SMALL.n_layers):
        np.testing.assert_array_equal(c1.K[l][:, :c1.length], c2.K[l][:, :c2.length])
        np.testing.assert_array_equal(c1.V[l][:, :c1.length], c2.V[l][:, :c2.length])


def test_prefill_segments_see_earlier_segments(small):
    """Prefill in canvas-sized segments: the first segment's cache does not depend
    on later tokens, the second one does depend on the first."""
    rng = np.random.default_rng(2)
    p = rng.integers(0, SMALL.vocab, 2 * SMALL.canvas)
    q = p.copy()
    q[-1] = (q[-1] + 1) % SMALL.vocab
    q2 = p.copy()
    q2[0] = (q2[0] + 1) % SMALL.vocab
    caches = []
    for toks in (p, q, q2):
        c = small.new_cache(2 * SMALL.canvas)
        small.prefill(c, toks)
        caches.append(c)
    n = SMALL.canvas
    l = SMALL.n_layers - 1
    np.testing.assert_array_equal(caches[0].K[l][:, :n], caches[1].K[l][:, :n])
    assert not np.allclose(caches[0].K[l][:, n:2 * n - 1], caches[2].K[l][:, n:2 * n - 1])


def test_generation_invariants(small):
    rng = np.random.default_rng(3)
    prompt = rng.integers(0, SMALL.vocab, 45)
    out, steps = small.generate(prompt, 2 * SMALL.canvas, seed=77)
    assert out.shape == (2 * SMALL.canvas,)
    assert all(s <= SMALL.max_steps for s in steps)
    assert out.min() >= 0 and out.max() < SMALL.vocab
    out2, steps2 = small.generate(prompt, 2 * SMALL.canvas, seed=77)
    np.testing.assert_array_equal(out, out2)
    assert steps == steps2


def test_tiny_generation_takes_twelve_steps():
    """Random N(0, 0.02) weights give entropies near ln V, far above 1 nat, so
    only the 22-most-confident clause fires: 11 * 22 + 14 = 256 -> 12 steps."""
    w = oracle_weights(make_weights(TINY, seed=0))
    ora = Oracle(TINY, w)
    prompt = make_tokens(TINY, 128, seed=0).numpy()
    cache = ora.new_cache(128 + 256)
    ora.prefill(cache, prompt)
    canvas, acc = ora.open_canvas(seed=0, block=0)
    rems = []
    for s in range(1, 13):
        canvas, acc, rem, st = ora.denoise_step(cache, canvas, acc, seed=0, block=0, step=s)
        assert st["entropy"].min() > 1.0
        rems.append(rem)
        if rem == 0:
            break
    assert rems == [256 - 22 * i for i in range(1, 12)] + [0]


@pytest.mark.parametrize("variant", [dict(temperature=0.7), dict(ffn_selfcond=32, selfcond_topk=4),
                                     dict(expert_fp8=1), dict(sampler=1),
                                     dict(temperature=0.7, ffn_selfcond=32, expert_fp8=1, sampler=1)])
def test_generation_invariants_of_the_variants(variant):
    """Every configuration knob keeps the loop's invariants: deterministic for a
    seed, at most max_steps steps per canvas, ids in range, and frozen tokens stay
    frozen step to step."""
    cfg = SMALL.with_(**variant)
    ora = Oracle(cfg, oracle_weights(make_weights(cfg, seed=1, std=0.15, gain_std=0.1)))
    rng = np.random.default_rng(5)
    prompt = rng.integers(0, cfg.vocab, 45)
    out, steps = ora.generate(prompt, 2 * cfg.canvas, seed=9)
    out2, steps2 = ora.generate(prompt, 2 * cfg.canvas, seed=9)
    np.testing.assert_array_equal(out, out2)
    assert steps == steps2 and all(1 <= s <= cfg.max_steps for s in steps)
    assert out.min() >= 0 and out.max() < cfg.vocab
    # frozen tokens persist through one canvas
    cache = ora.new_cache(45 + cfg.canvas)
    ora.prefill(cache, prompt)
    canvas, acc = ora.open_canvas(seed=9, block=0)
    prev = prev_logits = None
    for s in range(1, cfg.max_steps + 1):
        frozen = canvas[acc].copy()
        before = acc.copy()
        canvas, acc, rem, st = ora.denoise_step(cache, canvas, acc, seed=9, block=0, step=s, prev_argmax=prev,
                                                prev_logits=prev_logits)
        np.testing.assert_array_equal(canvas[before], frozen)
        prev, prev_logits = st["argmax"], st["logits"]
        if rem == 0:
            break
    assert rem == 0
