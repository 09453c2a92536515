"""Pins of the oracle's accept / freeze / re-noise rule (no GPU)."""
import itertools

import numpy as np
import pytest

from oracle import sampler as S
from oracle.philox import renoise_tokens


def _brute_accept(H, lc, acc, thr, k):
    """Definition restated: i in U is taken iff H_i <= thr, or fewer than
    min(k, |U|) members of U beat it in (logconf desc, position asc)."""
    U = [i for i in range(len(H)) if not acc[i]]
    n_top = min(k, len(U))
    out = np.zeros(len(H), dtype=bool)
    for i in U:
        better = sum(1 for j in U if (lc[j] > lc[i]) or (lc[j] == lc[i] and j < i))
        out[i] = H[i] <= thr or better < n_top
    return out


def test_exhaustive_small_canvases():
    rng = np.random.default_rng(0)
    levels = np.array([-3.0, -1.0, -1.0, 0.0])          # repeated values force ties
    n = 6
    for acc_bits in range(1 << n):
        acc = np.array([(acc_bits >> i) & 1 for i in range(n)], dtype=bool)
        for _ in range(6):
            lc = rng.choice(levels, size=n)
            H = rng.choice([0.5, 1.0, 1.5, 3.0], size=n)
            got = S.accept_set(H, lc, acc, 1.0, 2)
            np.testing.assert_array_equal(got, _brute_accept(H, lc, acc, 1.0, 2))


def test_all_permutations_of_distinct_scores():
    for perm in itertools.permutations(range(5)):
        lc = np.array(perm, dtype=np.float64)
        H = np.full(5, 9.0)
        got = S.accept_set(H, lc, np.zeros(5, bool), 1.0, 2)
        assert set(np.nonzero(got)[0]) == {perm.index(4), perm.index(3)}


def test_frozen_tokens_stay_and_min_accept():
    rng = np.random.default_rng(1)
    n, V = 256, 2048
    canvas, acc = S.init_canvas(n, seed=5, block=0, vocab=V)
    np.testing.assert_array_equal(canvas, renoise_tokens(5, 0, 0, np.arange(n), V))
    prev_rem = n
    for step in range(1, 13):
        frozen = canvas[acc].copy()
        H = rng.uniform(5, 8, size=n)                  # entropy clause never fires
        lc = rng.normal(size=n)
        am = rng.integers(0, V, size=n)
        before = acc.copy()
        canvas, acc, rem = S.sample_step(canvas, acc, am, H, lc, seed=5, block=0, step=step, vocab=V,
                                         entropy_thresh=1.0, min_accept=22, max_steps=12)
        np.testing.assert_array_equal(canvas[before], frozen)          # frozen stay frozen
        newly = acc & ~before
        assert newly.sum() == min(22, prev_rem)
        np.testing.assert_array_equal(canvas[newly], am[newly])
        rej = ~acc
        np.testing.assert_array_equal(canvas[rej], renoise_tokens(5, 0, step, np.nonzero(rej)[0], V))
        assert rem == rej.sum()
        prev_rem = rem
        if rem == 0:
            break
    assert step == 12 and rem == 0                    # 11 * 22 + 14 = 256


def test_entropy_clause_and_step_cap():
    n, V = 40, 64
    canvas, acc = S.init_canvas(n, seed=1, block=0, vocab=V)
    H = np.full(n, 4.0)
    H[[3, 30, 31]] = [1.0, 0.2, 1.0000001]
    lc = -np.arange(n, dtype=np.float64)              # position 0 most confident
    am = np.arange(n) % V
    c2, a2, rem = S.sample_step(canvas, acc, am, H, lc, seed=1, block=0, step=1, vocab=V,
                                entropy_thresh=1.0, min_accept=5, max_steps=12)
    assert set(np.nonzero(a2)[0]) == {0, 1, 2, 3, 4, 30}
    assert rem == n - 6
    # at the cap everything left is accepted
    c3, a3, rem3 = S.sample_step(c2, a2, am, H, lc, seed=1, block=0, step=12, vocab=V,
                                 entropy_thresh=1.0, min_accept=5, max_steps=12)
    assert rem3 == 0 and a3.all()
    np.testing.assert_array_equal(c3[~a2], am[~a2])
    np.testing.assert_array_equal(c3[a2], c2[a2])


def test_min_accept_larger_than_remaining():
    acc = np.ones(10, bool)
    acc[[2, 7]] = False
    got = S.accept_set(np.full(10, 5.0), np.zeros(10), acc, 1.0, 22)
    assert set(np.nonzero(got)[0]) == {2, 7}


# --- entropy-budget rule ----------------------------------------------------

def _budget_brute(H, lc, acc, budget):
    """The budget rule restated as a search: the largest k such that the k most
    confident open positions have total entropy (accumulated one by one)
    within the budget at every prefix past the first; at least one."""
    U = [i for i in range(len(H)) if not acc[i]]
    order = sorted(U, key=lambda i: (-lc[i], i))
    b = float(np.float32(budget))
    best = 1 if order else 0
    for k in range(2, len(order) + 1):
        prefix_ok = True
        s = 0.0
        for r in range(k):
            s += float(H[order[r]])
            if r > 0 and s > b:
                prefix_ok = False
        if prefix_ok:
            best = k
    A = np.zeros(len(H), dtype=bool)
    A[order[:best]] = True
    return A


def test_budget_rule_against_search():
    rng = np.random.default_rng(11)
    for trial in range(400):
        n = int(rng.integers(1, 9))
        H = rng.choice([0.0, 0.01, 0.02, 0.05, 0.08, 0.3], size=n)
        lc = rng.choice([-1.0, -0.5, -0.2], size=n)         # ties
        acc = rng.random(n) < 0.3
        budget = float(rng.choice([0.0, 0.05, 0.1, 0.2]))
        got = S.accept_set_budget(H, lc, acc, np.zeros(n, int), None, budget, 0.005)
        np.testing.assert_array_equal(got, _budget_brute(H, lc, acc, budget), err_msg=f"trial {trial}")
        if (~acc).any():
            assert got[~acc].sum() >= 1          # progress every step
        assert not (got & acc).any()             # frozen positions stay out


def test_budget_rule_zero_budget_takes_one_per_step():
    """Entropies above a zero budget: exactly one position (the most confident)
    per step, so a canvas of n takes n steps unless the cap comes first."""
    n, V = 10, 50
    H = np.full(n, 2.0)
    lc = -np.arange(n, dtype=float) * 0.1
    canvas, acc = S.init_canvas(n, seed=3, block=0, vocab=V)
    am = np.arange(n)
    for step in range(1, n + 1):
        canvas, acc, rem = S.sample_step(canvas, acc, am, H, lc, seed=3, block=0, step=step, vocab=V,
                                         entropy_thresh=1.0, min_accept=22, max_steps=100, rule="budget",
                                         entropy_budget=0.0, stop_entropy=0.005)
        assert rem == n - step and acc[:step].all() and not acc[step:].any()


def test_budget_rule_convergence_and_cap():
    n, V = 8, 50
    H = np.full(n, 1e-4)
    lc = np.zeros(n)
    am = np.arange(n) + 5
    acc = np.zeros(n, bool)
    # low mean entropy but no previous step: only the budget applies (all fit: 8e-4 <= 0.1)
    A = S.accept_set_budget(H, lc, acc, am, None, 0.0, 0.005)
    assert A.sum() == 1
    # same argmax as the previous step and mean entropy 1e-4 < 0.005: converged
    A = S.accept_set_budget(H, lc, acc, am, am.copy(), 0.0, 0.005)
    assert A.all()
    # one position changed its argmax: not converged
    prev = am.copy()
    prev[3] += 1
    assert S.accept_set_budget(H, lc, acc, am, prev, 0.0, 0.005).sum() == 1
    # mean entropy at the threshold is not below it
    H2 = np.full(n, float(np.float32(0.005)))
    assert S.accept_set_budget(H2, lc, acc, am, am, 0.0, 0.005).sum() == 1
    # the step cap takes everything
    assert S.accept_set_budget(np.full(n, 9.0), lc, acc, am, None, 0.0, 0.005, force_all=True).all()


# ---- candidate draw at a temperature ------------------------------------------------------

def _brute_two_level(weights, tile, u_row, u_tile):
    """The two-level inverse-CDF pick in exact rational arithmetic on integer weights."""
    from fractions import Fraction
    w = [int(v) for v in weights]
    n_t = len(w) // tile
    masses = [sum(w[j * tile:(j + 1) * tile]) for j in range(n_t)]
    tgt = Fraction(u_row) * sum(masses)
    cum, J = 0, None
    for j, m in enumerate(masses):
        cum += m
        if cum >= tgt:
            J = j
            break
    seg = w[J * tile:(J + 1) * tile]
    tgt2 = Fraction(u_tile[J]) * sum(seg)
    cum = 0
    for i, v in enumerate(seg):
        cum += v
        if cum >= tgt2:
            return J * tile + i
    raise AssertionError("unreachable")


def test_draw_matches_exact_rational_brute_force():
    """Integer weights w_v = exp(z_v / tau): the fp64 draw must pick the id the exact
    rational inverse CDF picks, for every uniform pair away from an interval edge."""
    rng = np.random.default_rng(3)
    tile, V = 4, 16
    for trial in range(300):
        w = rng.integers(1, 9, size=V)
        w[rng.random(V) < 0.2] = rng.integers(20, 40)          # a few heavy ids
        tau = [1.0, 0.5, 2.0][trial % 3]                        # exact in float32
        z = tau * np.log(w.astype(np.float64))
        u_row = S.uniform_from_word(rng.integers(0, 2**32, size=1, dtype=np.uint64))
        u_tile = S.uniform_from_word(rng.integers(0, 2**32, size=(1, V // tile), dtype=np.uint64))
        cand, margin = S.draw_candidates(z[None, :], tau, u_row, u_tile, tile=tile)
        if margin[0] < 1e-9:
            continue
        assert cand[0] == _brute_two_level(w, tile, u_row[0], u_tile[0])


def test_draw_frequencies_follow_the_tempered_softmax():
    """Many independent draws of one row: the id frequencies match softmax(z / tau)
    (chi-square over the ids with an expected count >= 5, the rest lumped)."""
    rng = np.random.default_rng(4)
    V, tau, n = 1024, 0.7, 30000
    z = rng.normal(0.0, 1.5, size=V)
    p = np.exp(z / tau - (z / tau).max())
    p /= p.sum()
    u_row = S.uniform_from_word(rng.integers(0, 2**32, size=n, dtype=np.uint64))
    u_tile = S.uniform_from_word(rng.integers(0, 2**32, size=(n, V // 256), dtype=np.uint64))
    cand, _ = S.draw_candidates(np.broadcast_to(z, (n, V)), tau, u_row, u_tile)
    counts = np.bincount(cand, minlength=V).astype(np.float64)
    exp_c = n * p
    big = exp_c >= 5
    obs = np.append(counts[big], counts[~big].sum())
    ex = np.append(exp_c[big], exp_c[~big].sum())
    chi2 = ((obs - ex) ** 2 / ex).sum()
    dof = obs.size - 1
    assert chi2 < dof + 6 * np.sqrt(2 * dof), (chi2, dof)
    # the tile level alone: four tiles, their masses
    tile_obs = counts.reshape(4, 256).sum(1)
    tile_p = p.reshape(4, 256).sum(1)
    assert np.all(np.abs(tile_obs - n * tile_p) < 5 * np.sqrt(n * tile_p * (1 - tile_p)) + 1)


def test_draw_special_cases():
    # a dominant logit is drawn for any uniforms; a tiny temperature gives the argmax
    z = np.zeros((3, 512))
    z[0, 300] = 80.0
    z[1] = np.linspace(-1, 1, 512)
    z[2] = np.linspace(1, -1, 512)
    u_row = np.array([2.0 ** -24, 0.5, 1 - 2.0 ** -24])
    u_tile = np.tile(np.array([[2.0 ** -24, 1 - 2.0 ** -24]]), (3, 1))
    cand, _ = S.draw_candidates(z, 1.0, u_row, u_tile)
    assert cand[0] == 300
    cand, _ = S.draw_candidates(z, 1e-4, u_row, u_tile)
    np.testing.assert_array_equal(cand, [300, 511, 0])
    # u -> 0 takes the first id of positive mass, u -> 1 the last
    flat = np.zeros((1, 512))
    assert S.draw_candidates(flat, 0.7, np.array([2.0 ** -24]), np.array([[2.0 ** -24, 0.5]]))[0][0] == 0
    assert S.draw_candidates(flat, 0.7, np.array([1 - 2.0 ** -24]), np.array([[0.5, 1 - 2.0 ** -24]]))[0][0] == 511


def test_uniforms_and_their_counters():
    w = np.array([0, 1, 511, 512, 2**31, 2**32 - 1], dtype=np.uint64)
    u = S.uniform_from_word(w)
    np.testing.assert_array_equal(u, [2.0 ** -24, 2.0 ** -24, 2.0 ** -24, 3 * 2.0 ** -24, 0.5 + 2.0 ** -24,
                                      1 - 2.0 ** -24])
    assert np.all(u.astype(np.float32).astype(np.float64) == u)      # exact in float32
    # row uniform = word 1 of the re-noise block, tile j = word 0 at request + 256 (j + 1)
    from oracle.philox import philox4, seed_key
    seed, block, step, req = 0x1234_5678_9ABC, 3, 5, 2
    u_row, u_tile = S.candidate_uniforms(seed, block, step, [0, 7, 255], 3, request=req)
    k = seed_key(seed)
    for i, pos in enumerate([0, 7, 255]):
        assert u_row[i] == S.uniform_from_word(philox4((pos, step, block, req), k, 32, 10)[1])
        for j in range(3):
            assert u_tile[i, j] == S.uniform_from_word(philox4((pos, step, block, req + 256 * (j + 1)), k, 32, 10)[0])


def test_sample_step_writes_candidates():
    n, V = 30, 64
    canvas, acc = S.init_canvas(n, seed=2, block=0, vocab=V)
    H = np.full(n, 9.0)
    lc = -np.arange(n, dtype=np.float64)
    am = np.arange(n) % V
    cand = (np.arange(n) * 7 + 3) % V
    c2, a2, _ = S.sample_step(canvas, acc, am, H, lc, seed=2, block=0, step=1, vocab=V, entropy_thresh=1.0,
                              min_accept=5, max_steps=12, candidates=cand)
    np.testing.assert_array_equal(c2[a2], cand[a2])
