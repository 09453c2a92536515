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
