"""Accept / freeze / re-noise rule of one denoising step.

The pages' loop ([P2] §"How the sampler actually works"): after the
bidirectional pass, take a candidate token at every position, accept positions
from most to least confident, re-randomise the rejected ones for the next
step, and stop when the canvas has converged or at a step cap.  Accepted
tokens stay fixed while the others are drawn again ([P2] §"What DiffusionGemma
is").

Default rule (the workload's sampler rule; the pages' cumulative entropy
budget of 0.1 is the second rule below):
  U = positions not yet accepted;
  A = {i in U : H_i <= entropy_thresh}
      union the min(min_accept, |U|) positions of U with the highest logconf
      (ties to the lower position);
  at the step cap every position of U is accepted;
  i in A:      c_i <- argmax_i, frozen for the rest of the canvas;
  i in U \\ A:  c_i <- tok(seed, block, step, i)  (Philox, see philox.py);
  remaining = |U \\ A|.
Candidates are the argmax (temperature 0), or, with a temperature tau > 0, a
draw from softmax(z / tau) of the position's logits z (the pages' step 2,
"sample a candidate token at every position"; the temperature of their
request example).  The entropy and confidence that order the positions stay
those of softmax(z): the temperature shapes the draw only.  The draw is
two-level over vocabulary tiles of 256 consecutive ids (see
`draw_candidates`), each level an inverse-CDF pick with its own Philox
uniform (see `candidate_uniforms`).

The pages' own default (the entropy-bound sampler of the same section) is the
second rule, `rule="budget"`, read as:
  order U from most to least confident (logconf descending, ties to the lower
  position); accept positions in that order while the running sum of their
  entropies (float64, summed in that order) stays <= entropy_budget, and
  always the first one;
  converged -- every position of U has the same argmax as at the previous step
  and the mean entropy of U (float64, summed in position order) is below
  stop_entropy -- accepts all of U;
  the step cap accepts all of U.
The thresholds are float32 values (the library's configuration type), so they
are rounded to float32 before the float64 comparisons.
"""
from __future__ import annotations

import numpy as np

from .philox import philox4x32_10_np, renoise_tokens, seed_key

DRAW_TILE = 256      # vocabulary ids per tile of the two-level candidate draw


def accept_set(entropy, logconf, accepted, entropy_thresh: float, min_accept: int,
               force_all: bool = False) -> np.ndarray:
    """Boolean mask of positions accepted this step (a subset of the unaccepted ones)."""
    entropy = np.asarray(entropy)
    logconf = np.asarray(logconf)
    accepted = np.asarray(accepted).astype(bool)
    n = entropy.shape[0]
    U = np.nonzero(~accepted)[0]
    A = np.zeros(n, dtype=bool)
    if force_all:
        A[U] = True
        return A
    A[U[entropy[U] <= entropy_thresh]] = True
    n_top = min(min_accept, U.size)
    # sort U by (-logconf, position); python sort keeps exact float comparisons
    order = sorted(U.tolist(), key=lambda i: (-logconf[i], i))
    A[order[:n_top]] = True
    return A


def accept_set_budget(entropy, logconf, accepted, argmax, prev_argmax, entropy_budget: float,
                      stop_entropy: float, force_all: bool = False) -> np.ndarray:
    """Entropy-budget rule: boolean mask of positions accepted this step."""
    entropy = np.asarray(entropy)
    logconf = np.asarray(logconf)
    accepted = np.asarray(accepted).astype(bool)
    argmax = np.asarray(argmax)
    n = entropy.shape[0]
    U = np.nonzero(~accepted)[0]
    A = np.zeros(n, dtype=bool)
    if force_all or U.size == 0:
        A[U] = True
        return A
    budget = float(np.float32(entropy_budget))
    stop = float(np.float32(stop_entropy))
    if prev_argmax is not None and all(int(argmax[i]) == int(prev_argmax[i]) for i in U):
        total = 0.0
        for i in U:                      # position order
            total += float(entropy[i])
        if total / U.size < stop:
            A[U] = True
            return A
    order = sorted(U.tolist(), key=lambda i: (-logconf[i], i))
    running = 0.0
    for r, i in enumerate(order):
        running += float(entropy[i])
        if r > 0 and running > budget:
            break
        A[i] = True
    return A


def uniform_from_word(w):
    """Map a 32-bit word to the odd multiples of 2^-24 in (0, 1): (2 (w >> 9) + 1) / 2^24.
    Exact in float32, never 0 or 1."""
    w = np.asarray(w, dtype=np.uint64)
    return (2.0 * (w >> np.uint64(9)).astype(np.float64) + 1.0) / float(1 << 24)


def candidate_uniforms(seed: int, block: int, step: int, positions, n_tiles: int, request: int = 0):
    """Uniforms of the candidate draw at one step.

    Row level: word 1 of Philox(position, step, block, request) (word 0 of the
    same block is the re-noise token).  Tile j: word 0 of
    Philox(position, step, block, request + 256 (j + 1)).  Returns
    (u_row [n], u_tile [n, n_tiles])."""
    pos = np.asarray(positions, dtype=np.uint64)
    n = pos.shape[0]
    k0, k1 = seed_key(seed)
    st = np.full(n, step, np.uint64)
    bl = np.full(n, block, np.uint64)
    _, w1, _, _ = philox4x32_10_np(pos, st, bl, np.full(n, request, np.uint64), k0, k1)
    u_row = uniform_from_word(w1)
    u_tile = np.empty((n, n_tiles))
    for j in range(n_tiles):
        w0, _, _, _ = philox4x32_10_np(pos, st, bl, np.full(n, request + 256 * (j + 1), np.uint64), k0, k1)
        u_tile[:, j] = uniform_from_word(w0)
    return u_row, u_tile


def _inverse_cdf(w, u):
    """Smallest index i with w_0 + ... + w_i >= u * sum(w), and the distance of
    u * sum(w) to the nearer edge of that index's interval, relative to sum(w)."""
    c = np.cumsum(w)
    S = c[-1]
    target = u * S
    i = int(np.searchsorted(c, target, side="left"))
    i = min(i, w.shape[0] - 1)
    lo = c[i - 1] if i > 0 else 0.0
    return i, min(target - lo, c[i] - target) / S


def draw_candidates(z, temperature: float, u_row, u_tile, tile: int = DRAW_TILE):
    """Candidate per row drawn from softmax(z / temperature), in two levels.

    With zt = z / temperature, tile j holding ids [j*tile, (j+1)*tile):
      J = inverse-CDF pick over the tile masses sum_{v in j} exp(zt_v) with u_row,
      v = inverse-CDF pick over exp(zt_v), v in J, with u_tile[J].
    P(v) = P(J) P(v | J) = softmax(zt)_v, so this is a draw from the full
    softmax.  Returns (candidates int64 [T], margin [T]): margin is the smaller
    relative distance of either pick's target to an interval edge (how far
    rounding would have to move a sum to change the pick)."""
    z = np.asarray(z, dtype=np.float64)
    T, V = z.shape
    zt = z / float(np.float32(temperature))
    n_tiles = V // tile
    cand = np.empty(T, dtype=np.int64)
    margin = np.empty(T)
    for r in range(T):
        zr = zt[r].reshape(n_tiles, tile)
        mt = zr.max(axis=1)
        lam = mt + np.log(np.exp(zr - mt[:, None]).sum(axis=1))      # log-mass of each tile
        J, m1 = _inverse_cdf(np.exp(lam - lam.max()), u_row[r])
        v, m2 = _inverse_cdf(np.exp(zr[J] - mt[J]), u_tile[r, J])
        cand[r] = J * tile + v
        margin[r] = min(m1, m2)
    return cand, margin


def sample_step(canvas, accepted, argmax, entropy, logconf, *, seed: int, block: int, step: int,
                vocab: int, entropy_thresh: float, min_accept: int, max_steps: int, request: int = 0,
                rule: str = "threshold", entropy_budget: float = 0.1, stop_entropy: float = 0.005,
                prev_argmax=None, candidates=None):
    """One application of the rule.  Returns (canvas, accepted, remaining).

    `prev_argmax` (budget rule) is the argmax of the previous step, None at
    the first step of a canvas.  `candidates` (default: the argmax) are the
    tokens written at accepted positions."""
    canvas = np.asarray(canvas, dtype=np.int64).copy()
    accepted = np.asarray(accepted).astype(bool).copy()
    if rule == "budget":
        A = accept_set_budget(entropy, logconf, accepted, argmax, prev_argmax, entropy_budget, stop_entropy,
                              force_all=step >= max_steps)
    else:
        A = accept_set(entropy, logconf, accepted, entropy_thresh, min_accept, force_all=step >= max_steps)
    cand = argmax if candidates is None else candidates
    canvas[A] = np.asarray(cand, dtype=np.int64)[A]
    rejected = (~accepted) & (~A)
    pos = np.nonzero(rejected)[0]
    if pos.size:
        canvas[pos] = renoise_tokens(seed, block, step, pos, vocab, request)
    accepted |= A
    return canvas, accepted, int(rejected.sum())


def init_canvas(n: int, *, seed: int, block: int, vocab: int, request: int = 0):
    """Fresh canvas: uniform random ids drawn with step 0, nothing accepted."""
    return renoise_tokens(seed, block, 0, np.arange(n), vocab, request), np.zeros(n, dtype=bool)
