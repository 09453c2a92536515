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
Candidates are the argmax (temperature 0).

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

from .philox import renoise_tokens


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


def sample_step(canvas, accepted, argmax, entropy, logconf, *, seed: int, block: int, step: int,
                vocab: int, entropy_thresh: float, min_accept: int, max_steps: int, request: int = 0,
                rule: str = "threshold", entropy_budget: float = 0.1, stop_entropy: float = 0.005,
                prev_argmax=None):
    """One application of the rule.  Returns (canvas, accepted, remaining).

    `prev_argmax` (budget rule) is the argmax of the previous step, None at
    the first step of a canvas."""
    canvas = np.asarray(canvas, dtype=np.int64).copy()
    accepted = np.asarray(accepted).astype(bool).copy()
    if rule == "budget":
        A = accept_set_budget(entropy, logconf, accepted, argmax, prev_argmax, entropy_budget, stop_entropy,
                              force_all=step >= max_steps)
    else:
        A = accept_set(entropy, logconf, accepted, entropy_thresh, min_accept, force_all=step >= max_steps)
    canvas[A] = np.asarray(argmax, dtype=np.int64)[A]
    rejected = (~accepted) & (~A)
    pos = np.nonzero(rejected)[0]
    if pos.size:
        canvas[pos] = renoise_tokens(seed, block, step, pos, vocab, request)
    accepted |= A
    return canvas, accepted, int(rejected.sum())


def init_canvas(n: int, *, seed: int, block: int, vocab: int, request: int = 0):
    """Fresh canvas: uniform random ids drawn with step 0, nothing accepted."""
    return renoise_tokens(seed, block, 0, np.arange(n), vocab, request), np.zeros(n, dtype=bool)
