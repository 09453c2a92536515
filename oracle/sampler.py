"""Accept / freeze / re-noise rule of one denoising step.

The pages' loop ([P2] §"How the sampler actually works"): after the
bidirectional pass, take a candidate token at every position, accept positions
from most to least confident, re-randomise the rejected ones for the next
step, and stop when the canvas has converged or at a step cap.  Accepted
tokens are kept ([P2] §"What DiffusionGemma is": the model "accepts the tokens
it is confident about, re-randomizes the rest").

Rule used here (the workload's sampler rule, which replaces the pages'
cumulative entropy budget of 0.1):
  U = positions not yet accepted;
  A = {i in U : H_i <= entropy_thresh}
      union the min(min_accept, |U|) positions of U with the highest logconf
      (ties to the lower position);
  at the step cap every position of U is accepted;
  i in A:      c_i <- argmax_i, frozen for the rest of the canvas;
  i in U \\ A:  c_i <- tok(seed, block, step, i)  (Philox, see philox.py);
  remaining = |U \\ A|.
Candidates are the argmax (temperature 0).
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


def sample_step(canvas, accepted, argmax, entropy, logconf, *, seed: int, block: int, step: int,
                vocab: int, entropy_thresh: float, min_accept: int, max_steps: int, request: int = 0):
    """One application of the rule.  Returns (canvas, accepted, remaining)."""
    canvas = np.asarray(canvas, dtype=np.int64).copy()
    accepted = np.asarray(accepted).astype(bool).copy()
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
