"""Philox counter-based generator and the re-noise token draw.

Philox-NxW-R follows [SC11] §"Philox": each round multiplies the even words
of the counter by fixed odd multipliers, takes the high and low halves of the
double-width products, XORs the high halves with the odd words and the round
key, and permutes the words; the key is bumped by fixed Weyl constants between
rounds.  The 4x32 and 4x64 variants differ only in word width and constants,
so both run through the same `philox4` below; the 4x64 instance is
cross-checked against NumPy's Philox bit generator in the tests, which pins
the round structure shared with the 4x32 instance used by the method.

The pages name no generator; they say only that rejected positions are
re-randomised for the next step ([P2] §"How the sampler actually works",
item 4; §"What DiffusionGemma is").  Reading taken:
  key     = (seed mod 2^32, seed >> 32)
  counter = (position, step, block, request)
  token   = floor(x0 * V / 2^32)   (x0 = first output word; exact for power-of-two V)
Canvas initialisation draws with step 0; the re-noise after step s uses s.
"""
from __future__ import annotations

import numpy as np

# multipliers and Weyl key increments, per word width [SC11]
_CONST = {
    32: dict(M0=0xD2511F53, M1=0xCD9E8D57, W0=0x9E3779B9, W1=0xBB67AE85),
    64: dict(M0=0xD2E7470EE14C6C93, M1=0xCA5A826395121157,
             W0=0x9E3779B97F4A7C15, W1=0xBB67AE8584CAA73B),
}


def _mulhilo(a: int, b: int, w: int):
    p = a * b
    mask = (1 << w) - 1
    return p >> w, p & mask


def philox4(counter, key, w: int = 32, rounds: int = 10):
    """Philox-4xW-R on python ints.  counter: 4 words, key: 2 words."""
    c = _CONST[w]
    mask = (1 << w) - 1
    x0, x1, x2, x3 = (int(v) & mask for v in counter)
    k0, k1 = (int(v) & mask for v in key)
    for r in range(rounds):
        if r > 0:
            k0 = (k0 + c["W0"]) & mask
            k1 = (k1 + c["W1"]) & mask
        hi0, lo0 = _mulhilo(c["M0"], x0, w)
        hi1, lo1 = _mulhilo(c["M1"], x2, w)
        x0, x1, x2, x3 = hi1 ^ x1 ^ k0, lo1, hi0 ^ x3 ^ k1, lo0
    return x0, x1, x2, x3


def philox4x32_10_np(c0, c1, c2, c3, k0: int, k1: int):
    """Vectorised Philox-4x32-10 over uint32 counter arrays (same rounds as `philox4`)."""
    M0, M1 = np.uint64(_CONST[32]["M0"]), np.uint64(_CONST[32]["M1"])
    W0, W1 = _CONST[32]["W0"], _CONST[32]["W1"]
    m32 = np.uint64(0xFFFFFFFF)
    x0, x1, x2, x3 = (np.asarray(v, dtype=np.uint64) & m32 for v in (c0, c1, c2, c3))
    k0, k1 = int(k0) & 0xFFFFFFFF, int(k1) & 0xFFFFFFFF
    for r in range(10):
        if r > 0:
            k0 = (k0 + W0) & 0xFFFFFFFF
            k1 = (k1 + W1) & 0xFFFFFFFF
        p0 = M0 * x0          # < 2^64, exact in uint64
        p1 = M1 * x2
        hi0, lo0 = p0 >> np.uint64(32), p0 & m32
        hi1, lo1 = p1 >> np.uint64(32), p1 & m32
        x0, x1, x2, x3 = hi1 ^ x1 ^ np.uint64(k0), lo1, hi0 ^ x3 ^ np.uint64(k1), lo0
    return tuple(v.astype(np.uint32) for v in (x0, x1, x2, x3))


def seed_key(seed: int):
    seed = int(seed) & ((1 << 64) - 1)
    return seed & 0xFFFFFFFF, seed >> 32


def token_from_word(x0, vocab: int):
    """Map a uniform 32-bit word to [0, vocab) by multiply-shift."""
    return ((np.asarray(x0, dtype=np.uint64) * np.uint64(vocab)) >> np.uint64(32)).astype(np.int64)


def renoise_tokens(seed: int, block: int, step: int, positions, vocab: int, request: int = 0):
    """tok(seed, block, step, i) for each position i (int64 array)."""
    pos = np.asarray(positions, dtype=np.uint64)
    k0, k1 = seed_key(seed)
    n = pos.shape[0]
    x0, _, _, _ = philox4x32_10_np(pos, np.full(n, step, np.uint64), np.full(n, block, np.uint64),
                                   np.full(n, request, np.uint64), k0, k1)
    return token_from_word(x0, vocab)


def renoise_token_scalar(seed: int, block: int, step: int, position: int, vocab: int, request: int = 0):
    k0, k1 = seed_key(seed)
    x0 = philox4((position, step, block, request), (k0, k1), 32, 10)[0]
    return (x0 * vocab) >> 32
