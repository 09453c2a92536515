"""Pins of the oracle's Philox generator and token draw (no GPU).

No known-answer vectors for Philox-4x32-10 are available here, so the round
structure is pinned through the 4x64 instance of the same generic code against
NumPy's Philox bit generator (an independent library implementation of
Philox-4x64-10), and the vectorised 4x32 path against the scalar one."""
import numpy as np
import pytest

from oracle import philox as P


@pytest.mark.parametrize("key", [(0, 0), (123456789, 987654321), (2**64 - 1, 2**63 + 5)])
@pytest.mark.parametrize("ctr", [(0, 0, 0, 0), (5, 6, 7, 8), (2**64 - 2, 2**64 - 1, 3, 2**40)])
def test_philox4x64_matches_numpy(key, ctr):
    bg = np.random.Philox(key=np.array(key, dtype=np.uint64), counter=np.array(ctr, dtype=np.uint64))
    raw = [int(v) for v in bg.random_raw(8)]
    # NumPy increments the 256-bit counter before each block
    c = sum(int(v) << (64 * i) for i, v in enumerate(ctr))
    for blk in range(2):
        c = (c + 1) % (1 << 256)
        words = [(c >> (64 * i)) & (2**64 - 1) for i in range(4)]
        assert list(P.philox4(words, key, 64, 10)) == raw[4 * blk: 4 * blk + 4]


def test_vectorised_4x32_matches_scalar():
    rng = np.random.default_rng(0)
    c = rng.integers(0, 2**32, size=(4, 300), dtype=np.uint64)
    c[:, 0] = 0
    c[:, 1] = 2**32 - 1
    for k0, k1 in [(0, 0), (0xDEADBEEF, 0x12345678), (2**32 - 1, 2**32 - 1)]:
        out = P.philox4x32_10_np(c[0], c[1], c[2], c[3], k0, k1)
        for i in range(c.shape[1]):
            ref = P.philox4([int(c[j, i]) for j in range(4)], (k0, k1), 32, 10)
            assert tuple(int(o[i]) for o in out) == ref


def test_round_count_and_width_matter():
    a = P.philox4((1, 2, 3, 4), (5, 6), 32, 10)
    assert a != P.philox4((1, 2, 3, 4), (5, 6), 32, 7)
    assert a != tuple(v & 0xFFFFFFFF for v in P.philox4((1, 2, 3, 4), (5, 6), 64, 10))


def test_token_map_power_of_two_is_top_bits():
    x = np.random.default_rng(1).integers(0, 2**32, size=10000, dtype=np.uint64)
    for logv in (11, 18):
        np.testing.assert_array_equal(P.token_from_word(x, 1 << logv), (x >> np.uint64(32 - logv)).astype(np.int64))
    # general V: floor(x * V / 2^32) stays in range and is monotone in x
    t = P.token_from_word(np.sort(x), 1000)
    assert t.min() >= 0 and t.max() < 1000 and np.all(np.diff(t) >= 0)


def test_renoise_deterministic_and_keyed():
    a = P.renoise_tokens(1234, 2, 5, np.arange(256), 2048)
    np.testing.assert_array_equal(a, P.renoise_tokens(1234, 2, 5, np.arange(256), 2048))
    for other in [P.renoise_tokens(1235, 2, 5, np.arange(256), 2048),
                  P.renoise_tokens(1234, 3, 5, np.arange(256), 2048),
                  P.renoise_tokens(1234, 2, 6, np.arange(256), 2048),
                  P.renoise_tokens(1234, 2, 5, np.arange(256), 2048, request=1)]:
        assert (other != a).mean() > 0.9
    assert [P.renoise_token_scalar(1234, 2, 5, i, 2048) for i in range(16)] == a[:16].tolist()
    # 64-bit seeds use both key words
    assert (P.renoise_tokens(7, 0, 0, np.arange(64), 2048) !=
            P.renoise_tokens(7 + (1 << 32), 0, 0, np.arange(64), 2048)).any()


def test_token_uniformity_chi_square():
    V = 2048
    n = 1 << 20
    pos = np.arange(n) % 4096
    step = np.arange(n) // 4096
    k0, k1 = P.seed_key(99)
    x0, _, _, _ = P.philox4x32_10_np(pos, step, np.zeros(n, np.uint64), np.zeros(n, np.uint64), k0, k1)
    tok = P.token_from_word(x0, V)
    counts = np.bincount(tok, minlength=V)
    exp = n / V
    chi2 = ((counts - exp) ** 2 / exp).sum()
    # dof 2047: mean 2047, sd 64; 6 sd bounds
    assert 2047 - 6 * 64 < chi2 < 2047 + 6 * 64
