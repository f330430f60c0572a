"""Pins of the oracle's tail-biting Viterbi encoder (oracle/encode.py) against things it
does not compute itself: brute force over every stream of small trellises, the exact
tail-biting optimum, closed forms, the independent T16 decoder and the Gaussian
rate-distortion bound."""
import itertools

import numpy as np
import pytest

from oracle import encode as OE
from oracle import t16 as OT


def brute_force(tau, K, vals, L):
    """Minimum cost over every tail-biting stream of n*K bits (n = len(tau))."""
    n = len(tau)
    best = None
    for word in range(1 << (n * K)):
        bits = np.array([(word >> j) & 1 for j in range(n * K)])
        w = OE.bits_windows(bits, K, L)
        c = int(((np.asarray(tau) - np.asarray(vals)[w]) ** 2).sum())
        best = c if best is None or c < best else best
    return best


@pytest.mark.parametrize("L,K,n,seed", [(6, 2, 5, 1), (6, 2, 6, 2), (6, 3, 4, 3), (8, 2, 6, 4), (7, 3, 5, 5)])
def test_viterbi_exact_tail_biting_equals_brute_force(L, K, n, seed):
    rng = np.random.default_rng(seed)
    vals = rng.integers(-40, 40, 1 << L)
    tau = rng.integers(-50, 50, n)
    opt = brute_force(tau, K, vals, L)
    exact = min(OE.viterbi(tau, K, vals, L, b=b)[0] for b in range(1 << (L - K)))
    assert exact == opt
    free, _ = OE.viterbi(tau, K, vals, L)
    assert free <= opt
    cost, w, c1 = OE.encode_windows(tau, K, vals, L)
    assert c1 == free and cost >= opt
    # the windows form a real tail-biting stream and the cost is theirs
    bits = OE.windows_to_bits(w, K, L)
    np.testing.assert_array_equal(OE.bits_windows(bits, K, L), w)
    assert cost == int(((tau - vals[w]) ** 2).sum())


def test_free_pass_matches_brute_force_over_open_paths():
    # without the closure every window path of the bitshift trellis is allowed
    rng = np.random.default_rng(9)
    L, K, n = 6, 2, 5
    vals = rng.integers(-30, 30, 1 << L)
    tau = rng.integers(-40, 40, n)
    best = None
    for w0 in range(1 << L):
        for us in itertools.product(range(1 << K), repeat=n - 1):
            w = [w0]
            for u in us:
                w.append((w[-1] >> K) | (u << (L - K)))
            c = int(((tau - vals[np.array(w)]) ** 2).sum())
            best = c if best is None or c < best else best
    assert OE.viterbi(tau, K, vals, L)[0] == best


@pytest.mark.parametrize("K", [2, 3, 4])
def test_constant_minimum_code_targets_give_the_zero_stream(K):
    # c = -255 only for window 0 (0x3A2F is odd: t = 0 iff the product is 0 iff w = 0)
    words, cost, c1 = OE.encode_tile(np.full((16, 16), -255.0), K)
    assert cost == 0 and c1 == 0
    assert not words.any()


@pytest.mark.parametrize("K", [2, 3, 4])
def test_representable_targets_and_decoder_agreement(K):
    rng = np.random.default_rng(20 + K)
    true_words = rng.integers(0, 2 ** 32, 8 * K, dtype=np.uint64).astype(np.uint32)
    codes = OT.decode_tile(true_words, K).astype(np.float64)
    words, cost, c1 = OE.encode_tile(codes, K)
    assert c1 == 0                          # a zero-error path exists: the free pass finds one
    got = OT.decode_tile(words, K).astype(np.int64)
    tau = OE.quarter_targets(codes)
    assert cost == int(((tau - 4 * got) ** 2).sum())
    if cost == 0:
        np.testing.assert_array_equal(got, codes.astype(np.int64))


@pytest.mark.parametrize("K", [2, 3])
def test_gaussian_error_respects_rate_distortion_and_beats_greedy(K):
    rng = np.random.default_rng(30 + K)
    sigma = 80.0
    x = rng.standard_normal((16, 32)) * sigma
    bits, costs = OE.encode_matrix(x, K)
    codes = OT.decode_matrix(bits, K, 16, 32).astype(np.float64)
    nmse = ((x - codes) ** 2).mean() / sigma ** 2
    # no K-bit-per-sample code beats D(R) = 2^(-2K) on a Gaussian source; the search
    # should land within a small factor of it
    assert 2.0 ** (-2 * K) < nmse < 2.5 * 2.0 ** (-2 * K)
    # the free Viterbi pass is never worse than greedy left-to-right window choice
    vals = 4 * OE.code_table()
    tau = OE.quarter_targets(x[:, :16].T.reshape(-1))
    w = [int(np.argmin((tau[0] - vals) ** 2))]
    greedy = (tau[0] - vals[w[0]]) ** 2
    for p in range(1, 256):
        cand = (w[-1] >> K) | (np.arange(1 << K) << (16 - K))
        d = (tau[p] - vals[cand]) ** 2
        w.append(int(cand[np.argmin(d)]))
        greedy += d.min()
    assert OE.viterbi(tau, K, vals)[0] <= greedy
