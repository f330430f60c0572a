"""Pins of the pair-trellis FP8 codebook oracle (oracle.pair_trellis), CPU only.

The codebook is the exlr8 card's pmcgx ("Stores": a pair trellis, two weights per 20-bit
state, each the sum of the two fp16 halves of the state's product with one of two 32-bit
multipliers, rounded to FP8 E4M3) under readings R20-R26.  The oracle is pinned by:
  * hand-derived weights of single states (tests/golden/pair_trellis_worked_values.txt);
  * its binary16 addition against numpy's float16 arithmetic, and its E4M3 rounding
    against torch's float8_e4m3fn conversion (library routines), exhaustively over every
    masked half and over random sums;
  * hand-derived states of single-bit tiles (tests/golden/pair_trellis_single_bit.txt)
    and a second formulation of the window (a shift register consuming 2K bits a pair);
  * closed forms: an all-zero stream decodes to 0 everywhere, an all-ones stream to the
    weights of state 0xFFFFF everywhere;
  * the tile layout (pair q at rows 2q, 2q+1 mod 16 of column q div 8);
  * the activation quantiser's scale range and rounding (torch float8_e4m3fn).
"""
import numpy as np
import pytest
import torch

from oracle import pair_trellis as PT
from tests.conftest import read_golden


def test_worked_values():
    rows = read_golden("pair_trellis_worked_values.txt")
    assert len(rows) >= 5
    for state, which, P, lo, hi, s16, w8 in rows:
        state, which = int(state), int(which)
        Pa, Pb = PT.products(np.array([state]))
        assert int((Pa, Pb)[which][0]) == int(P, 16)
        assert int(lo, 16) == int(P, 16) & 0xFFFF & PT.HALF_MASK
        assert int(hi, 16) == (int(P, 16) >> 16) & PT.HALF_MASK
        s = PT.fp16_round(PT.half_value(np.array([int(lo, 16)])) + PT.half_value(np.array([int(hi, 16)])))
        assert float(s[0]) == float(s16)
        assert PT.pair_weight(state, which) == float(w8)


def test_fp16_addition_matches_numpy_float16():
    rng = np.random.default_rng(9001)
    a = rng.integers(0, 1 << 16, size=400000).astype(np.uint64) & np.uint64(PT.HALF_MASK)
    b = rng.integers(0, 1 << 16, size=400000).astype(np.uint64) & np.uint64(PT.HALF_MASK)
    mine = PT.fp16_round(PT.half_value(a) + PT.half_value(b))
    lib = (a.astype(np.uint16).view(np.float16) + b.astype(np.uint16).view(np.float16)).astype(np.float64)
    np.testing.assert_array_equal(mine, lib)
    # every masked half is finite and below 2 in magnitude
    allh = np.arange(1 << 16, dtype=np.uint64) & np.uint64(PT.HALF_MASK)
    v = allh.astype(np.uint16).view(np.float16)
    assert np.isfinite(v).all() and np.abs(v).max() < 2
    np.testing.assert_array_equal(PT.half_value(allh), v.astype(np.float64))


def test_e4m3_rounding_matches_torch_float8():
    # every binary16 value below 4 in magnitude: all sums of two masked halves are among them
    allh = np.arange(1 << 16, dtype=np.uint64)
    v = allh.astype(np.uint16).view(np.float16).astype(np.float64)
    v = v[np.isfinite(v) & (np.abs(v) < 4)]
    lib = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    np.testing.assert_array_equal(PT.e4m3_round(v), lib)


def test_single_bit_tiles():
    for K, b, *entries in read_golden("pair_trellis_single_bit.txt"):
        K, b = int(K), int(b)
        words = np.zeros(8 * K, dtype=np.uint32)
        words[b // 32] = np.uint32(1 << (b % 32))
        want = np.zeros(128, dtype=np.uint64)
        for e in entries:
            q, st = e.split(":")
            want[int(q)] = int(st, 16)
        got = np.array([PT.pair_state(words, K, q) for q in range(128)], dtype=np.uint64)
        np.testing.assert_array_equal(got, want, err_msg="K=%d b=%d" % (K, b))
        np.testing.assert_array_equal(PT.pair_states_tiles(words[None], K)[0], want)


@pytest.mark.parametrize("K", [2, 3, 4])
def test_state_window_equals_a_shift_register(K):
    # second formulation: the state of pair q+1 is the state of pair q shifted right by 2K
    # with the next 2K stream bits entering at the top (bits 20-2K .. 19)
    rng = np.random.default_rng(9100 + K)
    n = 256 * K
    tiles = rng.integers(0, 1 << 32, size=(20, 8 * K), dtype=np.uint64).astype(np.uint32)
    states = PT.pair_states_tiles(tiles, K)
    for t in range(tiles.shape[0]):
        bits = [(int(tiles[t, j // 32]) >> (j % 32)) & 1 for j in range(n)]
        s = sum(bits[i] << i for i in range(20))
        for q in range(128):
            assert int(states[t, q]) == s, (t, q)
            top = sum(bits[(2 * K * (q + 1) + 20 - 2 * K + i) % n] << i for i in range(2 * K))
            s = (s >> (2 * K)) | (top << (20 - 2 * K))


@pytest.mark.parametrize("K", [2, 3, 4])
def test_constant_streams_and_tile_layout(K):
    zero = np.zeros((2, 8 * K), dtype=np.uint32)
    assert not PT.decode_tiles(zero, K).any()
    ones = np.full((1, 8 * K), 0xFFFFFFFF, dtype=np.uint32)
    wa, wb = PT.pair_weight(0xFFFFF, 0), PT.pair_weight(0xFFFFF, 1)
    t = PT.decode_tiles(ones, K)[0]
    # position p = 2q + which sits at row p mod 16, column p div 16
    assert np.all(t[0::2, :] == wa) and np.all(t[1::2, :] == wb)
    # single-bit tile: the nonzero pairs land at rows 2q, 2q + 1 of column q div 8
    words = np.zeros(8 * K, dtype=np.uint32)
    words[0] = 1
    t = PT.decode_tiles(words[None], K)[0]
    states = PT.pair_states_tiles(words[None], K)[0]
    for q in range(128):
        w = PT.pair_weights(np.array([states[q]]))[0]
        assert t[(2 * q) % 16, q // 8] == w[0] and t[(2 * q + 1) % 16, q // 8] == w[1]
    # a matrix of tiles in row-major tile order
    rng = np.random.default_rng(9200 + K)
    bits = rng.integers(0, 1 << 32, size=(2 * 3 * 8 * K), dtype=np.uint64).astype(np.uint32)
    M = PT.decode_matrix(bits, K, 32, 48)
    tiles = PT.decode_tiles(bits.reshape(6, 8 * K), K)
    for i in range(2):
        for j in range(3):
            np.testing.assert_array_equal(M[16 * i:16 * i + 16, 16 * j:16 * j + 16], tiles[3 * i + j])


def test_codebook_statistics_over_all_states():
    # all 2^20 states: finite E4M3 values, |w| <= 4 (sums below 4 may round up to 4), zero mean
    st = np.arange(1 << 20, dtype=np.uint64)
    w = PT.pair_weights(st)
    assert np.isfinite(w).all() and np.abs(w).max() <= 4
    lib = torch.from_numpy(w.astype(np.float32)).to(torch.float8_e4m3fn).float().numpy()
    np.testing.assert_array_equal(w, lib)        # every weight is an E4M3 value
    assert abs(w.mean()) < 1e-3


def test_activation_quantiser():
    rng = np.random.default_rng(9300)
    v = rng.standard_normal((64, 256)) * np.exp(rng.uniform(-20, 20, size=(64, 1)))
    v[3] = 0.0
    v[4, :] = 0.0
    v[4, 7] = 448.0                                   # exact power-of-two boundary cases
    v[5, :] = 2.0 ** -30
    v8, e = PT.quantize_rows_e4m3(v)
    m = np.abs(v).max(axis=1)
    nz = m > 0
    r = m[nz] / 2.0 ** e[nz]
    assert np.all((r > 224) & (r <= 448))
    assert e[3] == 0 and not v8[3].any()
    lib = torch.from_numpy((v / 2.0 ** e[:, None]).astype(np.float64)).to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(v8, lib)
