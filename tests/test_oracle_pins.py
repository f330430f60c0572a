"""Pins of the CPU oracle against facts that do not come from the oracle itself:
hand-derived worked values, closed forms, exhaustive invariants, a second formulation
of the trellis (shift-register walk), textbook Hadamard identities and a library
Hadamard, brute force on tiny inputs.

Source of the method: "DeepSeek-V4.1-Flash-1017 · dsx T16", "How T16 works" (items 1,
2, 4), the bitshift trellis of its intro, and the 128-wide Hadamard rotations named
there and in the exlr8 card's "Stores" section.
"""
import math

import numpy as np
import pytest

from oracle import layer as L
from oracle import t16
from tests.conftest import read_golden
from trellis_quantized_moe_gemv_b200 import inputs


# ----------------------------------------------------------------------------- T16 values

def test_worked_values_from_hand_arithmetic():
    rows = read_golden("t16_worked_values.txt")
    assert len(rows) >= 15
    for window, _P, t, c in rows:
        w = int(window, 16)
        assert t16.t16_value(w) == int(t), window
        assert t16.code(w) == int(c), window


def test_exhaustive_histogram_is_triangular():
    # 0x3A2F is odd, so multiplication by it permutes the 65,536 residues mod 2^16;
    # the sum of the two (unsigned) bytes of a uniformly distributed 16-bit number has
    # count(t) = t + 1 for t <= 255 and 511 - t above.  A signed-byte reading, a
    # product kept to more than 16 bits or a dropped byte would all break this.
    ts = np.array([t16.t16_value(w) for w in range(65536)])
    hist = np.bincount(ts, minlength=511)
    expected = np.array([t + 1 if t <= 255 else 511 - t for t in range(511)])
    assert hist.size == 511
    np.testing.assert_array_equal(hist, expected)
    codes = np.array([t16.code(w) for w in range(0, 65536, 1)])
    assert codes.sum() == 0 and codes.min() == -255 and codes.max() == 255


# ----------------------------------------------------------------------------- bitstream

@pytest.mark.parametrize("K", [2, 3, 4])
def test_constant_streams_closed_form(K):
    zeros = np.zeros(8 * K, dtype=np.uint32)
    ones = np.full(8 * K, 0xFFFFFFFF, dtype=np.uint32)
    np.testing.assert_array_equal(t16.decode_tile(zeros, K), np.full((16, 16), -255))
    np.testing.assert_array_equal(t16.decode_tile(ones, K), np.full((16, 16), 151))


def test_single_bit_tile_pins_bit_order_tail_biting_and_column_major():
    expected = {2: np.full((16, 16), -255), 3: np.full((16, 16), -255), 4: np.full((16, 16), -255)}
    for K, r, q, c in read_golden("tile_single_bit.txt"):
        expected[int(K)][int(r), int(q)] = int(c)
    for K in (2, 3, 4):
        words = np.zeros(8 * K, dtype=np.uint32)
        words[0] = 1
        np.testing.assert_array_equal(t16.decode_tile(words, K), expected[K], err_msg="K=%d" % K)


def test_tile_order_is_row_major_over_the_matrix():
    # 32 x 32 matrix = 2 x 2 tiles; tile index 1 is all ones, the rest zero.
    K = 2
    bits = np.zeros(4 * 8 * K, dtype=np.uint32)
    bits[8 * K:2 * 8 * K] = 0xFFFFFFFF
    codes = t16.decode_matrix(bits, K, 32, 32)
    expected = np.full((32, 32), -255)
    expected[0:16, 16:32] = 151
    np.testing.assert_array_equal(codes, expected)
    rows = t16.decode_rows(bits, K, 32, 32, [3, 20])
    np.testing.assert_array_equal(rows, expected[[3, 20]])


def _state_walk(words, n, K):
    """Second formulation: a 16-bit shift register that shifts right by K and takes
    the next K stream bits in at the top, started from the stream's first 16 bits
    (read as one big little-endian integer) and closed around the tail."""
    n_bits = n * K
    S = 0
    for i, w in enumerate(np.asarray(words, dtype=np.uint64)):
        S |= int(w) << (32 * i)
    stream = [(S >> j) & 1 for j in range(n_bits)]
    state = 0
    for i in range(16):
        state |= stream[i % n_bits] << i
    states = []
    for p in range(n):
        states.append(state)
        incoming = 0
        for i in range(K):
            incoming |= stream[(p * K + 16 + i) % n_bits] << i
        state = (state >> K) | (incoming << (16 - K))
    assert state == states[0], "tail-biting register must return to its start"
    return states


@pytest.mark.parametrize("K", [2, 3, 4])
def test_windows_match_shift_register_walk(K):
    rng = np.random.default_rng(10 + K)
    for _ in range(3):
        words = rng.integers(0, 2 ** 32, size=8 * K, dtype=np.uint64).astype(np.uint32)
        walk = _state_walk(words, 256, K)
        win = [t16.window(words, 256 * K, K, p) for p in range(256)]
        assert win == walk
        codes = t16.decode_stream(words, 256, K)
        assert list(codes) == [t16.code(w) for w in walk]


@pytest.mark.parametrize("n,K", [(8, 2), (5, 3)])
def test_exhaustive_tiny_trellis(n, K):
    # Every stream of a tiny tail-biting trellis (n*K = 16 and 15 bits: the window
    # wraps the whole stream): oracle windows equal the shift-register states, and
    # decoding is a function of the stream alone (re-encoding by exhaustive search
    # finds the true stream among the zero-error candidates).
    n_bits = n * K
    table = {}
    rng = np.random.default_rng(7)
    check = set(rng.integers(0, 2 ** n_bits, size=64).tolist())
    for s in range(2 ** n_bits):
        words = np.array([s], dtype=np.uint32)
        codes = tuple(t16.decode_stream(words, n, K))
        table.setdefault(codes, []).append(s)
        if s in check:
            walk = _state_walk(words, n, K)
            assert [t16.window(words, n_bits, K, p) for p in range(n)] == walk
    for s in check:
        codes = tuple(t16.decode_stream(np.array([s], dtype=np.uint32), n, K))
        assert s in table[codes]


# ----------------------------------------------------------------------------- Hadamard

def test_hadamard_textbook_identities():
    H = L.hadamard_matrix(128)
    np.testing.assert_array_equal(H @ H.T, 128 * np.eye(128))
    np.testing.assert_array_equal(H, H.T)
    e0 = np.zeros(128); e0[0] = 1
    np.testing.assert_array_equal(H @ e0, np.ones(128))
    np.testing.assert_array_equal(H @ np.ones(128), 128 * e0)
    scipy_linalg = pytest.importorskip("scipy.linalg")
    np.testing.assert_array_equal(H, scipy_linalg.hadamard(128))


def _fwht(v):
    v = np.array(v, dtype=np.float64)
    h = 1
    while h < v.size:
        for i in range(0, v.size, 2 * h):
            a = v[i:i + h].copy()
            b = v[i + h:i + 2 * h].copy()
            v[i:i + h], v[i + h:i + 2 * h] = a + b, a - b
        h *= 2
    return v


def test_rotate_matches_butterflies_and_is_an_involution():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((3, 512))
    r = L.rotate(x)
    for t in range(3):
        for c in range(4):
            np.testing.assert_allclose(r[t, 128 * c:128 * (c + 1)],
                                       _fwht(x[t, 128 * c:128 * (c + 1)]) / math.sqrt(128),
                                       rtol=0, atol=1e-12)
    np.testing.assert_allclose(L.rotate(r), x, rtol=0, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(r, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)


# ----------------------------------------------------------------------------- projection

@pytest.mark.parametrize("fill,code", [(0x00000000, -255), (0xFFFFFFFF, 151)])
def test_projection_constant_stream_closed_form(fill, code):
    # With every code equal to c, y_i = s_i*kappa*c*sum_j x'_j, and the columns of H sum
    # to 128*e_0, so sum_j x'_j = sqrt(128) * sum over chunks of each chunk's first entry.
    rows, cols, K = 64, 384, 2
    bits = np.full(inputs.words_per_matrix(rows, cols, K), fill, dtype=np.uint32)
    rng = np.random.default_rng(5)
    s = inputs.random_scales(rng, rows)
    x = inputs.random_activations(rng, (2, cols), "bf16")
    y, bound = L.single_projection(bits, K, rows, cols, s, x)
    chunk_first = x[:, ::128].astype(np.float64).sum(axis=1)
    expect = (s.astype(np.float64)[None, :] * 2.0 ** -12 * code
              * math.sqrt(128) * chunk_first[:, None])
    np.testing.assert_allclose(y, expect, rtol=1e-12, atol=1e-12)
    assert np.all(bound >= np.abs(y) - 1e-12)


def test_project_orientation_exact_on_integers():
    rng = np.random.default_rng(9)
    W = rng.integers(-255, 256, size=(5, 7))
    x = rng.integers(-100, 100, size=(3, 7))
    y = L.project(W, x)
    for b in range(3):
        for i in range(5):
            assert y[b, i] == sum(int(W[i, j]) * int(x[b, j]) for j in range(7))
    assert np.array_equal(L.abs_bound(W, x)[1, 2], sum(abs(int(W[2, j]) * int(x[1, j])) for j in range(7)))


def test_dequantize_applies_row_scale_and_kappa():
    codes = np.array([[1, -2], [3, 4]])
    s = np.array([0.5, 1.25], dtype=np.float16)
    np.testing.assert_array_equal(L.dequantize(codes, s),
                                  np.array([[0.5 / 4096, -1.0 / 4096], [3.75 / 4096, 5.0 / 4096]]))


# ----------------------------------------------------------------------------- routing

def test_topk_closed_form_and_ties():
    ids, w = L.route_topk(np.array([[0.0, 1.0, 3.0, 2.0]], dtype=np.float32), 2)
    assert ids.tolist() == [[2, 3]]
    e = math.e
    np.testing.assert_allclose(w[0], [e / (1 + e), 1 / (1 + e)], rtol=1e-15)
    ids, w = L.route_topk(np.zeros((1, 10), dtype=np.float32), 4)
    assert ids.tolist() == [[0, 1, 2, 3]]
    np.testing.assert_allclose(w[0], [0.25] * 4, rtol=1e-15)
    ids, _ = L.route_topk(np.array([[5.0, 7.0, 7.0, 1.0, 7.0]], dtype=np.float32), 3)
    assert ids.tolist() == [[1, 2, 4]]


def test_topk_weights_sum_to_one():
    rng = np.random.default_rng(1)
    logits = inputs.normal_logits(rng, 16)
    ids, w = L.route_topk(logits, 8)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-14)
    for t in range(16):
        assert len(set(ids[t].tolist())) == 8
        kept = logits[t, ids[t]]
        assert np.all(np.diff(kept) <= 0)
        assert kept.min() >= np.delete(logits[t], ids[t]).max()


def test_permute_worked_example():
    topk = np.array([[2, 0], [0, 1], [2, 2]])
    counts, offsets, perm, inv = L.route_permute(topk, 3)
    assert counts.tolist() == [2, 1, 3]
    assert offsets.tolist() == [0, 2, 3, 6]
    assert perm.tolist() == [1, 2, 3, 0, 4, 5]
    assert inv.tolist() == [3, 0, 1, 2, 4, 5]


def test_permute_invariants():
    rng = np.random.default_rng(2)
    ids, _ = L.route_topk(inputs.normal_logits(rng, 64, 40), 8)
    counts, offsets, perm, inv = L.route_permute(ids, 40)
    assert counts.sum() == 64 * 8 and offsets[-1] == 64 * 8
    np.testing.assert_array_equal(perm[inv], np.arange(64 * 8))
    flat = ids.reshape(-1)
    for e in range(40):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)


def test_combine_closed_forms():
    # k = 1 with unit weights is a pure gather; equal weights 1/k give the mean.
    rng = np.random.default_rng(4)
    y = rng.standard_normal((6, 5))
    inv = np.array([3, 0, 5, 1, 4, 2])
    np.testing.assert_array_equal(L.combine(y, inv, np.ones((6, 1))), y[inv])
    out = L.combine(y, np.arange(6), np.full((3, 2), 0.5))
    np.testing.assert_allclose(out, 0.5 * (y[0::2] + y[1::2]), rtol=1e-15)


# ----------------------------------------------------------------------------- expert

def test_silu_identities():
    z = np.linspace(-20, 20, 81)
    np.testing.assert_allclose(L.silu(z) - L.silu(-z), z, rtol=0, atol=1e-12)
    assert L.silu(0.0) == 0.0 and L.silu_prime(0.0) == 0.5
    np.testing.assert_allclose(L.silu(40.0), 40.0, rtol=1e-15)
    h = 1e-6
    np.testing.assert_allclose(L.silu_prime(z), (L.silu(z + h) - L.silu(z - h)) / (2 * h), atol=1e-8)


def test_moe_layer_closed_form_with_constant_streams():
    # Every stream all-zero -> every code -255.  For token t with chunk-first sum
    # X_t = sum_c x[t, 128c]:  g_f = s_g[f] * G, u_f = s_u[f] * G with
    # G = -255 kappa sqrt(128) X_t; with F = 128 (one chunk) the rotated h sums to
    # sqrt(128) h_0, so y_i = s_d[i] kappa (-255) sqrt(128) silu(g_0) u_0.
    lay = inputs.small_layer(11, E=5, D=256, F=128, split={2: 3, 3: 1, 4: 1})
    for g in lay.groups:
        g.gate[:] = 0
        g.up[:] = 0
        g.down[:] = 0
    rng = np.random.default_rng(12)
    x = inputs.random_activations(rng, (3, 256), "bf16")
    logits = inputs.normal_logits(rng, 3, 5)
    res = L.moe_layer(lay, x, logits, 2)
    kappa = 2.0 ** -12
    where = {int(e): (g, i) for g in lay.groups for i, e in enumerate(g.ids)}
    for t in range(3):
        G = -255 * kappa * math.sqrt(128) * float(x[t, ::128].astype(np.float64).sum())
        out = np.zeros(256)
        for s in range(2):
            g, i = where[int(res["topk_ids"][t, s])]
            g0 = float(g.s_gate[i, 0]) * G
            u0 = float(g.s_up[i, 0]) * G
            h0 = g0 / (1 + math.exp(-g0)) * u0
            out += res["topk_w"][t, s] * g.s_down[i].astype(np.float64) * kappa * (-255) * math.sqrt(128) * h0
        np.testing.assert_allclose(res["out"][t], out, rtol=1e-10, atol=1e-14)
        assert np.all(res["bound"][t] > 0)


# ----------------------------------------------------------------- two-sided transform

def _dense_rotation(n):
    """Block-diagonal orthonormal Hadamard of size n from scipy (independent of the
    oracle's own construction)."""
    import scipy.linalg
    H = scipy.linalg.hadamard(128).astype(np.float64) / np.sqrt(128.0)
    return np.kron(np.eye(n // 128), H)


def _two_sided_layer():
    layer = inputs.small_layer(4242, E=6, D=256, F=256, split={2: 3, 3: 2, 4: 1})
    return inputs.with_signs(layer, 4243)


def test_two_sided_expert_equals_dense_effective_matrices():
    # g = diag(s_gu) H W_gate H diag(s_x) x and y = diag(s_y) H W_down H diag(s_h) h,
    # with the rotations as explicit dense matrices.
    layer = _two_sided_layer()
    sg = layer.signs
    w = L.ExpertWeights(layer)
    rng = np.random.default_rng(4244)
    x = rng.standard_normal((3, layer.D))
    HD, HF = _dense_rotation(layer.D), _dense_rotation(layer.F)
    for e in (0, 3, 5):
        st = L.expert_forward(w, e, L.rotate_in(x, sg["x"]), signs=sg)
        Wg_eff = np.diag(sg["gu"].astype(float)) @ HF @ w.matrix(e, "gate") @ HD @ np.diag(sg["x"].astype(float))
        Wu_eff = np.diag(sg["gu"].astype(float)) @ HF @ w.matrix(e, "up") @ HD @ np.diag(sg["x"].astype(float))
        np.testing.assert_allclose(st["g"], x @ Wg_eff.T, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(st["u"], x @ Wu_eff.T, rtol=1e-10, atol=1e-12)
        h = L.silu(x @ Wg_eff.T) * (x @ Wu_eff.T)
        Wd_eff = np.diag(sg["y"].astype(float)) @ HD @ w.matrix(e, "down") @ HF @ np.diag(sg["h"].astype(float))
        np.testing.assert_allclose(st["y"], h @ Wd_eff.T, rtol=1e-9, atol=1e-12)


def test_two_sided_output_rotation_preserves_chunk_norms():
    layer = _two_sided_layer()
    w = L.ExpertWeights(layer)
    x_rot = L.rotate(np.random.default_rng(7).standard_normal((2, layer.D)))
    one = L.expert_forward(w, 2, x_rot)
    two = L.expert_forward(w, 2, x_rot, signs=layer.signs)
    g1 = one["g"].reshape(2, -1, 128)
    g2 = two["g"].reshape(2, -1, 128)
    np.testing.assert_allclose(np.linalg.norm(g2, axis=-1), np.linalg.norm(g1, axis=-1), rtol=1e-12)


def test_two_sided_selected_down_rows_match_full_rows():
    layer = _two_sided_layer()
    rng = np.random.default_rng(4245)
    x = rng.standard_normal((2, layer.D))
    logits = rng.standard_normal((2, layer.E)).astype(np.float32)
    full = L.moe_tokens(layer, x, logits, 2, [0, 1])
    rows = np.array([3, 130, 255, 7])
    part = L.moe_tokens(layer, x, logits, 2, [0, 1], down_rows=rows)
    np.testing.assert_allclose(part["out"], full["out"][:, rows], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(part["bound"], full["bound"][:, rows], rtol=1e-12, atol=1e-14)
