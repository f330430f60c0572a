"""Oracle of the pair-trellis FP8 codebook -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference arm of
``bench.py`` may use this module.  The product path never imports it.

Source: "deepseek-v4.1-flash-exlr8" model card, section "Stores": the pmcgx codebook
("V2 L20 0xCBAC1FED/0xBCA14C51") is a pair trellis -- two weights share one 20-bit
state, and each weight is the sum of the two fp16 halves of the state's product with
one of the two multipliers, rounded to FP8 E4M3; the stores hold exactly K bits per
weight (k2 / k3 / k4 units of 163,840 / 245,760 / 327,680 bytes per 655,360 weights).

Readings where the card is silent (listed with the T16 readings in the design notes):
  R20 state: a 16x16 tile's stream is 256*K bits, stream bit j = bit (j mod 32) of
      uint32 word j div 32 (as T16); pair q (0..127) takes the 20-bit window whose bit i
      is stream bit (2*K*q + i) mod 256K (tail-biting): a pair step consumes its two
      weights' 2K bits.
  R21 positions: pair q holds tile positions 2q and 2q + 1 in the column-major order of
      T16 (position p is row p mod 16 of column p div 16).
  R22 products: P_a = (state * 0xCBAC1FED) mod 2^32 gives position 2q, P_b = (state *
      0xBCA14C51) mod 2^32 position 2q + 1.
  R23 halves: each product's low and high 16 bits, with bit 14 (the exponent field's top
      bit) cleared, are binary16 numbers.  Read literally, 6 % of the halves are NaN or
      infinite and 41 % of the sums saturate E4M3; clearing that one bit is the smallest
      change that makes every half finite (|half| < 2).
  R24 rounding: the two halves are added in binary16 arithmetic (round to nearest, ties
      to even) and the sum is rounded to E4M3 (OCP e4m3fn: bias 7, 3 mantissa bits,
      subnormals down to 2^-9, largest 448; round to nearest, ties to even).  Every sum is
      below 4 in magnitude (the rounded weight at most 4), so nothing saturates.
  R25 weight: W[i][j] = s_i * 2^-5 * w[i][j], s_i the fp16 per-output scale (a fixed power
      of two like T16's 2^-12; the codes' RMS is about 0.62).
  R26 activations (FP8 tensor-core path): a route row v is scaled by the power of two 2^-e
      that puts max |v| in (224, 448] and rounded to E4M3 (nearest, ties to even); the
      contraction is s * 2^-5 * 2^e * sum_j w_j * v8_j.

Arithmetic is exact: binary16 and E4M3 values and their pairwise sums are exact in
float64, and rounding to a power-of-two quantum is done with exact float64 steps.
"""
import numpy as np

STATE_BITS = 20
MULT_A = 0xCBAC1FED
MULT_B = 0xBCA14C51
HALF_MASK = 0xBFFF          # clears bit 14 of a 16-bit half (R23)
KAPPA8 = 2.0 ** -5          # R25
E4M3_MAX = 448.0
UNIT = 2.0 ** -24           # every binary16 / E4M3 value is an integer multiple of this


# ------------------------------------------------------------------ bit stream (R20, R21)

def stream_bit(words, j: int) -> int:
    """Bit j of a stream of little-endian uint32 words (bit j mod 32 of word j div 32)."""
    return (int(words[j // 32]) >> (j % 32)) & 1


def pair_state(words, K: int, q: int) -> int:
    """20-bit state of pair q of one tile (8K words): bit i = stream bit (2Kq + i) mod 256K."""
    n = 256 * K
    return sum(stream_bit(words, (2 * K * q + i) % n) << i for i in range(STATE_BITS))


def pair_states_tiles(tiles, K: int) -> np.ndarray:
    """States [n_tiles, 128] of many tiles ([n_tiles, 8K] uint32), the same definition
    evaluated bit by bit for all tiles at once."""
    tiles = np.asarray(tiles, dtype=np.uint64)
    n = 256 * K
    out = np.zeros((tiles.shape[0], 128), dtype=np.uint64)
    for q in range(128):
        for i in range(STATE_BITS):
            j = (2 * K * q + i) % n
            bit = (tiles[:, j // 32] >> np.uint64(j % 32)) & np.uint64(1)
            out[:, q] |= bit << np.uint64(i)
    return out


# ------------------------------------------------------------------ codebook (R22 - R24)

def products(state):
    """(P_a, P_b): the state times each multiplier, mod 2^32."""
    s = np.asarray(state, dtype=np.uint64)
    m32 = np.uint64(0xFFFFFFFF)
    return (s * np.uint64(MULT_A)) & m32, (s * np.uint64(MULT_B)) & m32


def half_units(bits):
    """Value of binary16 bit patterns as signed integers in units of 2^-24 (finite inputs
    only: exponent field < 31)."""
    b = np.asarray(bits, dtype=np.int64)
    sign = np.where(b & 0x8000, -1, 1)
    e = (b >> 10) & 0x1F
    m = b & 0x3FF
    if np.any(e == 0x1F):
        raise ValueError("non-finite binary16")
    mag = np.where(e == 0, m, (1024 + m) << np.maximum(e - 1, 0))
    return sign * mag


def _binade(a):
    """floor(log2(a)) of positive float64 values, exactly (frexp: a = m 2^x, m in [0.5, 1))."""
    return np.frexp(a)[1] - 1


def round_to_quantum(x, quantum):
    """Round float64 values to multiples of a per-element power-of-two quantum, to nearest
    with ties to the even multiple (every step is exact in float64)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    n = np.floor(a / quantum)
    rem = a - n * quantum
    up = (rem > quantum / 2) | ((rem == quantum / 2) & (np.mod(n, 2) == 1))
    return np.sign(x) * (n + up) * quantum


def fp16_round(x):
    """Round to binary16 (nearest, ties to even): spacing 2^-24 below 2^-13 (subnormals and
    the first normal binade), 11 significant bits above."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    q = np.where(a < 2.0 ** -13, 2.0 ** -24, 2.0 ** (_binade(np.maximum(a, 2.0 ** -13)) - 10))
    r = round_to_quantum(x, q)
    if np.any(np.abs(r) > 65504.0):
        raise OverflowError("binary16 overflow")
    return r


def e4m3_round(x):
    """Round to E4M3 (nearest, ties to even): spacing 2^-9 below 2^-5 (subnormals and the
    first normal binade), 4 significant bits above; values beyond 448 are not expected."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    q = np.where(a < 2.0 ** -5, 2.0 ** -9, 2.0 ** (_binade(np.maximum(a, 2.0 ** -5)) - 3))
    r = round_to_quantum(x, q)
    if np.any(np.abs(r) > E4M3_MAX):
        raise OverflowError("E4M3 overflow")
    return r


def half_value(bits):
    """Value of finite binary16 bit patterns (float64, exact)."""
    return half_units(bits).astype(np.float64) * UNIT


def pair_weights(state):
    """E4M3 values (float64, exact) of the two weights of each state: [..., 2]."""
    Pa, Pb = products(state)
    out = []
    for P in (Pa, Pb):
        lo = (P & np.uint64(0xFFFF)) & np.uint64(HALF_MASK)
        hi = (P >> np.uint64(16)) & np.uint64(HALF_MASK)
        out.append(e4m3_round(fp16_round(half_value(lo) + half_value(hi))))
    return np.stack(out, axis=-1)


def pair_weight(state: int, which: int) -> float:
    """The E4M3 weight of one state; which = 0 (first, P_a) or 1 (second, P_b)."""
    return float(pair_weights(np.array([state]))[0, which])


# ------------------------------------------------------------------ matrices

def decode_tiles(tiles, K: int) -> np.ndarray:
    """E4M3 values [n_tiles, 16, 16] (row, column) of tiles [n_tiles, 8K]."""
    st = pair_states_tiles(tiles, K)                       # [n, 128]
    w = pair_weights(st)                                   # [n, 128, 2]
    pos = w.reshape(w.shape[0], 256)                       # position p = 2q + which
    return pos.reshape(w.shape[0], 16, 16).transpose(0, 2, 1)   # column-major positions


def decode_matrix(bits, K: int, rows: int, cols: int) -> np.ndarray:
    """E4M3 values [rows, cols] of a bit stream of row-major 16x16 tiles (8K words each)."""
    tiles = np.asarray(bits, dtype=np.uint32).reshape((rows // 16) * (cols // 16), 8 * K)
    t = decode_tiles(tiles, K).reshape(rows // 16, cols // 16, 16, 16)
    return t.transpose(0, 2, 1, 3).reshape(rows, cols)


def dequantize(codes, scales) -> np.ndarray:
    """W[i, j] = s_i * 2^-5 * w[i, j] (fp64)."""
    return np.asarray(scales, dtype=np.float64)[:, None] * KAPPA8 * np.asarray(codes, dtype=np.float64)


# ------------------------------------------------------------------ activations (R26)

def row_scale_exponent(v) -> np.ndarray:
    """e per row with max |v| / 2^e in (224, 448] (0 for an all-zero row)."""
    v = np.atleast_2d(np.asarray(v, dtype=np.float64))
    m = np.abs(v).max(axis=1)
    e = np.zeros(m.shape, dtype=np.int64)
    nz = m > 0
    e[nz] = np.ceil(np.log2(m[nz] / E4M3_MAX)).astype(np.int64)
    # exact correction of the float estimate
    e[nz & (m / 2.0 ** e > E4M3_MAX)] += 1
    e[nz & (m / 2.0 ** (e - 1) <= E4M3_MAX)] -= 1
    return e


def quantize_rows_e4m3(v):
    """(v8, e): each row scaled by 2^-e (row_scale_exponent) and rounded to E4M3 (R26)."""
    v = np.atleast_2d(np.asarray(v, dtype=np.float64))
    e = row_scale_exponent(v)
    return e4m3_round(v / 2.0 ** e[:, None]), e
