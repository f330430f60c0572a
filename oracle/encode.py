"""Tail-biting Viterbi encoder for T16 bit streams -- test infrastructure (oracle).

Only tests/, the package's smoke check and bench.py's CPU baseline import this module.

Source: "DeepSeek-V4.1-Flash-1017 · dsx T16" model card, section "How T16 works": the
experts' bit streams are a QTIP-style bitshift trellis found by a Viterbi search, read
through the T16 codebook of item 1, and item 4 describes the quantizer as one that
minimises squared error.  The card gives no details of the search; the readings taken
here (listed in the design notes as R19) are:

* Objective, per 16x16 tile: sum over its 256 positions of (tau_p - 4 c_p)^2, where
  c_p is the centred T16 code of window p and tau_p = rint(4 * target_p) clamped to
  [-1276, 1276] is the target in quarter code units (exact integers; at most
  256 * 2296^2 < 2^32 per path).
* Trellis: the state is the 16-bit window; window p+1 = (window p >> K) | (u << (16-K))
  for the K new bits u (the same bitshift the decoder reads, LSB first), and the stream
  is tail-biting, so window 0's low 16-K bits are window 255's high 16-K bits.
* Search: pass 1 with every start and end window allowed.  If its best path already
  closes (window 0's low 16-K bits equal window 255's high 16-K bits) it is the answer.
  Otherwise two closed passes, with the closure bits b taken from pass 1's last window
  (b = w_255 >> K) and from its first (b = w_0 & (2^(16-K) - 1)): window 0 restricted
  to low bits b and only final windows with w >> K == b; the cheaper one wins, the
  first on a tie.  Ties inside a pass go to the smaller dropped bits (the smaller
  predecessor) and to the smaller final window.  Exact tail-biting would run a closed
  pass for all 2^(16-K) values of b; ``viterbi`` takes b so the tests can do that on
  small trellises (where the two-candidate choice lands 6-8 % above the exact optimum
  on average, against 17 % for a single candidate).

Everything is written for a general window width L (16 for T16) and a table of window
values, so small trellises can be checked against brute force.
"""
import numpy as np

from . import t16

TAU_MAX = 1276              # quarter code units: 4 * (255 + 64)
BIG = 1 << 31               # cost of a start window pass 2 does not allow

_codes = None


def code_table() -> np.ndarray:
    """Centred code c of every 16-bit window (from the oracle's T16 definition)."""
    global _codes
    if _codes is None:
        _codes = np.array([t16.code(w) for w in range(1 << 16)], dtype=np.int64)
    return _codes


def quarter_targets(x) -> np.ndarray:
    """Targets in code units -> integer quarter units tau (round half to even, clamped)."""
    return np.clip(np.rint(4.0 * np.asarray(x, dtype=np.float64)), -TAU_MAX, TAU_MAX).astype(np.int64)


def viterbi(tau, K: int, vals, L: int = 16, b=None):
    """Minimum of sum_p (tau_p - vals[w_p])^2 over window paths w_0..w_{n-1} of the
    bitshift trellis.  b=None: any start and end window; else window 0 has low L-K bits
    b and the last window has high L-K bits b.  Returns (cost, windows)."""
    tau = np.asarray(tau, dtype=np.int64)
    vals = np.asarray(vals, dtype=np.int64)
    n, S, G = len(tau), 1 << L, 1 << K
    mask = (1 << (L - K)) - 1
    states = np.arange(S, dtype=np.int64)
    cost = (tau[0] - vals) ** 2
    if b is not None:
        cost = np.where((states & mask) == b, cost, BIG)
    back = []
    for p in range(1, n):
        grp = cost.reshape(S // G, G)          # predecessors of low bits m: (m << K) | d
        arg = grp.argmin(axis=1)                # first minimum: the smaller d
        best = grp[np.arange(S // G), arg]
        cost = best[states & mask] + (tau[p] - vals) ** 2
        back.append(arg)
    if b is None:
        last = int(np.argmin(cost))
    else:
        cand = (b << K) | np.arange(G, dtype=np.int64)
        last = int(cand[np.argmin(cost[cand])])
    w = np.empty(n, dtype=np.int64)
    w[n - 1] = last
    for p in range(n - 1, 0, -1):
        m = w[p] & mask
        w[p - 1] = (m << K) | back[p - 1][m]
    return int(cost[last]), w


def encode_windows(tau, K: int, vals=None, L: int = 16):
    """Tail-biting search (pass 1, then up to two closed passes); returns
    (cost, windows, pass-1 cost)."""
    vals = 4 * code_table() if vals is None else vals
    mask = (1 << (L - K)) - 1
    c1, w1 = viterbi(tau, K, vals, L)
    b_end, b_start = int(w1[-1]) >> K, int(w1[0]) & mask
    if b_end == b_start:
        return c1, w1, c1
    ca, wa = viterbi(tau, K, vals, L, b=b_end)
    cb, wb = viterbi(tau, K, vals, L, b=b_start)
    return (ca, wa, c1) if ca <= cb else (cb, wb, c1)


def windows_to_bits(w, K: int, L: int = 16) -> np.ndarray:
    """Stream bits (n*K of them) whose window p is w[p]: bit j is bit j - pK of w_p, p = j // K."""
    n = len(w)
    j = np.arange(n * K)
    p = j // K
    return ((np.asarray(w, dtype=np.int64)[p] >> (j - p * K)) & 1).astype(np.uint8)


def bits_windows(bits, K: int, L: int = 16) -> np.ndarray:
    """Windows of a tail-biting stream: w_p = bits[pK .. pK+L) (mod n*K), LSB first."""
    bits = np.asarray(bits, dtype=np.int64)
    nb = len(bits)
    n = nb // K
    idx = (np.arange(n)[:, None] * K + np.arange(L)[None, :]) % nb
    return (bits[idx] << np.arange(L)[None, :]).sum(axis=1)


def pack_words(bits) -> np.ndarray:
    """Pack stream bits LSB first into little-endian uint32 words."""
    bits = np.asarray(bits, dtype=np.uint64).reshape(-1, 32)
    return (bits << np.arange(32, dtype=np.uint64)[None, :]).sum(axis=1).astype(np.uint32)


def encode_tile(target, K: int):
    """One 16x16 tile of targets (code units, [row][col]) -> (8K words, cost, pass-1 cost).
    Position p sits at row p % 16, column p // 16 (column-major in the tile)."""
    target = np.asarray(target, dtype=np.float64)
    tau = quarter_targets(target.T.reshape(-1))      # p = 16 * col + row
    cost, w, c1 = encode_windows(tau, K)
    words = pack_words(windows_to_bits(w, K))
    return words, cost, c1


def encode_matrix(target, K: int):
    """Targets [R][C] (code units) -> bit streams [R/16][C/16][8K] uint32 (row-major tiles)
    and the cost of every tile [R/16][C/16]."""
    target = np.asarray(target, dtype=np.float64)
    R, C = target.shape
    bits = np.zeros((R // 16, C // 16, 8 * K), dtype=np.uint32)
    costs = np.zeros((R // 16, C // 16), dtype=np.int64)
    for i in range(R // 16):
        for j in range(C // 16):
            words, cost, _ = encode_tile(target[16 * i:16 * i + 16, 16 * j:16 * j + 16], K)
            bits[i, j] = words
            costs[i, j] = cost
    return bits, costs
