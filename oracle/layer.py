"""fp64 CPU oracle of the trellis-coded MoE layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference arm of
``bench.py`` may use this module.  The product path never imports it.

Sources (web pages on trellis-coded MoE experts):
  * "DeepSeek-V4.1-Flash-1017 · dsx T16", "How T16 works": experts quantised with a
    QTIP-style bitshift trellis and 128-wide Hadamard rotations (intro paragraph),
    T16 codebook (item 1), column-major 16x16 tiles (item 2), each output's stored
    scale (item 4).  Section "October 25 runtime checkpoint": warp Hadamard
    transforms and fused gate/up post-processing for the routed experts.
  * "DeepSeek-V4.1-Flash-1017 · exlr8", "Stores": 128 x 128 Hadamard rotation,
    per-channel scales.
  * "DeepSeek-V4.1-Flash-1017 TrellisMX K2 Mix", "What is stored": one tensor
    group per width present in a layer, each with its ascending global expert ids.

Where the pages are silent the plainest reading is taken (the readings are listed in
the project's design notes):
  * kappa = 2**-12 multiplies every code (W_ij = s_i * kappa * c_ij).
  * H_128 is the natural-order Sylvester matrix, H[a][b] = (-1)**popcount(a & b),
    applied as (1/sqrt(128)) * H to each contiguous 128-chunk of a projection's input.
  * Routing keeps the top-k logits (ties to the lower expert id); route weights are the
    softmax of the k kept logits.
  * The expert is SwiGLU: h = silu(gate(x')) * up(x'); the down projection reads the
    rotated h' = rotate(h).
  * Routes are grouped by expert, stable in (token, slot) order; the combine sums the k
    slots of a token in slot order.

Everything is fp64 numpy; numpy's matmul and stable sort are the only library
primitives used as steps.
"""
import numpy as np

from . import pair_trellis, t16

KAPPA = 2.0 ** -12
HADAMARD_N = 128

_H_CACHE = {}


def hadamard_matrix(n: int = HADAMARD_N) -> np.ndarray:
    """Explicit natural-order Sylvester matrix, entries (-1)**popcount(a & b)."""
    if n not in _H_CACHE:
        H = np.empty((n, n), dtype=np.float64)
        for a in range(n):
            for b in range(n):
                H[a, b] = -1.0 if bin(a & b).count("1") % 2 else 1.0
        _H_CACHE[n] = H
    return _H_CACHE[n]


def rotate(x) -> np.ndarray:
    """x'_chunk = (1/sqrt(128)) * H_128 @ x_chunk for every contiguous 128-chunk of
    the last axis (fp64)."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    if n % HADAMARD_N:
        raise ValueError("last axis must be a multiple of 128")
    H = hadamard_matrix()
    chunks = x.reshape(x.shape[:-1] + (n // HADAMARD_N, HADAMARD_N))
    out = np.einsum("ab,...b->...a", H, chunks) / np.sqrt(float(HADAMARD_N))
    return out.reshape(x.shape)


def rotate_in(x, signs=None) -> np.ndarray:
    """Input side of a projection: rotate(signs * x) (signs None: rotate(x))."""
    x = np.asarray(x, dtype=np.float64)
    return rotate(x if signs is None else x * np.asarray(signs, dtype=np.float64))


def rotate_out(v, signs=None) -> np.ndarray:
    """Output side of a projection in the two-sided transform: signs * rotate(v)
    (signs None: v unchanged, the input-side-only layer)."""
    v = np.asarray(v, dtype=np.float64)
    return v if signs is None else rotate(v) * np.asarray(signs, dtype=np.float64)


def dequantize(codes, scales) -> np.ndarray:
    """W[i, j] = s_i * kappa * c[i, j] (fp64); scales are fp16 values."""
    s = np.asarray(scales, dtype=np.float64)
    return s[:, None] * KAPPA * np.asarray(codes, dtype=np.float64)


def project(W, x_rot) -> np.ndarray:
    """y[b, i] = sum_j W[i, j] * x'[b, j] (fp64)."""
    return np.asarray(x_rot, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T


def abs_bound(W, x_rot) -> np.ndarray:
    """(|W| . |x'|)[b, i] = sum_j |W[i, j]| * |x'[b, j]|, the scale of the tolerance."""
    return np.abs(np.asarray(x_rot, dtype=np.float64)) @ np.abs(np.asarray(W, dtype=np.float64)).T


def single_projection(bits, K, rows, cols, scales, x):
    """One trellis-coded matrix times rotated activations: y = s * kappa * (C @ (H x)).

    Returns (y [B, rows], bound [B, rows]) with bound = |W| . |x'|.
    """
    codes = t16.decode_matrix(bits, K, rows, cols)
    W = dequantize(codes, scales)
    x_rot = rotate(np.atleast_2d(np.asarray(x, dtype=np.float64)))
    return project(W, x_rot), abs_bound(W, x_rot)


# ----------------------------------------------------------------------------- routing

def route_topk(logits, k: int):
    """Top-k experts per token (largest logit first, ties to the lower id) and the
    softmax of the k kept logits (fp64)."""
    L = np.asarray(logits, dtype=np.float64)
    T, E = L.shape
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    expert_index = np.arange(E)
    for t in range(T):
        order = np.lexsort((expert_index, -L[t]))   # primary: -logit, then id
        sel = order[:k]
        ids[t] = sel
        z = L[t, sel] - L[t, sel].max()
        e = np.exp(z)
        w[t] = e / e.sum()
    return ids, w


def route_permute(topk_ids, E: int):
    """Group the T*k (token, slot) pairs by expert, stable in pair order.

    Pair index i = t*k + s.  Returns counts[E], offsets[E+1], perm (sorted pair
    indices) and inv (inv[perm[j]] = j).
    """
    experts = np.asarray(topk_ids, dtype=np.int64).reshape(-1)
    perm = np.argsort(experts, kind="stable").astype(np.int32)
    counts = np.bincount(experts, minlength=E).astype(np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int32)
    return counts, offsets, perm, inv


def combine(y_perm, inv, topk_w):
    """out[t] = sum_s w[t, s] * y_perm[inv[t*k + s]], summed in slot order (fp64)."""
    y = np.asarray(y_perm, dtype=np.float64)
    w = np.asarray(topk_w, dtype=np.float64)
    T, k = w.shape
    inv = np.asarray(inv).reshape(T, k)
    out = np.zeros((T, y.shape[1]))
    for s in range(k):
        out += w[:, s:s + 1] * y[inv[:, s]]
    return out


# ----------------------------------------------------------------------------- experts

def silu(z):
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def silu_prime(z):
    z = np.asarray(z, dtype=np.float64)
    s = 1.0 / (1.0 + np.exp(-z))
    return s * (1.0 + z * (1.0 - s))


class ExpertWeights:
    """Decoded fp64 weights of one synthetic layer's experts, decoded on first use.

    The layer object carries, per width group g: K, ascending expert ``ids`` and the
    stored arrays ``gate``/``up`` [n, F/16*D/16*8K], ``down`` [n, D/16*F/16*8K] (uint32)
    and ``s_gate``/``s_up`` [n, F], ``s_down`` [n, D] (fp16).
    """

    def __init__(self, layer):
        self.layer = layer
        self._cache = {}
        self._where = {}
        for g in layer.groups:
            for idx, e in enumerate(g.ids):
                self._where[int(e)] = (g, idx)

    def width(self, e: int) -> int:
        return int(self._where[int(e)][0].K)

    def matrix(self, e: int, proj: str) -> np.ndarray:
        key = (int(e), proj)
        if key not in self._cache:
            g, idx = self._where[int(e)]
            D, F = self.layer.D, self.layer.F
            rows, cols = (F, D) if proj in ("gate", "up") else (D, F)
            bits = getattr(g, proj)[idx]
            scales = getattr(g, "s_" + proj)[idx]
            if getattr(self.layer, "codebook", "t16") == "pair_e4m3":
                # the exlr8 card's pair trellis decoded to E4M3, W = s * 2^-5 * w
                self._cache[key] = pair_trellis.dequantize(pair_trellis.decode_matrix(bits, g.K, rows, cols), scales)
            else:
                self._cache[key] = dequantize(t16.decode_matrix(bits, g.K, rows, cols), scales)
        return self._cache[key]

    def down_rows(self, e: int, row_ids) -> np.ndarray:
        """Selected rows of the down projection (fp64), without decoding the rest."""
        if getattr(self.layer, "codebook", "t16") == "pair_e4m3":
            return self.matrix(e, "down")[np.asarray(row_ids)]
        g, idx = self._where[int(e)]
        D, F = self.layer.D, self.layer.F
        codes = t16.decode_rows(g.down[idx], g.K, D, F, row_ids)
        s = np.asarray(g.s_down[idx], dtype=np.float64)[np.asarray(row_ids)]
        return s[:, None] * KAPPA * codes.astype(np.float64)


def expert_forward(weights: ExpertWeights, e: int, x_rot, down_rows=None, signs=None):
    """SwiGLU expert on rotated token rows x_rot [n, D].

    signs: the layer's sign vectors (dict x, gu, h, y) of the two-sided transform, or
    None (input side only).  Two-sided: g = s_gu * rotate(W_g x'), u likewise,
    h' = rotate(s_h * h), y = s_y * rotate(W_d h').
    Returns a dict with g, u, h, h_rot (fp64) and y [n, D or len(down_rows)], plus the
    per-projection tolerance scales bound_g, bound_u, bound_y = |W| . |input| (of the
    projections before their output rotation).
    """
    two = signs is not None
    Wg = weights.matrix(e, "gate")
    Wu = weights.matrix(e, "up")
    g_raw = project(Wg, x_rot)
    u_raw = project(Wu, x_rot)
    g = rotate_out(g_raw, signs["gu"] if two else None)
    u = rotate_out(u_raw, signs["gu"] if two else None)
    h = silu(g) * u
    h_rot = rotate_in(h, signs["h"] if two else None)
    if down_rows is None:
        rows = None
    elif two:
        # the output rotation mixes 128 consecutive rows: compute whole 128-row chunks
        chunks = np.unique(np.asarray(down_rows) // HADAMARD_N)
        rows = (chunks[:, None] * HADAMARD_N + np.arange(HADAMARD_N)[None, :]).reshape(-1)
    else:
        rows = np.asarray(down_rows)
    Wd = weights.matrix(e, "down") if rows is None else weights.down_rows(e, rows)
    y_raw = project(Wd, h_rot)
    if two:
        if rows is None:
            y = rotate_out(y_raw, signs["y"])
        else:
            y_rows = rotate(y_raw) * np.asarray(signs["y"], dtype=np.float64)[rows]
            pos = {int(r): i for i, r in enumerate(rows)}
            sel = [pos[int(r)] for r in down_rows]
            y = y_rows[:, sel]
    else:
        y = y_raw
    return dict(g=g, u=u, h=h, h_rot=h_rot, y=y, two_sided=two, rows=rows, down_rows=down_rows,
                bound_g=abs_bound(Wg, x_rot), bound_u=abs_bound(Wu, x_rot),
                bound_y=abs_bound(Wd, h_rot), Wd=Wd)


def rot_abs_bound(v) -> np.ndarray:
    """Elementwise bound on |rotate(dv)| given |dv| <= v elementwise: every output of a
    128-chunk's orthonormal rotation is a +-1/sqrt(128) combination of that chunk's
    inputs, so |rotate(dv)_j| <= (sum of v over j's chunk) / sqrt(128).  The bound is
    attained at j by dv = v * (sign pattern of H_128's row j within the chunk)."""
    v = np.asarray(v, dtype=np.float64)
    n = v.shape[-1]
    chunk = v.reshape(v.shape[:-1] + (n // HADAMARD_N, HADAMARD_N)).sum(-1)
    return np.repeat(chunk, HADAMARD_N, axis=-1) / np.sqrt(float(HADAMARD_N))


_rot_abs = rot_abs_bound


SILU_D2_MAX = 0.5    # max |silu''(z)| (attained at z = 0)


def swiglu_error_bound(g, u, dg, du) -> np.ndarray:
    """Elementwise bound on |silu(g + a) * (u + b) - silu(g) * u| for |a| <= dg, |b| <= du.

    silu(g + a) * (u + b) - silu(g) * u = (silu(g + a) - silu(g)) * (u + b) + silu(g) * b, and
    by Taylor's theorem |silu(g + a) - silu(g)| <= |silu'(g)| dg + (max|silu''| / 2) dg^2, so
    the change is at most (|silu'(g)| dg + 0.25 dg^2) (|u| + du) + |silu(g)| du."""
    g, u = np.asarray(g, dtype=np.float64), np.asarray(u, dtype=np.float64)
    dsilu = np.abs(silu_prime(g)) * dg + 0.5 * SILU_D2_MAX * dg * dg
    return dsilu * (np.abs(u) + du) + np.abs(silu(g)) * du


def e2e_error_bound(stage, eps_proj: float, w_abs):
    """First-order-exact bound on |out_gpu - out| of one route's contribution, given that
    each projection meets |dy| <= eps_proj * (|W| . |input|) (h' rounding included).

    The projection errors are carried through the layer stage by stage:
      * gate/up: dg = eps * (|W_g| . |x'|), du likewise; with the two-sided transform the
        raw projections' errors are spread by their output rotations (rot_abs_bound);
      * SwiGLU: dh = swiglu_error_bound(g, u, dg, du);
      * rotation of h: |d h'| <= rot_abs_bound(dh);
      * down: its own budget applies to the perturbed input, eps * (|W_d| . (|h'| + |dh'|)), so
        |dy| <= (1 + eps) |W_d| . rot_abs_bound(dh) + eps * (|W_d| . |h'|), spread by the down
        projection's output rotation when two-sided.

    stage: the dict of ``expert_forward`` for that route's rows; w_abs: |route weight|.
    Returns the bound for the route's y scaled by its weight.
    """
    g, u = stage["g"], stage["u"]
    dg = eps_proj * stage["bound_g"]
    du = eps_proj * stage["bound_u"]
    if stage.get("two_sided"):
        # errors of the raw projections spread by their output rotation
        dg, du = rot_abs_bound(dg), rot_abs_bound(du)
    dh = swiglu_error_bound(g, u, dg, du)
    dh_rot = rot_abs_bound(dh)
    dy = (1.0 + eps_proj) * (dh_rot @ np.abs(stage["Wd"]).T) + eps_proj * stage["bound_y"]
    if stage.get("two_sided"):
        dy = rot_abs_bound(dy)
        if stage.get("down_rows") is not None:
            pos = {int(r): i for i, r in enumerate(stage["rows"])}
            dy = dy[:, [pos[int(r)] for r in stage["down_rows"]]]
    return w_abs[:, None] * dy


# ----------------------------------------------------------------------------- layer

def moe_tokens(layer, x, logits, k: int, token_ids, weights: ExpertWeights = None,
               down_rows=None, eps_proj: float = 1e-3):
    """fp64 MoE layer output for selected tokens.

    x: [T, D] activations (bf16/fp16 values as float), logits: [T, E] fp32.
    Returns dict(out [n_tok, D or len(down_rows)], bound [same], topk_ids, topk_w).
    """
    weights = weights or ExpertWeights(layer)
    signs = getattr(layer, "signs", None)
    ids, w = route_topk(logits, k)
    token_ids = np.asarray(token_ids)
    x_rot = rotate_in(np.asarray(x, dtype=np.float64)[token_ids], signs["x"] if signs is not None else None)
    n_out = layer.D if down_rows is None else len(down_rows)
    out = np.zeros((token_ids.size, n_out))
    bound = np.zeros((token_ids.size, n_out))
    for a, t in enumerate(token_ids):
        for s in range(k):
            st = expert_forward(weights, int(ids[t, s]), x_rot[a:a + 1], down_rows, signs)
            out[a] += w[t, s] * st["y"][0]
            bound[a] += e2e_error_bound(st, eps_proj, np.abs(w[t, s:s + 1]))[0]
    return dict(out=out, bound=bound, topk_ids=ids, topk_w=w)


def moe_layer(layer, x, logits, k: int, eps_proj: float = 1e-3):
    """fp64 MoE layer output for every token (small layers / token counts only)."""
    T = np.asarray(x).shape[0]
    return moe_tokens(layer, x, logits, k, np.arange(T), eps_proj=eps_proj)
