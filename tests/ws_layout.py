"""Views of the MoE entry points' device workspaces, for the staged parity tests.

The layouts are the library's (moe_trellis_workspace_size in include/trellis_moe.h
describes their contents); this module only slices the caller-owned workspace tensor
after a call.  Every region starts on a 256-byte boundary.
"""
import numpy as np
import torch


def _a256(n):
    return (n + 255) // 256 * 256


def _take(ws, off, nbytes, dtype, shape):
    t = ws[off:off + nbytes].view(dtype).reshape(shape)
    return t, off + _a256(nbytes)


def gate_up_splits(E, T, k, D, F):
    """Column splits of the GEMV's gate/up items (the library's rule): about 3 CTAs per SM
    at the largest possible number of active experts, at most 8 and at most D / 128."""
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    items = min(E, T * k) * (F // 64)
    want = -(-3 * sms // items)
    return max(1, min(8, want, D // 128))


def gemv_views(ws, T, k, D, F, E):
    """moe_trellis_gemv workspace: raw gate/up results gu [R][S][2][F] fp32 (R = T*k routes in
    expert-grouped order, S column splits whose partial sums add up to g and u), the
    quantised h' rows hq [R][4][F] (half-word planes holding the high and the low signed
    byte, each twice, of the main word x_q and of the residual word r_q) with meta [R][4]
    int32 (e, sum x_q, residual flag, sum r_q), and the quantised x' rows xq [T][4][D] with
    their meta."""
    R = T * k
    S = gate_up_splits(E, T, k, D, F)
    v = {"splits": S}
    off = 0
    v["gu_parts"], off = _take(ws, off, R * S * 2 * F * 4, torch.float32, (R, S, 2, F))
    v["gu"] = v["gu_parts"].sum(dim=1) if S > 1 else v["gu_parts"][:, 0]
    v["hq"], off = _take(ws, off, R * 4 * F * 2, torch.int16, (R, 4, F))
    v["hmeta"], off = _take(ws, off, R * 16, torch.int32, (R, 4))
    v["xq"], off = _take(ws, off, T * 4 * D * 2, torch.int16, (T, 4, D))
    v["xmeta"], off = _take(ws, off, T * 16, torch.int32, (T, 4))
    return v


def _signed_byte(p):
    return np.where(p >= 128, p - 256, p)


def fixed_point_rows(q, meta):
    """Words of quantised rows: dict(xq, rq int64 [n, cols], e, res int64 [n]); x_q = 256 hi + lo
    from planes 0 and 1, r_q likewise from planes 2 and 3 (zero unless res).  A row's value is
    x_q 2^e + r_q 2^(e - 15)."""
    q = q.cpu().numpy().astype(np.int64) & 0xFF
    m = meta.cpu().numpy().astype(np.int64)
    xq = 256 * _signed_byte(q[:, 0]) + _signed_byte(q[:, 1])
    rq = 256 * _signed_byte(q[:, 2]) + _signed_byte(q[:, 3])
    res = m[:, 2]
    rq = np.where(res[:, None] != 0, rq, 0)
    return dict(xq=xq, rq=rq, e=m[:, 0], res=res)


def fixed_point_values(fp):
    """fp64 values x_q 2^e + r_q 2^(e - 15) of fixed_point_rows."""
    e = fp["e"].astype(np.float64)[:, None]
    return fp["xq"] * 2.0 ** e + fp["rq"] * 2.0 ** (e - 15)


def gemm_views(ws, T, k, D, F, two_sided):
    """moe_trellis_gemm workspace: route-ordered fp16 x' rows xr [R][D] and their fp32 sums,
    then h [R][F] fp32 (two-sided: raw g and u [R][2][F]), the rotated h' rows stored as
    fp16 hr [R][F] = h' / hr_scale, their fp32 sums and the power-of-two scales hr_scale [R]."""
    R = T * k
    v = {}
    off = 0
    v["xr"], off = _take(ws, off, R * D * 2, torch.float16, (R, D))
    v["xr_sum"], off = _take(ws, off, R * 4, torch.float32, (R,))
    if two_sided:
        v["gu"], off = _take(ws, off, R * 2 * F * 4, torch.float32, (R, 2, F))
    else:
        v["h"], off = _take(ws, off, R * F * 4, torch.float32, (R, F))
    v["hr"], off = _take(ws, off, R * F * 2, torch.float16, (R, F))
    v["hr_sum"], off = _take(ws, off, R * 4, torch.float32, (R,))
    v["hr_scale"], off = _take(ws, off, R * 4, torch.float32, (R,))
    return v


def route_experts(offsets):
    """Expert of every expert-grouped route position, from route_permute's offsets."""
    off = np.asarray(offsets)
    counts = np.diff(off)
    return np.repeat(np.arange(counts.size), counts)


def gemm_views_e4m3(ws, T, k, D, F, two_sided):
    """moe_trellis_gemm workspace of a pair-trellis (E4M3) layer: the same regions as
    gemm_views, with the route-ordered x' rows as E4M3 bytes xr8 [R][D] and their
    power-of-two scales x_scale [R] (in the row-sum slot), and h' as E4M3 bytes hr8 [R][F]
    with hr_scale [R]."""
    R = T * k
    v = {}
    off = 0
    v["xr8"] = ws[0:R * D].view(torch.float8_e4m3fn).reshape(R, D)
    off = _a256(R * D * 2)
    v["x_scale"], off = _take(ws, off, R * 4, torch.float32, (R,))
    if two_sided:
        v["gu"], off = _take(ws, off, R * 2 * F * 4, torch.float32, (R, 2, F))
    else:
        v["h"], off = _take(ws, off, R * F * 4, torch.float32, (R, F))
    v["hr8"] = ws[off:off + R * F].view(torch.float8_e4m3fn).reshape(R, F)
    off += _a256(R * F * 2)
    off += _a256(R * 4)                      # h' row sums (unused by the E4M3 path)
    v["hr_scale"], off = _take(ws, off, R * 4, torch.float32, (R,))
    return v
