"""Staged parity of the MoE layer at full size: each projection against the oracle on its
own input, in the launch configurations the benchmark times.

Stages (SwiGLU experts with fused gate/up post-processing, dsx T16 card "October 25
runtime checkpoint"; projections of "How T16 works", items 1, 2 and 4):
  1. gate/up: the GPU's g and u against the oracle's W x' (x' the fp64 rotation of the
     layer input), |g - g_ref| <= 1e-3 * (|W_g| . |x'|) elementwise;
  2. SwiGLU and rotation of h: the GPU's h' against rotate(silu(g_gpu) * u_gpu) in fp64,
     within its quantisation step (GEMV: 16-bit fixed point) or fp16 rounding (GEMM);
  3. down: y_perm against the oracle's W_d h'_gpu on the GPU's own h',
     |y - y_ref| <= 1e-3 * (|W_d| . |h'_gpu|);
  4. combine: out against the fp64 slot-order sum of the GPU's y_perm, to 1e-6 relative.
Sampled routes include the hottest and the coldest expert with routes.
"""
import numpy as np
import pytest
import torch

from oracle import layer as OL
from trellis_quantized_moe_gemv_b200 import inputs
from ws_layout import fixed_point_rows, fixed_point_values, gemm_views, gemv_views, route_experts

pytestmark = pytest.mark.gpu
EPS = 1e-3


@pytest.fixture(scope="module")
def api():
    import trellis_quantized_moe_gemv_b200.build as b
    b.build()
    from trellis_quantized_moe_gemv_b200 import api as A
    A.device_status(clear=True)
    return A


def run(api, w, path):
    layer, k = w["layer"], 8
    T = w["x"].shape[0]
    dl = api.DeviceLayer.from_synthetic(layer)
    bufs = api.MoeBuffers(dl, T, k)
    api.moe_layer(dl, torch.from_numpy(w["x"]).to(torch.bfloat16).cuda(), torch.from_numpy(w["logits"]).cuda(), k,
                  bufs=bufs, path=path)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    return dl, bufs


def sample_routes(bufs, n_random, seed):
    """Route positions (expert-grouped): the first route of the hottest and of the coldest
    expert with routes, plus n_random others."""
    counts = bufs.routing.counts.cpu().numpy()
    offsets = bufs.routing.offsets.cpu().numpy()
    hot = int(np.argmax(counts))
    cold = int(np.argmin(np.where(counts > 0, counts, np.iinfo(np.int32).max)))
    rng = np.random.default_rng(seed)
    picks = [int(offsets[hot]), int(offsets[cold])] + list(rng.choice(int(offsets[-1]), n_random, replace=False))
    return sorted(set(picks)), hot, cold


def check_combine(api, bufs, T):
    y = bufs.y_perm.cpu().numpy().astype(np.float64)
    out = bufs.out.cpu().numpy().astype(np.float64)
    inv = bufs.routing.inv.cpu().numpy()
    wts = bufs.w.cpu().numpy().astype(np.float64)
    ref = OL.combine(y, inv, wts)
    scale = np.zeros_like(ref)
    k = wts.shape[1]
    for s in range(k):
        scale += np.abs(wts[:, s:s + 1]) * np.abs(y[inv.reshape(T, k)[:, s]])
    assert np.all(np.abs(out - ref) <= 1e-6 * scale + 1e-30), (np.abs(out - ref) / (scale + 1e-30)).max()


def test_gemv_staged_full_size_decode_layer(api):
    w = inputs.moe_decode_t16()
    layer, k, T = w["layer"], 8, 16
    dl, bufs = run(api, w, "gemv")
    v = gemv_views(bufs.ws, T, k, layer.D, layer.F, layer.E)
    routes, hot, cold = sample_routes(bufs, 4, 6001)
    perm = bufs.routing.perm.cpu().numpy()
    experts = route_experts(bufs.routing.offsets.cpu().numpy())
    gu = v["gu"].cpu().numpy().astype(np.float64)
    fp = fixed_point_rows(v["hq"], v["hmeta"])
    h_rot_all = fixed_point_values(fp)
    y = bufs.y_perm.cpu().numpy().astype(np.float64)
    weights = OL.ExpertWeights(layer)
    x_rot = OL.rotate(w["x"].astype(np.float64))
    for j in routes:
        e, t = int(experts[j]), int(perm[j]) // k
        # 1. gate / up on the layer input
        for p, proj in enumerate(("gate", "up")):
            W = weights.matrix(e, proj)
            ref = OL.project(W, x_rot[t:t + 1])[0]
            tol = EPS * OL.abs_bound(W, x_rot[t:t + 1])[0]
            assert np.all(np.abs(gu[j, p] - ref) <= tol), (j, proj, (np.abs(gu[j, p] - ref) / tol).max())
        # 2. SwiGLU + rotation + 16-bit fixed point of h'
        h = OL.silu(gu[j, 0]) * gu[j, 1]
        h_rot_ref = OL.rotate(h[None])[0]
        h_rot = h_rot_all[j]
        step = 2.0 ** float(fp["e"][j] - (15 if fp["res"][j] else 0))
        tol = 0.5 * step * (1 + 1e-6) + 1e-5 * OL.rot_abs_bound(np.abs(h)[None])[0]
        assert np.all(np.abs(h_rot - h_rot_ref) <= tol), (j, (np.abs(h_rot - h_rot_ref) / tol).max())
        # 3. down on the GPU's own h'
        Wd = weights.matrix(e, "down")
        ref = OL.project(Wd, h_rot[None])[0]
        tol = EPS * OL.abs_bound(Wd, h_rot[None])[0]
        assert np.all(np.abs(y[j] - ref) <= tol), (j, (np.abs(y[j] - ref) / tol).max())
    # 4. combine
    check_combine(api, bufs, T)


def test_gemm_staged_full_size_prefill_layer(api):
    w = inputs.moe_prefill_t8192()
    layer, k, T = w["layer"], 8, 8192
    dl, bufs = run(api, w, "gemm")
    v = gemm_views(bufs.ws, T, k, layer.D, layer.F, two_sided=False)
    routes, hot, cold = sample_routes(bufs, 3, 6002)
    idx = torch.as_tensor(routes, dtype=torch.long, device="cuda")
    h = v["h"][idx].cpu().numpy().astype(np.float64)
    hr = v["hr"][idx].cpu().numpy().astype(np.float64) * v["hr_scale"][idx].cpu().numpy().astype(np.float64)[:, None]
    y = bufs.y_perm[idx].cpu().numpy().astype(np.float64)
    perm = bufs.routing.perm.cpu().numpy()
    experts = route_experts(bufs.routing.offsets.cpu().numpy())
    weights = OL.ExpertWeights(layer)
    for n, j in enumerate(routes):
        e, t = int(experts[j]), int(perm[j]) // k
        x_rot = OL.rotate(w["x"][t:t + 1].astype(np.float64))
        # 1. gate / up (the GEMM's epilogue applies the SwiGLU directly): h within the
        # SwiGLU propagation of the two projections' 1e-3 budgets, plus fp32 rounding
        Wg, Wu = weights.matrix(e, "gate"), weights.matrix(e, "up")
        g, u = OL.project(Wg, x_rot)[0], OL.project(Wu, x_rot)[0]
        dh = OL.swiglu_error_bound(g, u, EPS * OL.abs_bound(Wg, x_rot)[0], EPS * OL.abs_bound(Wu, x_rot)[0])
        ref = OL.silu(g) * u
        tol = dh + 1e-6 * np.abs(ref)
        assert np.all(np.abs(h[n] - ref) <= tol), (j, e, (np.abs(h[n] - ref) / tol).max())
        # 2. rotation of the GPU's h to fp16 h' (stored as h' / 2^e, largest magnitude in
        # [2^14, 2^15): fp16 keeps 11 significant bits down to 2^-14 of that, 2^-24 below)
        h_rot_ref = OL.rotate(h[n][None])[0]
        sc = float(v["hr_scale"][idx[n]].item())
        tol = 2.0 ** -11 * np.abs(h_rot_ref) + 2.0 ** -25 * sc + 1e-6 * OL.rot_abs_bound(np.abs(h[n])[None])[0]
        assert np.all(np.abs(hr[n] - h_rot_ref) <= tol), (j, (np.abs(hr[n] - h_rot_ref) / tol).max())
        # 3. down on the GPU's own h'
        Wd = weights.matrix(e, "down")
        ref = OL.project(Wd, hr[n][None])[0]
        tol = EPS * OL.abs_bound(Wd, hr[n][None])[0]
        assert np.all(np.abs(y[n] - ref) <= tol), (j, (np.abs(y[n] - ref) / tol).max())
    assert cold != hot
    # 4. combine (tokens of the sampled routes)
    y_all = bufs.y_perm
    inv = bufs.routing.inv.cpu().numpy().reshape(T, k)
    wts = bufs.w.cpu().numpy().astype(np.float64)
    toks = sorted({int(perm[j]) // k for j in routes})
    out = bufs.out[torch.as_tensor(toks, device="cuda")].cpu().numpy().astype(np.float64)
    for n, t in enumerate(toks):
        rows = y_all[torch.as_tensor(inv[t], dtype=torch.long, device="cuda")].cpu().numpy().astype(np.float64)
        ref = (wts[t][:, None] * rows).sum(0)
        scale = (np.abs(wts[t])[:, None] * np.abs(rows)).sum(0)
        assert np.all(np.abs(out[n] - ref) <= 1e-6 * scale + 1e-30)
