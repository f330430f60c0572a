"""The pair-trellis FP8 path (exlr8 card, "Stores": pmcgx, a pair trellis decoded to FP8
E4M3) through the C ABI: trellis_decode_e4m3 and moe_trellis_gemm with E4M3 operands on
kind::f8f6f4 tensor-core MMAs, against the oracle (oracle.pair_trellis, readings R20-R26).

  * decode: every code of 1024x4096 matrices at K = 2, 3, 4 equals the oracle's; the
    GEMM's own decode is exposed bit for bit by one-hot activations (x' = e_j scales to
    E4M3 256 exactly, so g = s * 2^-5 * w);
  * staged: the GPU's E4M3 x' rows and scales equal the oracle's rounding of the GPU's
    fp16 x'; each projection equals the exact sum over the GPU's own E4M3 activations up
    to fp32 accumulation; the GPU's E4M3 h' rows are the oracle's rounding of the GPU's h
    (a value sitting on a rounding boundary may differ by one E4M3 step);
  * layer: against the unquantised fp64 oracle within the oracle's propagated bound at
    the format's precision: E4M3 activations carry 2^-4 relative rounding (2^-10 of the
    row scale below the normal range), so eps_proj = 2^-4 + 2^-10.
"""
import numpy as np
import pytest
import torch

from oracle import layer as OL
from oracle import pair_trellis as PT
from trellis_quantized_moe_gemv_b200 import inputs
from ws_layout import gemm_views_e4m3, route_experts

pytestmark = pytest.mark.gpu
EPS_E4M3 = 2.0 ** -4 + 2.0 ** -10


@pytest.fixture(scope="module")
def api():
    import trellis_quantized_moe_gemv_b200.build as b
    b.build()
    from trellis_quantized_moe_gemv_b200 import api as A
    A.device_status(clear=True)
    return A


@pytest.mark.parametrize("K", [2, 3, 4])
def test_decode_e4m3_matches_oracle(api, K):
    rng = np.random.default_rng(8100 + K)
    rows, cols = 1024, 4096
    bits = inputs.random_bits(rng, rows, cols, K)[0]
    got = api.trellis_decode_e4m3(torch.from_numpy(bits.view(np.int32)).cuda(), K, rows, cols)
    torch.cuda.synchronize()
    got = got.float().cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(got, PT.decode_matrix(bits, K, rows, cols))


def test_decode_e4m3_small_and_ragged(api):
    for K, rows, cols, seed in ((2, 16, 16, 1), (3, 48, 80, 2), (4, 32, 16, 3)):
        bits = inputs.random_bits(np.random.default_rng(8200 + seed), rows, cols, K)[0]
        got = api.trellis_decode_e4m3(torch.from_numpy(bits.view(np.int32)).cuda(), K, rows, cols)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(got.float().cpu().numpy().astype(np.float64),
                                      PT.decode_matrix(bits, K, rows, cols))


def fp8_layer(seed, two_sided=False, E=6, D=512, F=256, split=None):
    layer = inputs.small_layer(seed, E=E, D=D, F=F, split=split or {2: 3, 3: 2, 4: 1}, codebook="pair_e4m3")
    if two_sided:
        inputs.with_signs(layer, seed + 1)
    return layer


def routes_for(T, k, E):
    return np.array([[(t + 2 * s) % E for s in range(k)] for t in range(T)], dtype=np.int32)


@pytest.mark.parametrize("T", [5, 300])
def test_gemm_gate_up_decode_one_hot(api, T):
    layer = fp8_layer(8301, two_sided=True)
    dl = api.DeviceLayer.from_synthetic(layer)
    weights = OL.ExpertWeights(layer)
    k, D, F = 3, layer.D, layer.F
    cols = (np.arange(T) * 53 + 11) % D
    x_rot = torch.zeros((T, D), dtype=torch.float16)
    x_rot[torch.arange(T), torch.as_tensor(cols, dtype=torch.long)] = 1.0
    routing = api.route_permute(torch.from_numpy(routes_for(T, k, layer.E)).cuda(), layer.E)
    ws = torch.zeros(api.moe_trellis_workspace_size(dl, T, k), dtype=torch.uint8, device="cuda")
    api.moe_trellis_gemm(dl, x_rot.cuda(), routing, T, k, ws=ws)
    torch.cuda.synchronize()
    gu = gemm_views_e4m3(ws, T, k, D, F, two_sided=True)["gu"].cpu().numpy().astype(np.float64)
    perm = routing.perm.cpu().numpy()
    experts = route_experts(routing.offsets.cpu().numpy())
    for j in range(T * k):
        e, t = int(experts[j]), int(perm[j]) // k
        for p, proj in enumerate(("gate", "up")):
            want = weights.matrix(e, proj)[:, cols[t]].astype(np.float32)   # s * 2^-5 * w, exact
            np.testing.assert_array_equal(gu[j, p].astype(np.float32), want,
                                          err_msg="route %d expert %d %s" % (j, e, proj))
    assert api.device_status() == 0


def run_fp8(api, layer, T, k, rng, routes=None):
    dl = api.DeviceLayer.from_synthetic(layer)
    x = inputs.random_activations(rng, (T, layer.D), "bf16")
    xd = torch.from_numpy(x).to(torch.bfloat16).cuda()
    x_rot = api.hadamard128_signed(xd, dl.signs["x"]) if layer.signs is not None else api.hadamard128(xd)
    ids = routes if routes is not None else routes_for(T, k, layer.E)
    routing = api.route_permute(torch.from_numpy(ids).cuda(), layer.E)
    ws = torch.zeros(api.moe_trellis_workspace_size(dl, T, k), dtype=torch.uint8, device="cuda")
    y = api.moe_trellis_gemm(dl, x_rot, routing, T, k, ws=ws)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    return dl, x, x_rot, routing, ws, y


@pytest.mark.parametrize("two_sided", [False, True])
def test_gemm_staged_against_exact_sums(api, two_sided):
    layer = fp8_layer(8401, two_sided=two_sided)
    T, k = 40, 3
    dl, x, x_rot, routing, ws, y = run_fp8(api, layer, T, k, np.random.default_rng(8402))
    v = gemm_views_e4m3(ws, T, k, layer.D, layer.F, two_sided)
    perm = routing.perm.cpu().numpy()
    experts = route_experts(routing.offsets.cpu().numpy())
    xr = x_rot.cpu().numpy().astype(np.float64)
    x8 = v["xr8"].float().cpu().numpy().astype(np.float64)
    xs = v["x_scale"].cpu().numpy().astype(np.float64)
    # 1. E4M3 route rows of x': the oracle's rounding of the GPU's fp16 x' (exact inputs)
    want8, we = PT.quantize_rows_e4m3(xr[perm // k])
    np.testing.assert_array_equal(x8, want8)
    np.testing.assert_array_equal(xs, 2.0 ** we)
    weights = OL.ExpertWeights(layer)
    y = y.cpu().numpy().astype(np.float64)
    h8 = v["hr8"].float().cpu().numpy().astype(np.float64)
    hs = v["hr_scale"].cpu().numpy().astype(np.float64)
    flips = 0
    for j in range(T * k):
        e = int(experts[j])
        xv = x8[j] * xs[j]
        # 2. gate / up: exact sums over the GPU's E4M3 x' (fp32 accumulation only)
        Wg, Wu = weights.matrix(e, "gate"), weights.matrix(e, "up")
        g_ref, u_ref = Wg @ xv, Wu @ xv
        sg, su = np.abs(Wg) @ np.abs(xv), np.abs(Wu) @ np.abs(xv)
        if two_sided:
            g, u = v["gu"][j, 0].cpu().numpy(), v["gu"][j, 1].cpu().numpy()
            assert np.all(np.abs(g - g_ref) <= 1e-5 * sg + 1e-30), j
            assert np.all(np.abs(u - u_ref) <= 1e-5 * su + 1e-30), j
            g = OL.rotate_out(g[None].astype(np.float64), layer.signs["gu"])[0]
            u = OL.rotate_out(u[None].astype(np.float64), layer.signs["gu"])[0]
            h = OL.silu(g) * u
            h_rot = OL.rotate_in(h[None], layer.signs["h"])[0]
        else:
            h = v["h"][j].cpu().numpy().astype(np.float64)
            dh = OL.swiglu_error_bound(g_ref, u_ref, 1e-5 * sg, 1e-5 * su)
            assert np.all(np.abs(h - OL.silu(g_ref) * u_ref) <= dh + 1e-6 * np.abs(h) + 1e-30), j
            h_rot = OL.rotate(h[None])[0]
        # 3. E4M3 h' rows: the oracle's rounding of the rotated GPU h (one E4M3 step where
        # the fp32 and fp64 rotations fall on either side of a rounding boundary)
        ref8, re = PT.quantize_rows_e4m3(h_rot[None])
        assert hs[j] == 2.0 ** re[0]
        diff = h8[j] != ref8[0]
        flips += int(diff.sum())
        step = np.where(np.abs(ref8[0]) < 2.0 ** -5, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref8[0]), 2.0 ** -5))) - 3))
        assert np.all(np.abs(h8[j] - ref8[0])[diff] <= step[diff] * (1 + 1e-12)), j
        # 4. down: exact sums over the GPU's own E4M3 h'
        Wd = weights.matrix(e, "down")
        hv = h8[j] * hs[j]
        y_ref = Wd @ hv
        assert np.all(np.abs(y[j] - y_ref) <= 1e-5 * (np.abs(Wd) @ np.abs(hv)) + 1e-30), j
    assert flips <= 1e-3 * T * k * layer.F, flips


@pytest.mark.parametrize("two_sided", [False, True])
@pytest.mark.parametrize("T", [7, 200])
def test_layer_against_fp64_oracle(api, two_sided, T):
    layer = fp8_layer(8501 + T, two_sided=two_sided, E=8, D=512, F=256, split={2: 4, 3: 3, 4: 1})
    rng = np.random.default_rng(8502 + T)
    x = inputs.random_activations(rng, (T, 512), "bf16")
    logits = inputs.normal_logits(rng, T, 8)
    dl = api.DeviceLayer.from_synthetic(layer)
    bufs = api.MoeBuffers(dl, T, 3)
    out = api.moe_layer(dl, torch.from_numpy(x).to(torch.bfloat16).cuda(), torch.from_numpy(logits).cuda(), 3,
                        bufs=bufs, path="auto")
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    toks = np.arange(T) if T <= 16 else np.random.default_rng(1).choice(T, 12, replace=False)
    res = OL.moe_tokens(layer, x, logits, 3, toks, eps_proj=EPS_E4M3)
    np.testing.assert_array_equal(bufs.ids.cpu().numpy()[toks], res["topk_ids"][toks])
    tol = res["bound"] + 1e-6 * np.abs(res["out"]) + 1e-12
    err = np.abs(got[toks] - res["out"])
    assert np.all(err <= tol), "max err/tol %.3e" % (err / tol).max()
    assert api.device_status() == 0


def test_full_size_prefill_layer_sampled_tokens(api):
    # the prefill layer shape with pair-trellis K = 3 streams, 8192 Zipf-routed tokens
    w = inputs.moe_prefill_t8192_fp8()
    dl = api.DeviceLayer.from_synthetic(w["layer"])
    T, k = 8192, 8
    bufs = api.MoeBuffers(dl, T, k)
    out = api.moe_layer(dl, torch.from_numpy(w["x"]).to(torch.bfloat16).cuda(), torch.from_numpy(w["logits"]).cuda(),
                        k, bufs=bufs, path="gemm")
    torch.cuda.synchronize()
    assert api.device_status() == 0
    counts = bufs.routing.counts.cpu().numpy()
    ids = bufs.ids.cpu().numpy()
    hot = int(np.argmax(counts))
    cold = int(np.argmin(np.where(counts > 0, counts, np.iinfo(np.int32).max)))
    # one token (the oracle decodes its 8 experts' 24 matrices): the first routed to the
    # hottest expert; the cold end is covered by the staged test's small experts
    toks = [int(np.nonzero((ids == hot).any(1))[0][0])]
    assert cold != hot
    res = OL.moe_tokens(w["layer"], w["x"][toks], w["logits"][toks], k, np.arange(len(toks)), eps_proj=EPS_E4M3)
    got = out[torch.as_tensor(toks, device="cuda")].cpu().numpy().astype(np.float64)
    tol = res["bound"] + 1e-6 * np.abs(res["out"]) + 1e-12
    assert np.all(np.abs(got - res["out"]) <= tol)


def test_gemv_rejects_pair_trellis_layers(api):
    layer = fp8_layer(8601)
    dl = api.DeviceLayer.from_synthetic(layer)
    T, k = 4, 3
    x_rot = torch.zeros((T, layer.D), dtype=torch.float16, device="cuda")
    routing = api.route_permute(torch.from_numpy(routes_for(T, k, layer.E)).cuda(), layer.E)
    with pytest.raises(api.TQError, match="UNSUPPORTED"):
        api.moe_trellis_gemv(dl, x_rot, routing, T, k)
