"""Bit-exact checks of the T16 decode inside the hot-path kernels, through the C ABI.

The single-projection GEMV, the MoE GEMV and the MoE GEMM decode the trellis in their
own code (registers, or swizzled shared memory), not through trellis_decode.  Fed with
one-hot rotated activations, their contractions are exact:
  * GEMV: x_q = 2^14 exactly, the int32 sums hold t * 2^14, and the epilogue forms
    s * 2^-12 * 2^-14 * (2^14 t - 255 * 2^14) = s * 2^-12 * c;
  * GEMM: the fp32 accumulator holds t * 2^-24 (one fp16 subnormal product), the epilogue
    forms s * 2^-12 * (2^24 D - 255 * 1) = s * 2^-12 * c;
so every output equals s * 2^-12 * c (at most 20 significant bits, exact in fp32) for the
code c of the weight that the one-hot column selects, and is compared bit for bit with the
oracle's decode ("How T16 works", items 1 and 2 of the dsx T16 card: the T16 value of
each weight's 16-bit window, column-major positions in 16x16 tiles).

The down projection of the MoE GEMV contracts the GPU's own quantised h' (16-bit fixed
point x_q * 2^e): its integer sum sum_f c[d][f] * x_q[f] is exact and the epilogue scales
it by s * 2^-12 * 2^e in double (exact: < 53 significant bits) before one rounding to fp32,
so y_perm is reproduced bit for bit from the oracle's codes and the GPU's h'.
"""
import numpy as np
import pytest
import torch

from oracle import t16 as OT
from trellis_quantized_moe_gemv_b200 import inputs
from ws_layout import fixed_point_rows, gemm_views, gemv_views, route_experts

pytestmark = pytest.mark.gpu

KAPPA = 2.0 ** -12


@pytest.fixture(scope="module")
def api():
    import trellis_quantized_moe_gemv_b200.build as b
    b.build()
    from trellis_quantized_moe_gemv_b200 import api as A
    A.device_status(clear=True)
    return A


def weights_f32(codes, scales):
    """s * 2^-12 * c, exact in float64 and in float32."""
    return (scales.astype(np.float64)[:, None] * KAPPA * codes).astype(np.float32)


def one_hot(rows, cols, columns):
    x = torch.zeros((rows, cols), dtype=torch.float16)
    x[torch.arange(rows), torch.as_tensor(columns, dtype=torch.long)] = 1.0
    return x.cuda()


@pytest.mark.parametrize("K", [2, 3, 4])
def test_trellis_gemv_one_hot_rows_give_every_decoded_weight(api, K):
    # 8 routes per pass (batch > 4): the 1024x4096 projection against all 4096 one-hot
    # rows, so y^T is the whole dequantised matrix
    rng = np.random.default_rng(5100 + K)
    rows, cols = 1024, 4096
    bits = inputs.random_bits(rng, rows, cols, K)[0]
    scales = inputs.random_scales(rng, rows)
    W = weights_f32(OT.decode_matrix(bits, K, rows, cols), scales)
    bd = torch.from_numpy(bits.view(np.int32)).cuda()
    sd = torch.from_numpy(scales).cuda()
    y = api.trellis_gemv(bd, sd, K, rows, cols, one_hot(cols, cols, np.arange(cols)))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y.cpu().numpy(), W.T)
    assert api.device_status() == 0


@pytest.mark.parametrize("K", [2, 3, 4])
def test_trellis_gemv_one_hot_batches_of_four(api, K):
    # 4 routes per pass (batch <= 4): 64 calls of 4 one-hot rows cover every column of a
    # 256x256 matrix
    rng = np.random.default_rng(5200 + K)
    n = 256
    bits = inputs.random_bits(rng, n, n, K)[0]
    scales = inputs.random_scales(rng, n)
    W = weights_f32(OT.decode_matrix(bits, K, n, n), scales)
    bd = torch.from_numpy(bits.view(np.int32)).cuda()
    sd = torch.from_numpy(scales).cuda()
    order = rng.permutation(n)
    for q in range(n // 4):
        cols = order[4 * q:4 * q + 4]
        y = api.trellis_gemv(bd, sd, K, n, n, one_hot(4, n, cols))
        torch.cuda.synchronize()
        np.testing.assert_array_equal(y.cpu().numpy(), W[:, cols].T, err_msg="columns %s" % cols)


def mixed_layer():
    return inputs.small_layer(5301, E=6, D=512, F=256, split={2: 3, 3: 2, 4: 1})


def decoded(layer):
    """{(expert, proj): s * 2^-12 * c (float32)} from the oracle's decode."""
    out = {}
    for g in layer.groups:
        for i, e in enumerate(g.ids):
            for proj, (r, c) in (("gate", (layer.F, layer.D)), ("up", (layer.F, layer.D)),
                                 ("down", (layer.D, layer.F))):
                codes = OT.decode_matrix(getattr(g, proj)[i], g.K, r, c)
                out[(int(e), proj)] = (codes, getattr(g, "s_" + proj)[i])
    return out


def routes_for(T, k, E):
    """Every token routed to k distinct experts, cycling over all experts."""
    return np.array([[(t + 2 * s) % E for s in range(k)] for t in range(T)], dtype=np.int32)


@pytest.mark.parametrize("T", [4, 64])      # 4 routes per pass (12 routes) / 8 (192 routes)
def test_moe_gemv_gate_up_decode_one_hot(api, T):
    layer = mixed_layer()
    dec = decoded(layer)
    dl = api.DeviceLayer.from_synthetic(layer)
    k = 3
    D, F = layer.D, layer.F
    cols = (np.arange(T) * 37 + 5) % D                    # spread over lanes, tiles, chunks
    x_rot = one_hot(T, D, cols)
    routing = api.route_permute(torch.from_numpy(routes_for(T, k, layer.E)).cuda(), layer.E)
    ws = torch.zeros(api.moe_trellis_workspace_size(dl, T, k), dtype=torch.uint8, device="cuda")
    api.moe_trellis_gemv(dl, x_rot, routing, T, k, ws=ws)
    torch.cuda.synchronize()
    v = gemv_views(ws, T, k, D, F, layer.E)
    gu = v["gu"].cpu().numpy()
    perm = routing.perm.cpu().numpy()
    experts = route_experts(routing.offsets.cpu().numpy())
    for j in range(T * k):
        e, t = int(experts[j]), int(perm[j]) // k
        for p, proj in enumerate(("gate", "up")):
            codes, s = dec[(e, proj)]
            want = weights_f32(codes[:, cols[t]:cols[t] + 1], s)[:, 0]
            np.testing.assert_array_equal(gu[j, p], want, err_msg="route %d expert %d %s" % (j, e, proj))
    assert api.device_status() == 0


def exact_down_from_fixed_point(codes, scales, fp, j):
    """y[d] = fp32(s_d * 2^-12 * 2^e * a_d), a_d = sum_f c[d][f] x_q[f] (integer), or for a
    two-word row 2^-15 (2^15 a_d + sum_f c[d][f] r_q[f]) (exact below 2^53): the double
    product with the scale is rounded once, then to fp32, as the kernel's epilogue does."""
    c = codes.astype(np.int64)
    a = c @ fp["xq"][j]
    e = int(fp["e"][j])
    if fp["res"][j]:
        a = a * 2 ** 15 + c @ fp["rq"][j]
        e -= 15
    assert np.abs(a).max() < 2 ** 53
    return (a.astype(np.float64) * scales.astype(np.float64) * 2.0 ** (e - 12)).astype(np.float32)


@pytest.mark.parametrize("T", [4, 64])
def test_moe_gemv_down_bit_exact_on_its_own_h(api, T):
    layer = mixed_layer()
    dec = decoded(layer)
    dl = api.DeviceLayer.from_synthetic(layer)
    k = 3
    D, F = layer.D, layer.F
    rng = np.random.default_rng(5400 + T)
    x = inputs.random_activations(rng, (T, D), "bf16")
    x_rot = api.hadamard128(torch.from_numpy(x).to(torch.bfloat16).cuda())
    routing = api.route_permute(torch.from_numpy(routes_for(T, k, layer.E)).cuda(), layer.E)
    ws = torch.zeros(api.moe_trellis_workspace_size(dl, T, k), dtype=torch.uint8, device="cuda")
    y = api.moe_trellis_gemv(dl, x_rot, routing, T, k, ws=ws)
    torch.cuda.synchronize()
    v = gemv_views(ws, T, k, D, F, layer.E)
    fp = fixed_point_rows(v["hq"], v["hmeta"])
    y = y.cpu().numpy()
    experts = route_experts(routing.offsets.cpu().numpy())
    for j in range(T * k):
        codes, s = dec[(int(experts[j]), "down")]
        want = exact_down_from_fixed_point(codes, s, fp, j)
        np.testing.assert_array_equal(y[j], want, err_msg="route %d" % j)


def test_moe_gemv_down_bit_exact_full_size_decode_layer(api):
    # The 384-expert mixed-width layer at 16 tokens (the benchmark's launch configuration):
    # sampled routes of each width, reproduced bit for bit from the GPU's own h'
    w = inputs.moe_decode_t16()
    layer, k, T = w["layer"], 8, 16
    dl = api.DeviceLayer.from_synthetic(layer)
    bufs = api.MoeBuffers(dl, T, k)
    api.moe_layer(dl, torch.from_numpy(w["x"]).to(torch.bfloat16).cuda(), torch.from_numpy(w["logits"]).cuda(), k,
                  bufs=bufs, path="gemv")
    torch.cuda.synchronize()
    v = gemv_views(bufs.ws, T, k, layer.D, layer.F, layer.E)
    fp = fixed_point_rows(v["hq"], v["hmeta"])
    y = bufs.y_perm.cpu().numpy()
    experts = route_experts(bufs.routing.offsets.cpu().numpy())
    K_of = {int(e): g.K for g in layer.groups for e in g.ids}
    picked = {}
    for j, e in enumerate(experts):
        picked.setdefault(K_of[int(e)], [])
        if len(picked[K_of[int(e)]]) < 3:
            picked[K_of[int(e)]].append(j)
    where = {int(e): (g, i) for g in layer.groups for i, e in enumerate(g.ids)}
    for K, js in picked.items():
        for j in js:
            g, i = where[int(experts[j])]
            codes = OT.decode_matrix(g.down[i], g.K, layer.D, layer.F)
            want = exact_down_from_fixed_point(codes, g.s_down[i], fp, j)
            np.testing.assert_array_equal(y[j], want, err_msg="K=%d route %d" % (K, j))
    assert api.device_status() == 0


@pytest.mark.parametrize("T", [5, 300])      # one small route tile per expert / several
def test_moe_gemm_gate_up_decode_one_hot(api, T):
    # With the two-sided transform the GEMM's gate/up epilogue stores the raw projections
    # g = W_g x' and u = W_u x' (the rotations and SwiGLU follow in a separate pass), so
    # one-hot x' rows expose the decoded fp16 operands bit for bit.
    layer = inputs.with_signs(mixed_layer(), 5501)
    dec = decoded(layer)
    dl = api.DeviceLayer.from_synthetic(layer)
    k = 3
    D, F = layer.D, layer.F
    cols = (np.arange(T) * 53 + 11) % D
    x_rot = one_hot(T, D, cols)
    routing = api.route_permute(torch.from_numpy(routes_for(T, k, layer.E)).cuda(), layer.E)
    ws = torch.zeros(api.moe_trellis_workspace_size(dl, T, k), dtype=torch.uint8, device="cuda")
    api.moe_trellis_gemm(dl, x_rot, routing, T, k, ws=ws)
    torch.cuda.synchronize()
    gu = gemm_views(ws, T, k, D, F, two_sided=True)["gu"].cpu().numpy()
    perm = routing.perm.cpu().numpy()
    experts = route_experts(routing.offsets.cpu().numpy())
    for j in range(T * k):
        e, t = int(experts[j]), int(perm[j]) // k
        for p, proj in enumerate(("gate", "up")):
            codes, s = dec[(e, proj)]
            want = weights_f32(codes[:, cols[t]:cols[t] + 1], s)[:, 0]
            np.testing.assert_array_equal(gu[j, p], want, err_msg="route %d expert %d %s" % (j, e, proj))
    assert api.device_status() == 0


@pytest.mark.parametrize("T", [5, 300])
def test_moe_gemm_down_against_exact_sums_of_its_own_h(api, T):
    # The down GEMM accumulates t * 2^-24 * h'_f (exact products) in fp32 tensor memory,
    # so it is compared with the exact sum over the GPU's own fp16 h' rows: the difference
    # is fp32 accumulation only, far below the change of a single wrong code.
    layer = mixed_layer()
    dec = decoded(layer)
    dl = api.DeviceLayer.from_synthetic(layer)
    k = 3
    D, F = layer.D, layer.F
    rng = np.random.default_rng(5600 + T)
    x = inputs.random_activations(rng, (T, D), "bf16")
    x_rot = api.hadamard128(torch.from_numpy(x).to(torch.bfloat16).cuda())
    routing = api.route_permute(torch.from_numpy(routes_for(T, k, layer.E)).cuda(), layer.E)
    ws = torch.zeros(api.moe_trellis_workspace_size(dl, T, k), dtype=torch.uint8, device="cuda")
    y = api.moe_trellis_gemm(dl, x_rot, routing, T, k, ws=ws)
    torch.cuda.synchronize()
    v = gemm_views(ws, T, k, D, F, two_sided=False)
    hr = v["hr"].cpu().numpy().astype(np.float64) * v["hr_scale"].cpu().numpy().astype(np.float64)[:, None]
    y = y.cpu().numpy().astype(np.float64)
    experts = route_experts(routing.offsets.cpu().numpy())
    worst = 0.0
    for j in range(T * k):
        codes, s = dec[(int(experts[j]), "down")]
        W = s.astype(np.float64)[:, None] * KAPPA * codes
        want = W @ hr[j]
        scale = np.abs(W) @ np.abs(hr[j])
        # one wrong code moves y_d by >= s * 2^-12 * |h'_f|, about 1e-3 of this scale for a
        # typical column; fp32 accumulation stays below 1e-5 of it
        err = np.abs(y[j] - want) / scale
        worst = max(worst, err.max())
        assert np.all(err <= 2e-5), "route %d: max err/scale %.3e" % (j, err.max())
    print("GEMM down: max |y - exact| / (|W| . |h'|) = %.3e" % worst)
