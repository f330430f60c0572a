"""GPU parity of the two-sided transform (128-wide Hadamard rotation on both sides of
every projection, layer sign vectors shared by the experts) against the fp64 oracle,
through the C ABI, for the GEMV and the GEMM paths; same tolerance as the one-sided
layer (the oracle's propagated bound, whose output rotations spread each projection's
error over its 128-chunk)."""
import numpy as np
import pytest
import torch

from oracle import layer as OL
from trellis_quantized_moe_gemv_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    import trellis_quantized_moe_gemv_b200.build as b
    b.build()
    from trellis_quantized_moe_gemv_b200 import api as A
    A.device_status(clear=True)
    return A


def run(api, layer, x, logits, k, path, dl=None):
    dl = dl or api.DeviceLayer.from_synthetic(layer)
    xd = torch.from_numpy(x).to(torch.bfloat16).cuda()
    ld = torch.from_numpy(logits).cuda()
    bufs = api.MoeBuffers(dl, x.shape[0], k)
    out = api.moe_layer(dl, xd, ld, k, bufs=bufs, path=path)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), bufs, dl


def check(got, res, tokens=None):
    ref, bound = res["out"], res["bound"]
    if tokens is not None:
        got = got[tokens]
    tol = bound + 1e-6 * np.abs(ref) + 1e-12
    err = np.abs(got - ref)
    assert np.all(err <= tol), "max err/tol %.3e" % (err / tol).max()


def test_signed_rotation_and_combine_match_oracle(api):
    rng = np.random.default_rng(31)
    x = inputs.random_activations(rng, (5, 512), "bf16")
    signs = inputs.random_signs(rng, 512)
    got = api.hadamard128_signed(torch.from_numpy(x).to(torch.bfloat16).cuda(), torch.from_numpy(signs).cuda())
    ref = OL.rotate_in(x.astype(np.float64), signs)
    np.testing.assert_allclose(got.float().cpu().numpy(), ref, rtol=2.0 ** -10, atol=1e-6)
    # combine then output rotation: signs * rotate(sum_s w y)
    T, k, D = 6, 3, 256
    y = rng.standard_normal((T * k, D)).astype(np.float32)
    w = rng.random((T, k)).astype(np.float32)
    inv = rng.permutation(T * k).astype(np.int32)
    sy = inputs.random_signs(rng, D)
    out = api.route_unpermute_signed(torch.from_numpy(y).cuda(), torch.from_numpy(inv).cuda(),
                                     torch.from_numpy(w).cuda(), torch.from_numpy(sy).cuda())
    ref = OL.rotate_out(OL.combine(y, inv, w), sy)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("T", [1, 7, 40])
@pytest.mark.parametrize("split", [{2: 9, 3: 2, 4: 1}, {3: 12}])
def test_two_sided_gemv_layer(api, T, split):
    layer = inputs.with_signs(inputs.small_layer(900 + T, E=12, D=256, F=256, split=split), 950 + T)
    rng = np.random.default_rng(960 + T)
    x = inputs.random_activations(rng, (T, 256), "bf16")
    logits = inputs.normal_logits(rng, T, 12)
    got, bufs, _ = run(api, layer, x, logits, 4, "gemv")
    res = OL.moe_layer(layer, x, logits, 4)
    np.testing.assert_array_equal(bufs.ids.cpu().numpy(), res["topk_ids"])
    check(got, res)
    assert api.device_status() == 0


@pytest.mark.parametrize("T,k", [(3, 2), (300, 3)])
def test_two_sided_gemm_layer_and_gemv_agree(api, T, k):
    layer = inputs.with_signs(inputs.small_layer(1100 + T, E=6, D=512, F=256, split={2: 3, 3: 2, 4: 1}), 1150)
    rng = np.random.default_rng(1160 + T)
    x = inputs.random_activations(rng, (T, 512), "bf16")
    logits = inputs.normal_logits(rng, T, 6)
    got, _, dl = run(api, layer, x, logits, k, "gemm")
    assert np.isfinite(got).all()
    tokens = np.arange(T) if T <= 64 else np.random.default_rng(2).choice(T, 16, replace=False)
    res = OL.moe_tokens(layer, x, logits, k, tokens)
    check(got, res, tokens)
    got_v, _, _ = run(api, layer, x, logits, k, "gemv", dl=dl)
    check(got_v, res, tokens)
    assert api.device_status() == 0


def test_two_sided_full_size_decode_layer(api):
    # the 384-expert mixed-width decode layer with layer signs; the oracle computes 2
    # tokens over a subset of the output rows (whole 128-row chunks are decoded).
    w = inputs.moe_decode_t16()
    layer = inputs.with_signs(w["layer"], 1203)
    got, bufs, _ = run(api, layer, w["x"], w["logits"], 8, "gemv")
    assert np.isfinite(got).all()
    rows = np.array([0, 1, 127, 128, 2049, 4095])
    res = OL.moe_tokens(layer, w["x"], w["logits"], 8, [0, 11], down_rows=rows)
    ref, bound = res["out"], res["bound"]
    sel = got[[0, 11]][:, rows]
    assert np.all(np.abs(sel - ref) <= bound + 1e-6 * np.abs(ref) + 1e-12)
    layer.signs = None
