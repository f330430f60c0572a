"""moe_trellis_gemv_noalloc -- the entry point for callers that cannot allocate device
memory at call time (fixed-pool runtimes, plugin or sandboxed engines, allocation-free
latency paths) -- against moe_trellis_gemv with a caller-provided workspace.

Two calls in a row on different tokens and routes: the second call runs on scratch
still holding the first call's contents.  Both entry points run the same kernels on the
same inputs, so each result must equal the workspace entry point's bit for bit (a stale
scratch read would show up here even when it stays within the error bound); each is also
checked against the oracle within the tolerance the MoE parity tests use (the oracle's
error bound of the composed layer).  The host-side checks must reject calls beyond the
compiled-in scratch, and report bad arguments with the same status as the workspace
entry point.  Collected last so that a stop at the first failure has already
run every other test; self-contained so it also passes alone in a fresh process.
"""
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


def layer_output(api, dl, x, logits, k, use_noalloc):
    """Full layer through the C ABI; the expert stage through either entry point."""
    T = x.shape[0]
    xd = torch.from_numpy(x).to(torch.bfloat16).cuda()
    ld = torch.from_numpy(logits).cuda()
    ids, w = api.route_topk(ld, k)
    routing = api.route_permute(ids, dl.E)
    x_rot = api.hadamard128(xd)
    y_perm = torch.empty((T * k, dl.D), dtype=torch.float32, device="cuda")
    if use_noalloc:
        api.moe_trellis_gemv_noalloc(dl, x_rot, routing, T, k, y_perm)
    else:
        api.moe_trellis_gemv(dl, x_rot, routing, T, k, y_perm)
    out = api.route_unpermute(y_perm, routing.inv, w)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def test_noalloc_matches_workspace_entry_point_twice(api):
    layer = inputs.small_layer(314, E=12, D=512, F=256, split={2: 8, 3: 3, 4: 1})
    dl = api.DeviceLayer.from_synthetic(layer)
    k = 4
    for call, (T, seed) in enumerate([(24, 315), (9, 316)]):
        rng = np.random.default_rng(seed)
        x = inputs.random_activations(rng, (T, 512), "bf16")
        logits = inputs.normal_logits(rng, T, 12)
        got = layer_output(api, dl, x, logits, k, use_noalloc=True)
        ref_gpu = layer_output(api, dl, x, logits, k, use_noalloc=False)
        res = OL.moe_layer(layer, x, logits, k)
        tol = res["bound"] + 1e-6 * np.abs(res["out"]) + 1e-12
        assert np.isfinite(got).all(), "call %d" % call
        np.testing.assert_array_equal(got, ref_gpu, err_msg="call %d" % call)
        # and against the oracle itself
        err = np.abs(got - res["out"])
        assert np.all(err <= tol), "call %d: max err/tol %.3e" % (call, (err / tol).max())
    assert api.device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch(api):
    layer = inputs.small_layer(5, E=12, D=256, F=128)
    dl = api.DeviceLayer.from_synthetic(layer)
    T, k = 6000, 1          # 6000 routes x F = 128 x 12 bytes of workspace > 4 MiB
    x_rot = torch.zeros((T, 256), dtype=torch.float16, device="cuda")
    routing = api.Routing.empty(T, k, 12, "cuda")
    y = torch.empty((T * k, 256), dtype=torch.float32, device="cuda")
    with pytest.raises(api.TQError, match="WORKSPACE"):
        api.moe_trellis_gemv_noalloc(dl, x_rot, routing, T, k, y)


def test_noalloc_reports_bad_arguments_like_the_workspace_entry_point(api):
    # k > E is an invalid argument for both entry points, even when the call would also
    # be too large for the scratch
    layer = inputs.small_layer(5, E=12, D=256, F=128)
    dl = api.DeviceLayer.from_synthetic(layer)
    T, k = 6000, 13
    x_rot = torch.zeros((T, 256), dtype=torch.float16, device="cuda")
    routing = api.Routing.empty(T, k, 12, "cuda")
    y = torch.empty((T * k, 256), dtype=torch.float32, device="cuda")
    with pytest.raises(api.TQError, match="INVALID_ARG"):
        api.moe_trellis_gemv_noalloc(dl, x_rot, routing, T, k, y)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(api.TQError, match="INVALID_ARG"):
        api.moe_trellis_gemv(dl, x_rot, routing, T, k, y, ws)
