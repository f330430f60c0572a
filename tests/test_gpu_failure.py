"""Failure detection without a GPU fault: the library's bounded device wait, run on an
mbarrier that nothing arrives on, gives up after its limit, raises device flag bit 1 and
returns; the context stays usable (a layer computed right after matches the oracle)."""
import time

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


def test_bounded_wait_gives_up_and_flags(api):
    api.device_status(clear=True)
    torch.cuda.synchronize()
    t0 = time.time()
    api.selftest_bounded_wait(20000)          # 20 ms
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert api.device_status(clear=True) == 2
    assert 0.015 <= elapsed < 5.0


def test_context_usable_after_a_wait_gave_up(api):
    api.selftest_bounded_wait(5000)
    torch.cuda.synchronize()
    assert api.device_status(clear=True) == 2
    layer = inputs.small_layer(808, E=12, D=256, F=128)
    rng = np.random.default_rng(809)
    x = inputs.random_activations(rng, (6, 256), "bf16")
    logits = inputs.normal_logits(rng, 6, 12)
    dl = api.DeviceLayer.from_synthetic(layer)
    out = api.moe_layer(dl, torch.from_numpy(x).to(torch.bfloat16).cuda(), torch.from_numpy(logits).cuda(), 4,
                        path="gemv")
    torch.cuda.synchronize()
    res = OL.moe_layer(layer, x, logits, 4)
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - res["out"]) <= res["bound"] + 1e-6 * np.abs(res["out"]) + 1e-12)
    assert api.device_status() == 0


def test_selftest_rejects_bad_limits(api):
    with pytest.raises(api.TQError, match="INVALID"):
        api.selftest_bounded_wait(0)


@pytest.mark.parametrize("path,T", [("gemv", 4), ("gemv", 16), ("gemm", 16)])   # split GEMV, fused GEMV, GEMM
def test_route_to_an_expert_the_layer_does_not_hold(api, path, T):
    """Routes to an expert missing from the layer's width groups: the expert path flags
    device bit 0, skips that expert's work and still completes (the fused GEMV's counters
    and flags of that expert advance as for any other); every token with no route to it
    matches the oracle."""
    layer = inputs.small_layer(4242, E=12, D=256, F=128)
    rng = np.random.default_rng(4243)
    x = inputs.random_activations(rng, (T, 256), "bf16")
    logits = inputs.normal_logits(rng, T, 12)
    missing = 5
    logits[::3, missing] += 10.0          # every third token routes to the missing expert
    groups = []
    for g in layer.groups:
        keep = g.ids != missing
        groups.append(dict(K=g.K, ids=g.ids[keep], gate=g.gate[keep], up=g.up[keep], down=g.down[keep],
                           s_gate=g.s_gate[keep], s_up=g.s_up[keep], s_down=g.s_down[keep]))
    dl = api.DeviceLayer(layer.E, layer.D, layer.F, groups)
    api.device_status(clear=True)
    out = api.moe_layer(dl, torch.from_numpy(x).to(torch.bfloat16).cuda(), torch.from_numpy(logits).cuda(), 4,
                        path=path)
    torch.cuda.synchronize()
    assert api.device_status(clear=True) & 1
    res = OL.moe_layer(layer, x, logits, 4)
    top = np.argsort(-logits, axis=1, kind="stable")[:, :4]
    clean = ~(top == missing).any(axis=1)
    assert clean.any() and (~clean).any()
    got = out.cpu().numpy().astype(np.float64)
    err = np.abs(got[clean] - res["out"][clean])
    assert np.all(err <= res["bound"][clean] + 1e-6 * np.abs(res["out"][clean]) + 1e-12)
    # the context stays usable: the full layer right after matches the oracle
    dl_full = api.DeviceLayer.from_synthetic(layer)
    logits2 = inputs.normal_logits(rng, T, 12)
    out2 = api.moe_layer(dl_full, torch.from_numpy(x).to(torch.bfloat16).cuda(), torch.from_numpy(logits2).cuda(),
                         4, path=path)
    torch.cuda.synchronize()
    res2 = OL.moe_layer(layer, x, logits2, 4)
    got2 = out2.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got2 - res2["out"]) <= res2["bound"] + 1e-6 * np.abs(res2["out"]) + 1e-12)
    assert api.device_status() == 0
