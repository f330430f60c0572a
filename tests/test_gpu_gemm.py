"""GPU parity of the prefill path (moe_trellis_gemm: tcgen05 MMAs on decoded fp16
operands, accumulators in tensor memory) against the fp64 oracle, through the C ABI.

Same tolerance as the decode path: the oracle's first-order bound of the composed layer
given |dy| <= 1e-3 * (|W| . |input|) per projection, plus 1e-6 relative.
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


@pytest.mark.parametrize("E,D,F,T,k,split", [
    (4, 256, 128, 3, 2, {2: 2, 3: 1, 4: 1}),       # tiny: 2 K-blocks, N = 16
    (4, 256, 128, 600, 2, {2: 2, 3: 1, 4: 1}),     # ~300 routes per expert: 2 route tiles
    (6, 1024, 512, 200, 3, {3: 6}),                # 16 / 8 K-blocks: stage ring wraps
    (12, 512, 256, 333, 4, {2: 9, 3: 2, 4: 1}),    # mixed widths, ragged tiles
])
def test_gemm_matches_oracle(api, E, D, F, T, k, split):
    layer = inputs.small_layer(700 + T, E=E, D=D, F=F, split=split)
    rng = np.random.default_rng(800 + T)
    x = inputs.random_activations(rng, (T, D), "bf16")
    logits = inputs.normal_logits(rng, T, E)
    got, bufs, dl = run(api, layer, x, logits, k, "gemm")
    assert np.isfinite(got).all()
    assert api.device_status() == 0
    tokens = np.arange(T) if T <= 64 else np.random.default_rng(1).choice(T, 24, replace=False)
    res = OL.moe_tokens(layer, x, logits, k, tokens)
    check(got, res, tokens)
    # the decode path on the same inputs agrees within the same tolerance
    got_v, _, _ = run(api, layer, x, logits, k, "gemv", dl=dl)
    tol = res["bound"] + 1e-6 * np.abs(res["out"]) + 1e-12
    assert np.all(np.abs(got[tokens] - got_v[tokens]) <= 2 * tol)


def test_gemm_full_size_prefill_sampled_tokens(api):
    # The 384-expert all-K=3 layer with 8192 Zipf-routed tokens (the prefill workload);
    # the oracle computes 2 tokens, one of them routed to the hottest expert.
    w = inputs.moe_prefill_t8192()
    got, bufs, _ = run(api, w["layer"], w["x"], w["logits"], 8, "gemm")
    assert np.isfinite(got).all()
    assert api.device_status() == 0
    counts = bufs.routing.counts.cpu().numpy()
    ids = bufs.ids.cpu().numpy()
    hot = int(np.argmax(counts))
    t_hot = int(np.nonzero((ids == hot).any(1))[0][0])
    tokens = [0, t_hot] if t_hot != 0 else [0, 1]
    res = OL.moe_tokens(w["layer"], w["x"], w["logits"], 8, tokens)
    np.testing.assert_array_equal(ids[tokens], res["topk_ids"][tokens])
    check(got, res, tokens)
