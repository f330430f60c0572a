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


def test_gemm_mixed_width_routes_bit_identical_to_single_width(api):
    # The TrellisMX K2 Mix card's layer test for the GEMM path: every width's routes in the
    # mixed-width launch equal, bit for bit, the same routes in a launch whose layer holds
    # only that width's experts.
    layer = inputs.small_layer(1077, E=12, D=512, F=256, split={2: 6, 3: 4, 4: 2})
    rng = np.random.default_rng(1078)
    T, k = 200, 4
    x = inputs.random_activations(rng, (T, 512), "bf16")
    logits = inputs.normal_logits(rng, T, 12)
    dl = api.DeviceLayer.from_synthetic(layer)
    _, bufs, _ = run(api, layer, x, logits, k, "gemm", dl=dl)
    ids = bufs.ids.cpu().numpy()
    inv = bufs.routing.inv.cpu().numpy()
    y_mixed = bufs.y_perm.cpu().numpy()
    x_rot = api.hadamard128(torch.from_numpy(x).to(torch.bfloat16).cuda())
    for g in layer.groups:
        single = api.DeviceLayer(layer.E, layer.D, layer.F,
                                 [dict(K=g.K, ids=g.ids, gate=g.gate, up=g.up, down=g.down,
                                       s_gate=g.s_gate, s_up=g.s_up, s_down=g.s_down)])
        mine = np.isin(ids, g.ids)
        # routes of other widths go to experts absent from this layer (slot -1): the
        # expert-grouped order of this width's routes, and so their route tiles, are the
        # same as in the mixed launch
        r = api.route_permute(torch.from_numpy(ids.astype(np.int32)).cuda(), layer.E)
        y = api.moe_trellis_gemm(single, x_rot, r, T, k)
        torch.cuda.synchronize()
        inv_s = r.inv.cpu().numpy()
        y_s = y.cpu().numpy()
        for t in range(T):
            for s in range(k):
                if mine[t, s]:
                    np.testing.assert_array_equal(y_s[inv_s[t * k + s]], y_mixed[inv[t * k + s]])
    assert api.device_status() & 1    # routes of absent experts were skipped and flagged
    api.device_status(clear=True)


@pytest.mark.parametrize("T", [2048, 16384])
@pytest.mark.parametrize("path", ["gemm", "auto"])
def test_sweep_sizes_mixed_width_layer_through_the_gemm(api, T, path):
    # The batch sweep's GEMM sizes on the mixed-width 384-expert layer (368/15/1 experts at
    # K = 2/3/4, uniform top-8): sampled tokens against the oracle, including a token routed
    # to the coldest expert with routes and one routed to the hottest.
    w = inputs.moe_sweep_tokens(T, layer=inputs.moe_decode_t16()["layer"])
    got, bufs, dl = run(api, w["layer"], w["x"], w["logits"], 8, path)
    assert np.isfinite(got).all()
    assert api.device_status() == 0
    ids = bufs.ids.cpu().numpy()
    counts = bufs.routing.counts.cpu().numpy()
    hot = int(np.argmax(counts))
    cold = int(np.argmin(np.where(counts > 0, counts, np.iinfo(np.int32).max)))
    t_hot = int(np.nonzero((ids == hot).any(1))[0][0])
    t_cold = int(np.nonzero((ids == cold).any(1))[0][0])
    tokens = sorted({t_hot, t_cold, T // 2})
    sub = dict(x=w["x"][tokens], logits=w["logits"][tokens])
    res = OL.moe_tokens(w["layer"], sub["x"], sub["logits"], 8, np.arange(len(tokens)))
    np.testing.assert_array_equal(ids[tokens], res["topk_ids"])
    check(got[tokens], res)
