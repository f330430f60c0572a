"""GPU parity of the MoE layer path (route_topk -> route_permute -> hadamard128 ->
moe_trellis_gemv -> route_unpermute) against the fp64 oracle, through the C ABI.

Tolerance: the oracle's first-order error bound of the composed layer given that every
projection meets |dy| <= 1e-3 * (|W| . |input|) (see oracle.layer.e2e_error_bound),
plus 1e-6 relative for the fp32 combine.  Routing ids are compared exactly.
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


def run_layer(api, layer, x, logits, k, path="gemv", dl=None):
    dl = dl or api.DeviceLayer.from_synthetic(layer)
    xd = torch.from_numpy(x).to(torch.bfloat16).cuda()
    ld = torch.from_numpy(logits).cuda()
    bufs = api.MoeBuffers(dl, x.shape[0], k)
    out = api.moe_layer(dl, xd, ld, k, bufs=bufs, path=path)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), bufs, dl


def check_against_oracle(got, res, tokens=None):
    ref, bound = res["out"], res["bound"]
    if tokens is not None:
        got = got[tokens]
    tol = bound + 1e-6 * np.abs(ref) + 1e-12
    err = np.abs(got - ref)
    assert np.all(err <= tol), "max err/tol %.3e" % (err / tol).max()


@pytest.mark.parametrize("T", [1, 5, 16, 40])
@pytest.mark.parametrize("split", [{2: 9, 3: 2, 4: 1}, {3: 12}])
def test_small_layer_matches_oracle(api, T, split):
    layer = inputs.small_layer(500 + T, E=12, D=256, F=128, split=split)
    rng = np.random.default_rng(600 + T)
    x = inputs.random_activations(rng, (T, 256), "bf16")
    logits = inputs.normal_logits(rng, T, 12)
    got, bufs, _ = run_layer(api, layer, x, logits, 4)
    res = OL.moe_layer(layer, x, logits, 4)
    np.testing.assert_array_equal(bufs.ids.cpu().numpy(), res["topk_ids"])
    check_against_oracle(got, res)
    assert api.device_status() == 0


def test_wider_layer_more_tokens_per_expert(api):
    # D = 512, F = 256: several Hadamard chunks per projection; 4 experts and 40 tokens
    # with k = 2 give ~20 routes per expert (several token passes).
    layer = inputs.small_layer(42, E=4, D=512, F=256, split={2: 2, 3: 1, 4: 1})
    rng = np.random.default_rng(43)
    x = inputs.random_activations(rng, (40, 512), "bf16")
    logits = inputs.normal_logits(rng, 40, 4)
    got, _, _ = run_layer(api, layer, x, logits, 2)
    check_against_oracle(got, OL.moe_layer(layer, x, logits, 2))


def test_multi_pass_experts_with_stage_reuse(api):
    # D = 1024, F = 512: every warp streams several shared-memory stages per pass (stage
    # buffers and their barriers are reused), and with 64 tokens, top-2 of 4 experts
    # each expert has ~32 routes, i.e. several 8-route passes per work item.
    layer = inputs.small_layer(61, E=4, D=1024, F=512, split={2: 2, 3: 1, 4: 1})
    rng = np.random.default_rng(62)
    x = inputs.random_activations(rng, (64, 1024), "bf16")
    logits = inputs.normal_logits(rng, 64, 4)
    got, _, _ = run_layer(api, layer, x, logits, 2)
    check_against_oracle(got, OL.moe_layer(layer, x, logits, 2))
    assert api.device_status() == 0


def test_mixed_width_routes_bit_identical_to_single_width(api):
    # After the TrellisMX K2 Mix card's layer test: every width's routes computed in the
    # mixed-width launch equal, bit for bit, the same routes in a launch whose layer holds
    # only that width's experts.
    layer = inputs.small_layer(77, E=12, D=256, F=128, split={2: 6, 3: 4, 4: 2})
    rng = np.random.default_rng(78)
    T, k = 24, 4
    x = inputs.random_activations(rng, (T, 256), "bf16")
    logits = inputs.normal_logits(rng, T, 12)
    dl = api.DeviceLayer.from_synthetic(layer)
    _, bufs, _ = run_layer(api, layer, x, logits, k, dl=dl)
    ids = bufs.ids.cpu().numpy()
    inv = bufs.routing.inv.cpu().numpy()
    y_mixed = bufs.y_perm.cpu().numpy()
    xd = torch.from_numpy(x).to(torch.bfloat16).cuda()
    x_rot = api.hadamard128(xd)
    for g in layer.groups:
        single = api.DeviceLayer(layer.E, layer.D, layer.F,
                                 [dict(K=g.K, ids=g.ids, gate=g.gate, up=g.up, down=g.down,
                                       s_gate=g.s_gate, s_up=g.s_up, s_down=g.s_down)])
        mine = np.isin(ids, g.ids)
        # routing restricted to this width: each token keeps its own routes of width K,
        # the rest are sent to a placeholder expert of this width and ignored below.
        sub = np.where(mine, ids, g.ids[0]).astype(np.int32)
        r = api.route_permute(torch.from_numpy(sub).cuda(), layer.E)
        y = api.moe_trellis_gemv(single, x_rot, r, T, k)
        torch.cuda.synchronize()
        inv_s = r.inv.cpu().numpy()
        y_s = y.cpu().numpy()
        for t in range(T):
            for s in range(k):
                if mine[t, s]:
                    np.testing.assert_array_equal(y_s[inv_s[t * k + s]], y_mixed[inv[t * k + s]])


def test_graph_replay_with_changing_routes(api):
    # After the TrellisMX K2 Mix card's "FULL CUDA graph replay with changing routes":
    # one captured layer call replayed on new inputs equals eager calls bit for bit.
    layer = inputs.small_layer(90, E=12, D=256, F=128)
    T, k = 8, 4
    dl = api.DeviceLayer.from_synthetic(layer)
    bufs = api.MoeBuffers(dl, T, k)
    x_in = torch.empty((T, 256), dtype=torch.bfloat16, device="cuda")
    l_in = torch.empty((T, 12), dtype=torch.float32, device="cuda")
    rng = np.random.default_rng(91)
    first = [inputs.random_activations(rng, (T, 256), "bf16"), inputs.normal_logits(rng, T, 12)]
    x_in.copy_(torch.from_numpy(first[0]).to(torch.bfloat16))
    l_in.copy_(torch.from_numpy(first[1]))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        api.moe_layer(dl, x_in, l_in, k, bufs=bufs, path="gemv")   # warm-up (kernel attributes)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        api.moe_layer(dl, x_in, l_in, k, bufs=bufs, path="gemv")
    for trial in range(3):
        xv = inputs.random_activations(rng, (T, 256), "bf16")
        lv = inputs.normal_logits(rng, T, 12)
        x_in.copy_(torch.from_numpy(xv).to(torch.bfloat16))
        l_in.copy_(torch.from_numpy(lv))
        g.replay()
        torch.cuda.synchronize()
        replayed = bufs.out.clone()
        eager, _, _ = run_layer(api, layer, xv, lv, k, dl=dl)
        np.testing.assert_array_equal(replayed.cpu().numpy().astype(np.float64), eager)
        check_against_oracle(eager, OL.moe_layer(layer, xv, lv, k))


@pytest.mark.parametrize("path,T", [("gemv", 8), ("gemm", 40)])
def test_moe_graph_with_host_buffers(api, path, T):
    # api.MoeGraph: pinned host inputs -> device, the layer, device -> pinned host output,
    # replayed as one graph; new inputs written into the same host buffers each step
    layer = inputs.small_layer(92, E=12, D=256, F=128)
    k = 4
    dl = api.DeviceLayer.from_synthetic(layer)
    x_host = torch.empty((T, 256), dtype=torch.bfloat16).pin_memory()
    l_host = torch.empty((T, 12), dtype=torch.float32).pin_memory()
    rng = np.random.default_rng(93)
    x_host.copy_(torch.from_numpy(inputs.random_activations(rng, (T, 256), "bf16")).to(torch.bfloat16))
    l_host.copy_(torch.from_numpy(inputs.normal_logits(rng, T, 12)))
    mg = api.MoeGraph(dl, x_host, l_host, k, path=path)
    for trial in range(3):
        xv = inputs.random_activations(rng, (T, 256), "bf16")
        lv = inputs.normal_logits(rng, T, 12)
        x_host.copy_(torch.from_numpy(xv).to(torch.bfloat16))
        l_host.copy_(torch.from_numpy(lv))
        out = mg.replay()
        mg.stream.synchronize()
        eager, _, _ = run_layer(api, layer, xv, lv, k, path=path, dl=dl)
        np.testing.assert_array_equal(out.numpy().astype(np.float64), eager)
        check_against_oracle(eager, OL.moe_layer(layer, xv, lv, k))
    with pytest.raises(ValueError):
        api.MoeGraph(dl, x_host.cuda(), l_host, k)


def test_full_size_decode_layer_sampled_tokens(api):
    # The 384-expert mixed-width decode layer (D = 4096, F = 1024, 16 tokens, top-8) in
    # the launch configuration the benchmark times; the oracle computes 2 tokens.
    w = inputs.moe_decode_t16()
    got, bufs, _ = run_layer(api, w["layer"], w["x"], w["logits"], 8)
    assert np.isfinite(got).all()
    res = OL.moe_tokens(w["layer"], w["x"], w["logits"], 8, token_ids=[0, 11])
    np.testing.assert_array_equal(bufs.ids.cpu().numpy(), res["topk_ids"])
    check_against_oracle(got, res, tokens=[0, 11])
    assert api.device_status() == 0


def test_full_size_decode_layer_eight_routes_per_pass(api):
    # The same layer at 320 tokens (6.7 routes per active expert): the GEMV runs 8 routes
    # per pass; sampled tokens against the oracle
    w = inputs.moe_sweep_tokens(320, layer=inputs.moe_decode_t16()["layer"])
    got, bufs, _ = run_layer(api, w["layer"], w["x"], w["logits"], 8, path="gemv")
    assert np.isfinite(got).all()
    res = OL.moe_tokens(w["layer"], w["x"], w["logits"], 8, token_ids=[3, 319])
    check_against_oracle(got, res, tokens=[3, 319])
    assert api.device_status() == 0


def test_workspace_too_small_is_an_error(api):
    layer = inputs.small_layer(5, E=12, D=256, F=128)
    dl = api.DeviceLayer.from_synthetic(layer)
    T, k = 4, 4
    bufs = api.MoeBuffers(dl, T, k)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(api.TQError, match="WORKSPACE"):
        api.moe_trellis_gemv(dl, bufs.x_rot, bufs.routing, T, k, bufs.y_perm, small)
