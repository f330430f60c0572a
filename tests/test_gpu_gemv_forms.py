"""GPU parity of the routed-expert GEMV over varied shapes, covering both forms of
moe_trellis_gemv: below 32 routes (T*k) the split form (gate/up items, h' quantisation,
down items as three launches), from 32 routes the fused persistent launch with its work
queue, per-expert counters and ready flags.  The cases vary the column splits of the
gate/up items (1 to 8, from the number of active experts), 4- and 8-route passes, ragged
D and F (multiples of 128), experts with no routes and with many (Zipf-skewed logits),
and k from 1 to 8.  Each case checks the routing ids exactly, sampled tokens against the
fp64 oracle within the layer tolerance, and that no device flag was raised."""
import numpy as np
import pytest
import torch

from oracle import layer as OL
from trellis_quantized_moe_gemv_b200 import inputs

pytestmark = pytest.mark.gpu

#        E,    D,   F,  T, k, logits, widths
CASES = [
    (5, 256, 128, 1, 1, "normal", {2: 3, 3: 1, 4: 1}),      # 1 route: split form
    (12, 256, 128, 3, 8, "normal", {2: 9, 3: 2, 4: 1}),     # 24 routes: split form
    (12, 256, 128, 4, 8, "normal", {2: 9, 3: 2, 4: 1}),     # 32 routes: fused, 2 column splits
    (33, 512, 256, 7, 5, "normal", {2: 30, 3: 2, 4: 1}),    # fused, 4 splits
    (33, 1024, 128, 9, 6, "zipf", {2: 20, 3: 10, 4: 3}),    # fused, 7 splits, skewed
    (12, 256, 256, 64, 4, "zipf", {2: 6, 3: 3, 4: 3}),      # fused, 8-route passes
    (7, 384, 128, 50, 2, "normal", {2: 5, 3: 1, 4: 1}),     # D = 3 chunks
    (40, 256, 384, 20, 8, "zipf", {2: 36, 3: 3, 4: 1}),     # F = 384, experts without routes
    (3, 256, 128, 30, 2, "normal", {2: 1, 3: 1, 4: 1}),     # 3 experts, 8-route passes
    (16, 640, 640, 17, 3, "normal", {2: 12, 3: 3, 4: 1}),   # D, F = 5 chunks
    (9, 256, 128, 11, 3, "normal", {2: 7, 3: 1, 4: 1}),     # 33 routes: fused
    (9, 256, 128, 10, 3, "normal", {2: 7, 3: 1, 4: 1}),     # 30 routes: split
]


@pytest.fixture(scope="module")
def api():
    import trellis_quantized_moe_gemv_b200.build as b
    b.build()
    from trellis_quantized_moe_gemv_b200 import api as A
    A.device_status(clear=True)
    return A


@pytest.mark.parametrize("case", range(len(CASES)))
def test_gemv_forms_match_oracle(api, case):
    E, D, F, T, k, kind, widths = CASES[case]
    layer = inputs.small_layer(5100 + case, E=E, D=D, F=F, split=widths)
    rng = np.random.default_rng(5200 + case)
    x = inputs.random_activations(rng, (T, D), "bf16")
    logits = inputs.zipf_gumbel_logits(rng, T, E) if kind == "zipf" else inputs.normal_logits(rng, T, E)
    dl = api.DeviceLayer.from_synthetic(layer)
    bufs = api.MoeBuffers(dl, T, k)
    api.device_status(clear=True)
    out = api.moe_layer(dl, torch.from_numpy(x).to(torch.bfloat16).cuda(), torch.from_numpy(logits).cuda(), k,
                        bufs=bufs, path="gemv")
    torch.cuda.synchronize()
    assert api.device_status() == 0
    got = out.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    tokens = np.arange(T) if T <= 12 else np.sort(np.random.default_rng(5300 + case).choice(T, 12, replace=False))
    res = OL.moe_tokens(layer, x, logits, k, tokens)
    # routing: the same experts per token as the oracle's top-k
    ids = bufs.ids.cpu().numpy().reshape(T, k)
    ref_ids = res["topk_ids"]                      # every token's, [T, k]
    np.testing.assert_array_equal(ids, ref_ids)
    tol = res["bound"] + 1e-6 * np.abs(res["out"]) + 1e-12
    err = np.abs(got[tokens] - res["out"])
    assert np.all(err <= tol), "max err/tol %.3e" % (err / tol).max()
