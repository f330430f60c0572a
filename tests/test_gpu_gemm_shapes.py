"""GPU parity of the tcgen05 expert GEMM (moe_trellis_gemm) over varied shapes: route
tiles on both sides of the 256-route block (ragged last blocks, experts with a single
route and with thousands), Zipf-skewed and uniform routing, 2 to 64 K-blocks (D, F from
256 to 4096), mixed widths and both codebooks (T16 fp16 operands; the pair-trellis E4M3
codebook, kind::f8f6f4).  Each case checks every token's routing ids exactly, sampled
tokens against the fp64 oracle within the layer tolerance (the E4M3 activation rounding
for the FP8 codebook), and that no device flag was raised."""
import numpy as np
import pytest
import torch

from oracle import layer as OL
from trellis_quantized_moe_gemv_b200 import inputs

pytestmark = pytest.mark.gpu

EPS_E4M3 = 2.0 ** -4 + 2.0 ** -10     # E4M3 activation rounding per projection (R26)

#        E,    D,    F,    T, k, logits, widths, codebook
CASES = [
    (4, 256, 128, 1, 1, "normal", {2: 2, 3: 1, 4: 1}, "t16"),        # one route, 4 / 2 K-blocks
    (3, 512, 256, 600, 1, "zipf", {2: 1, 3: 1, 4: 1}, "t16"),         # 325 routes: blocks of 256 + 69
    (5, 256, 384, 700, 2, "zipf", {2: 2, 3: 2, 4: 1}, "t16"),         # hottest expert: several blocks
    (20, 1024, 512, 333, 8, "normal", {2: 15, 3: 4, 4: 1}, "t16"),    # 16 / 8 K-blocks, uniform
    (3, 4096, 256, 96, 2, "normal", {2: 1, 3: 1, 4: 1}, "t16"),       # 64 K-blocks (gate/up)
    (12, 768, 1024, 150, 4, "zipf", {2: 9, 3: 2, 4: 1}, "t16"),       # D = 3 x 256
    (3, 512, 256, 600, 1, "zipf", {2: 1, 3: 1, 4: 1}, "pair_e4m3"),   # FP8: 343 routes, 256 + 87
    (10, 1024, 384, 200, 3, "zipf", {2: 5, 3: 4, 4: 1}, "pair_e4m3"),  # FP8: 8 / 3 K-blocks
]


@pytest.fixture(scope="module")
def api():
    import trellis_quantized_moe_gemv_b200.build as b
    b.build()
    from trellis_quantized_moe_gemv_b200 import api as A
    A.device_status(clear=True)
    return A


@pytest.mark.parametrize("case", range(len(CASES)))
def test_gemm_shapes_match_oracle(api, case):
    E, D, F, T, k, kind, widths, codebook = CASES[case]
    layer = inputs.small_layer(6100 + case, E=E, D=D, F=F, split=widths, codebook=codebook)
    rng = np.random.default_rng(6200 + case)
    x = inputs.random_activations(rng, (T, D), "bf16")
    logits = inputs.zipf_gumbel_logits(rng, T, E) if kind == "zipf" else inputs.normal_logits(rng, T, E)
    dl = api.DeviceLayer.from_synthetic(layer)
    bufs = api.MoeBuffers(dl, T, k)
    api.device_status(clear=True)
    out = api.moe_layer(dl, torch.from_numpy(x).to(torch.bfloat16).cuda(), torch.from_numpy(logits).cuda(), k,
                        bufs=bufs, path="gemm")
    torch.cuda.synchronize()
    assert api.device_status() == 0
    got = out.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    tokens = np.arange(T) if T <= 10 else np.sort(np.random.default_rng(6300 + case).choice(T, 10, replace=False))
    eps = EPS_E4M3 if codebook == "pair_e4m3" else 1e-3
    res = OL.moe_tokens(layer, x, logits, k, tokens, eps_proj=eps)
    np.testing.assert_array_equal(bufs.ids.cpu().numpy(), res["topk_ids"])
    tol = res["bound"] + 1e-6 * np.abs(res["out"]) + 1e-12
    err = np.abs(got[tokens] - res["out"])
    assert np.all(err <= tol), "max err/tol %.3e" % (err / tol).max()
