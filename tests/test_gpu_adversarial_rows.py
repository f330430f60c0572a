"""Activation rows far from Gaussian, on every path, against the oracle.

The decode GEMV contracts activations as fixed point with power-of-two scales; these rows
are the cases where a single scale per row would round small elements to a step set by
the row's largest one:
  * one 128-chunk of the input 10^3 or 10^4 times larger than the rest of the row;
  * a row that is zero except one chunk;
  * tokens aligned with one expert's gate and up rows, so that a few SwiGLU outputs h_i
    are far larger than the rest (the down projection's input h' then carries one large
    chunk);
  * for the single projection, whose input is already rotated, single elements of x'
    10^3 .. 10^5 times the rest and a row of one nonzero element.
The projection criterion is |y - y_ref| <= 1e-3 * (|W| . |x'|) elementwise (single
projection; "How T16 works", items 1, 2 and 4 of the dsx T16 card); the layer uses the
oracle's propagated bound of that criterion (oracle.layer.e2e_error_bound).
"""
import numpy as np
import pytest
import torch

from oracle import layer as OL
from oracle import t16 as OT
from trellis_quantized_moe_gemv_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    import trellis_quantized_moe_gemv_b200.build as b
    b.build()
    from trellis_quantized_moe_gemv_b200 import api as A
    A.device_status(clear=True)
    return A


def bf16(x):
    return inputs.to_bf16_values(np.asarray(x, dtype=np.float32))


def layer_rows(kind, rng, T, D):
    x = rng.standard_normal((T, D))
    chunks = D // 128
    for t in range(T):
        c = (3 * t + 1) % chunks
        if kind == "spike_chunk_1e3":
            x[t, 128 * c:128 * c + 128] *= 1e3
        elif kind == "spike_chunk_1e4":
            x[t, 128 * c:128 * c + 128] *= 1e4
        elif kind == "one_chunk":
            keep = x[t, 128 * c:128 * c + 128].copy()
            x[t] = 0.0
            x[t, 128 * c:128 * c + 128] = keep
    return bf16(x)


def run_layer(api, layer, x, logits, k, path):
    dl = api.DeviceLayer.from_synthetic(layer)
    bufs = api.MoeBuffers(dl, x.shape[0], k)
    out = api.moe_layer(dl, torch.from_numpy(x).to(torch.bfloat16).cuda(), torch.from_numpy(logits).cuda(), k,
                        bufs=bufs, path=path)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def check(got, res):
    tol = res["bound"] + 1e-6 * np.abs(res["out"]) + 1e-12
    err = np.abs(got - res["out"])
    assert np.all(err <= tol), "max err/tol %.3e" % (err / tol).max()


@pytest.mark.parametrize("kind", ["spike_chunk_1e3", "spike_chunk_1e4", "one_chunk"])
@pytest.mark.parametrize("path", ["gemv", "gemm"])
def test_layer_rows_with_one_dominant_chunk(api, kind, path):
    layer = inputs.small_layer(7001, E=8, D=1024, F=256, split={2: 5, 3: 2, 4: 1})
    rng = np.random.default_rng(7002)
    T, k = 12, 3
    x = layer_rows(kind, rng, T, 1024)
    logits = inputs.normal_logits(rng, T, 8)
    got = run_layer(api, layer, x, logits, k, path)
    assert np.isfinite(got).all()
    check(got, OL.moe_layer(layer, x, logits, k))
    assert api.device_status() == 0


@pytest.mark.parametrize("path", ["gemv", "gemm"])
def test_layer_tokens_with_a_few_huge_swiglu_outputs(api, path):
    # token t is routed to expert e_t (largest logit) and its rotated input is aligned with
    # rows i of that expert's gate and up matrices, so g_i and u_i (and h_i) are far larger
    # than the other channels of h
    layer = inputs.small_layer(7101, E=6, D=512, F=256, split={2: 3, 3: 2, 4: 1})
    weights = OL.ExpertWeights(layer)
    rng = np.random.default_rng(7102)
    T, k = 6, 2
    x = np.zeros((T, 512))
    logits = inputs.normal_logits(rng, T, 6)
    for t in range(T):
        e = t % 6
        logits[t, e] = 10.0
        rows = [(37 * t + 5) % 256, (91 * t + 200) % 256]
        v = rng.standard_normal(512) * 0.05
        for i in rows:
            for proj in ("gate", "up"):
                wr = weights.matrix(e, proj)[i]
                v += 3.0 * wr / np.linalg.norm(wr)
        x[t] = OL.rotate(v[None])[0]          # the rotation is its own inverse
    x = bf16(x)
    res = OL.moe_layer(layer, x, logits, k)
    got = run_layer(api, layer, x, logits, k, path)
    assert np.isfinite(got).all()
    check(got, res)


@pytest.mark.parametrize("case", ["element_1e3", "element_1e5", "single_element", "chunk_1e4"])
@pytest.mark.parametrize("batch", [1, 8])
def test_single_projection_rows_with_spikes(api, case, batch):
    rng = np.random.default_rng(7201)
    rows, cols, K = 512, 1024, 2
    bits = inputs.random_bits(rng, rows, cols, K)[0]
    scales = inputs.random_scales(rng, rows)
    x = rng.standard_normal((batch, cols))
    for b in range(batch):
        j = (211 * b + 17) % cols
        if case == "element_1e3":
            x[b, j] = 1e3 * (1 + b)
        elif case == "element_1e5":
            x[b, j] = 1e4 * (1 + b)
        elif case == "single_element":
            x[b] = 0.0
            x[b, j] = 3.0
        else:
            c = j // 128
            x[b, 128 * c:128 * c + 128] *= 1e4
    x16 = np.clip(x, -65504, 65504).astype(np.float16)
    W = OL.dequantize(OT.decode_matrix(bits, K, rows, cols), scales)
    xr = x16.astype(np.float64)
    ref = OL.project(W, xr)
    tol = 1e-3 * OL.abs_bound(W, xr)
    y = api.trellis_gemv(torch.from_numpy(bits.view(np.int32)).cuda(), torch.from_numpy(scales).cuda(), K, rows, cols,
                         torch.from_numpy(x16).cuda())
    torch.cuda.synchronize()
    err = np.abs(y.cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= tol), "max err/tol %.3e" % (err / tol).max()
