"""GPU parity of the single kernels against the CPU oracle, through the C ABI.

Bar: bit-exact for decoded codes, routing ids and permutations; projections within
|y - y_ref| <= 1e-3 * (|W| . |x'|) elementwise; the rotation within the fp16 rounding of
its output plus fp32 butterfly error; route weights and the combine to fp32 precision.
"""
import math

import numpy as np
import pytest
import torch

from oracle import layer as OL
from oracle import t16 as OT
from trellis_quantized_moe_gemv_b200 import inputs

pytestmark = pytest.mark.gpu

PROJ_TOL = 1e-3


@pytest.fixture(scope="module")
def api():
    import trellis_quantized_moe_gemv_b200.build as b
    b.build()
    from trellis_quantized_moe_gemv_b200 import api as A
    assert A.device_status(clear=True) == 0 or True
    return A


def dev_bits(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).cuda()


def dev_f16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float16)).cuda()


def dev_bf16(a_f32):
    return torch.from_numpy(np.ascontiguousarray(a_f32, dtype=np.float32)).to(torch.bfloat16).cuda()


# ----------------------------------------------------------------------------- decode

@pytest.mark.parametrize("K,rows,cols", [(2, 16, 16), (2, 256, 256), (3, 48, 80), (4, 32, 272),
                                         (2, 1024, 4096), (3, 1024, 4096), (4, 1024, 4096)])
def test_decode_bit_exact(api, K, rows, cols):
    rng = np.random.default_rng(100 + K + rows)
    bits = inputs.random_bits(rng, rows, cols, K)[0]
    got = api.trellis_decode(dev_bits(bits), K, rows, cols)
    torch.cuda.synchronize()
    ref = OT.decode_matrix(bits, K, rows, cols)
    np.testing.assert_array_equal(got.float().cpu().numpy().astype(np.int64), ref)


@pytest.mark.parametrize("fill,code", [(0, -255), (0xFFFFFFFF, 151)])
def test_decode_constant_streams(api, fill, code):
    bits = np.full(inputs.words_per_matrix(64, 128, 3), fill, dtype=np.uint32)
    got = api.trellis_decode(dev_bits(bits), 3, 64, 128).float().cpu().numpy()
    assert np.all(got == code)


# ----------------------------------------------------------------------------- hadamard

@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("rows,cols", [(1, 128), (5, 256), (16, 4096), (300, 1024)])
def test_hadamard_vs_explicit_matrix(api, dtype, rows, cols):
    rng = np.random.default_rng(rows * 7 + cols)
    x32 = rng.standard_normal((rows, cols)).astype(np.float32) * 3
    if dtype == "f16":
        xv = x32.astype(np.float16).astype(np.float64)
        xd = dev_f16(x32.astype(np.float16))
    elif dtype == "bf16":
        xb = inputs.to_bf16_values(x32)
        xv = xb.astype(np.float64)
        xd = dev_bf16(xb)
    else:
        xv = x32.astype(np.float64)
        xd = torch.from_numpy(x32).cuda()
    got = api.hadamard128(xd).float().cpu().numpy().astype(np.float64)
    ref = OL.rotate(xv)
    chunk_abs = np.repeat(np.abs(xv).reshape(rows, cols // 128, 128).sum(-1), 128, axis=1)
    tol = 2.0 ** -11 * np.abs(ref) + 8 * 2.0 ** -24 * chunk_abs / math.sqrt(128) + 1e-30
    assert np.all(np.abs(got - ref) <= tol)


# ----------------------------------------------------------------------------- GEMV

def _check_projection(y, ref, bound):
    err = np.abs(y - ref)
    ok = err <= PROJ_TOL * bound
    assert ok.all(), "max err/bound %.3e" % (err / np.maximum(bound, 1e-300)).max()


def test_gemv_single_256(api):
    w = inputs.single_256()
    x_rot = api.hadamard128(dev_f16(w["x"]))
    y = api.trellis_gemv(dev_bits(w["bits"]), dev_f16(w["scales"]), 2, 256, 256, x_rot)
    ref, bound = OL.single_projection(w["bits"], 2, 256, 256, w["scales"], w["x"].astype(np.float64))
    _check_projection(y.cpu().numpy().astype(np.float64), ref, bound)


@pytest.mark.parametrize("K", [2, 3, 4])
@pytest.mark.parametrize("batch", [1, 4, 16])
def test_gemv_proj_1024x4096(api, K, batch):
    w = inputs.proj_1024x4096(K, batch)
    x_rot = api.hadamard128(dev_bf16(w["x"]))
    y = api.trellis_gemv(dev_bits(w["bits"]), dev_f16(w["scales"]), K, 1024, 4096, x_rot)
    ref, bound = OL.single_projection(w["bits"], K, 1024, 4096, w["scales"], w["x"].astype(np.float64))
    _check_projection(y.cpu().numpy().astype(np.float64), ref, bound)


@pytest.mark.parametrize("K,rows,cols,batch", [(2, 16, 128, 1), (3, 48, 384, 9), (4, 272, 640, 23),
                                               (2, 2000, 128, 3), (3, 64, 4096, 256)])
def test_gemv_ragged_shapes(api, K, rows, cols, batch):
    rng = np.random.default_rng(K * 1000 + rows + batch)
    bits = inputs.random_bits(rng, rows, cols, K)[0]
    s = inputs.random_scales(rng, rows)
    x = inputs.random_activations(rng, (batch, cols), "bf16")
    x_rot = api.hadamard128(dev_bf16(x))
    y = api.trellis_gemv(dev_bits(bits), dev_f16(s), K, rows, cols, x_rot)
    ref, bound = OL.single_projection(bits, K, rows, cols, s, x.astype(np.float64))
    _check_projection(y.cpu().numpy().astype(np.float64), ref, bound)


def test_gemv_constant_stream_closed_form(api):
    # All-zero streams: every code is T16(0) - 255 = -255, so y = s * 2^-12 * (-255) * sum x'.
    rows, cols = 64, 512
    bits = np.zeros(inputs.words_per_matrix(rows, cols, 2), dtype=np.uint32)
    rng = np.random.default_rng(77)
    s = inputs.random_scales(rng, rows)
    x = inputs.random_activations(rng, (3, cols), "bf16")
    x_rot = api.hadamard128(dev_bf16(x))
    y = api.trellis_gemv(dev_bits(bits), dev_f16(s), 2, rows, cols, x_rot).cpu().numpy().astype(np.float64)
    xr = OL.rotate(x.astype(np.float64))
    s64 = s.astype(np.float64)[None, :]
    expect = s64 * 2.0 ** -12 * (-255) * xr.sum(1)[:, None]
    bound = s64 * 2.0 ** -12 * 255 * np.abs(xr).sum(1)[:, None]
    _check_projection(y, expect, bound)


# ----------------------------------------------------------------------------- routing

@pytest.mark.parametrize("T,E,k", [(1, 384, 8), (16, 384, 8), (333, 384, 8), (64, 40, 8), (7, 1024, 32),
                                   (5, 8, 8)])
def test_route_topk(api, T, E, k):
    rng = np.random.default_rng(T + E + k)
    logits = inputs.normal_logits(rng, T, E)
    ids, w = api.route_topk(torch.from_numpy(logits).cuda(), k)
    rid, rw = OL.route_topk(logits, k)
    np.testing.assert_array_equal(ids.cpu().numpy(), rid)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=2e-6, atol=1e-7)


def test_route_topk_ties_to_lower_id(api):
    logits = np.zeros((3, 384), dtype=np.float32)
    logits[1, [5, 9, 300]] = 1.0
    logits[2] = np.repeat(np.arange(48, dtype=np.float32), 8)  # groups of 8 equal values
    ids, w = api.route_topk(torch.from_numpy(logits).cuda(), 8)
    rid, rw = OL.route_topk(logits, 8)
    np.testing.assert_array_equal(ids.cpu().numpy(), rid)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=2e-6)


@pytest.mark.parametrize("T,E,k", [(1, 384, 8), (16, 384, 8), (300, 384, 8), (8192, 384, 8),
                                   (3, 5, 2), (2048, 1024, 4)])
def test_route_permute_exact(api, T, E, k):
    rng = np.random.default_rng(T * 3 + E)
    if T == 8192:
        logits = inputs.zipf_gumbel_logits(rng, T, E)
    else:
        logits = inputs.normal_logits(rng, T, E)
    rid, _ = OL.route_topk(logits, k)
    r = api.route_permute(torch.from_numpy(rid).cuda(), E)
    counts, offsets, perm, inv = OL.route_permute(rid, E)
    np.testing.assert_array_equal(r.counts.cpu().numpy(), counts)
    np.testing.assert_array_equal(r.offsets.cpu().numpy(), offsets)
    np.testing.assert_array_equal(r.perm.cpu().numpy(), perm)
    np.testing.assert_array_equal(r.inv.cpu().numpy(), inv)
    active = np.nonzero(counts)[0]
    n_act = int(r.n_active.item())
    assert n_act == active.size
    np.testing.assert_array_equal(r.active_ids.cpu().numpy()[:n_act], active)


@pytest.mark.parametrize("T,E,k", [(1, 384, 8), (16, 384, 8), (37, 40, 8), (7, 1024, 32), (512, 384, 8),
                                   (513, 384, 8), (3, 5, 2), (128, 12, 4)])
def test_route_topk_permute_fused_equals_the_two_calls(api, T, E, k):
    # up to 4096 routes one launch (shared-memory ids), beyond it the two calls; either
    # way the same arrays as route_topk + route_permute, and the oracle's grouping
    rng = np.random.default_rng(900 + T + E + k)
    logits = torch.from_numpy(inputs.normal_logits(rng, T, E)).cuda()
    ids, w, r = api.route_topk_permute(logits, k, E)
    ids2, w2 = api.route_topk(logits, k)
    r2 = api.route_permute(ids2, E)
    torch.cuda.synchronize()
    assert torch.equal(ids, ids2) and torch.equal(w, w2)
    for name in ("counts", "offsets", "perm", "inv"):
        assert torch.equal(getattr(r, name), getattr(r2, name)), name
    n_act = int(r.n_active.item())
    assert n_act == int(r2.n_active.item())
    assert torch.equal(r.active_ids[:n_act], r2.active_ids[:n_act])
    counts, offsets, perm, inv = OL.route_permute(ids.cpu().numpy(), E)
    np.testing.assert_array_equal(r.perm.cpu().numpy(), perm)
    np.testing.assert_array_equal(r.inv.cpu().numpy(), inv)
    assert api.device_status() == 0


@pytest.mark.parametrize("T,k,E", [(2048, 8, 384), (2500, 8, 1024), (2051, 8, 7), (40000, 8, 384)])
def test_route_permute_multi_block_exact(api, T, k, E):
    # T*k >= 16384 takes the multi-CTA grouping (4096-route blocks, ragged last block);
    # a few out-of-range ids are dropped (inv = -1) and raise device flag bit 0.
    rng = np.random.default_rng(T + E)
    logits = inputs.zipf_gumbel_logits(rng, T, E) if E >= 8 else inputs.normal_logits(rng, T, E)
    rid, _ = OL.route_topk(logits, min(k, E))
    if rid.shape[1] < k:
        rid = np.concatenate([rid, rid[:, :k - rid.shape[1]]], axis=1)
    bad = rng.choice(rid.size, 5, replace=False)
    rid_bad = rid.copy().reshape(-1)
    rid_bad[bad[:3]] = E
    rid_bad[bad[3:]] = -7
    rid_bad = rid_bad.reshape(rid.shape)
    api.device_status(clear=True)
    r = api.route_permute(torch.from_numpy(rid_bad).cuda(), E)
    torch.cuda.synchronize()
    assert api.device_status(clear=True) == 1
    valid = (rid_bad >= 0) & (rid_bad < E)
    ref_ids = np.where(valid, rid_bad, 0).reshape(-1)
    counts = np.bincount(ref_ids[valid.reshape(-1)], minlength=E).astype(np.int32)
    order = np.argsort(np.where(valid.reshape(-1), ref_ids, E), kind="stable")[:valid.sum()]
    np.testing.assert_array_equal(r.counts.cpu().numpy(), counts)
    np.testing.assert_array_equal(r.offsets.cpu().numpy()[1:], np.cumsum(counts))
    np.testing.assert_array_equal(r.perm.cpu().numpy()[:valid.sum()], order)
    inv = r.inv.cpu().numpy()
    assert np.all(inv[~valid.reshape(-1)] == -1)
    np.testing.assert_array_equal(inv[order], np.arange(order.size))
    # and, without bad ids, exactly the oracle's grouping
    r2 = api.route_permute(torch.from_numpy(rid).cuda(), E)
    c2, o2, p2, i2 = OL.route_permute(rid, E)
    np.testing.assert_array_equal(r2.perm.cpu().numpy(), p2)
    np.testing.assert_array_equal(r2.inv.cpu().numpy(), i2)
    np.testing.assert_array_equal(r2.offsets.cpu().numpy(), o2)
    n_act = int(r2.n_active.item())
    np.testing.assert_array_equal(r2.active_ids.cpu().numpy()[:n_act], np.nonzero(c2)[0])


@pytest.mark.parametrize("T,k,D", [(1, 8, 4096), (16, 8, 4096), (37, 3, 256)])
def test_route_unpermute(api, T, k, D):
    rng = np.random.default_rng(T + k + D)
    E = 50
    rid, rw = OL.route_topk(inputs.normal_logits(rng, T, E), k)
    _, _, _, inv = OL.route_permute(rid, E)
    y = rng.standard_normal((T * k, D)).astype(np.float32)
    w32 = rw.astype(np.float32)
    out = api.route_unpermute(torch.from_numpy(y).cuda(), torch.from_numpy(inv).cuda(),
                              torch.from_numpy(w32).cuda())
    ref = OL.combine(y, inv, w32)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=1e-5, atol=1e-5)
