"""GPU parity of trellis_encode against the oracle's tail-biting Viterbi encoder: the
streams and per-tile costs must be identical (integer search, same tie rules)."""
import numpy as np
import pytest
import torch

from oracle import encode as OE
from oracle import t16 as OT

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    import trellis_quantized_moe_gemv_b200.build as b
    b.build()
    from trellis_quantized_moe_gemv_b200 import api as A
    A.device_status(clear=True)
    return A


def gaussian_targets(seed, rows, cols, sigma=80.0):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((rows, cols)) * sigma).astype(np.float32)
    x[0, 0] = 900.0           # clamped to tau = 1276
    x[1, 3] = -1000.0
    x[2, 5] = 0.125           # a quarter-unit half-way value: rint to even
    return x


@pytest.mark.parametrize("K,rows,cols", [(2, 32, 48), (3, 16, 64), (4, 48, 16)])
def test_encode_matches_oracle_bit_exactly(api, K, rows, cols):
    x = gaussian_targets(40 + K, rows, cols)
    bits, cost = api.trellis_encode(torch.from_numpy(x).cuda(), K)
    torch.cuda.synchronize()
    ref_bits, ref_cost = OE.encode_matrix(x, K)
    np.testing.assert_array_equal(bits.cpu().numpy().view(np.uint32), ref_bits)
    np.testing.assert_array_equal(cost.cpu().numpy().view(np.uint32).astype(np.int64), ref_cost)
    # and the GPU decoder reads the GPU streams as the oracle's decoder does
    codes = api.trellis_decode(bits, K, rows, cols).float().cpu().numpy()
    np.testing.assert_array_equal(codes, OT.decode_matrix(ref_bits, K, rows, cols))
    assert api.device_status() == 0


@pytest.mark.parametrize("K", [2, 3, 4])
def test_encode_closed_form_zero_stream(api, K):
    x = np.full((32, 32), -255.0, dtype=np.float32)
    bits, cost = api.trellis_encode(torch.from_numpy(x).cuda(), K)
    assert not bits.cpu().numpy().any()
    assert not cost.cpu().numpy().any()


def test_encode_many_tiles_persistent_grid(api):
    # more tiles than SMs: every CTA walks several tiles through its backpointer rows
    K, rows, cols = 4, 16 * 20, 16 * 16
    x = gaussian_targets(77, rows, cols, sigma=60.0)
    bits, cost = api.trellis_encode(torch.from_numpy(x).cuda(), K)
    got = bits.cpu().numpy().view(np.uint32)
    cst = cost.cpu().numpy().view(np.uint32)
    rng = np.random.default_rng(5)
    for t in rng.choice(20 * 16, 6, replace=False):
        i, j = divmod(int(t), 16)
        words, c, _ = OE.encode_tile(x[16 * i:16 * i + 16, 16 * j:16 * j + 16], K)
        np.testing.assert_array_equal(got[i, j], words)
        assert int(cst[i, j]) == c


def test_encode_rejects_bad_arguments(api):
    x = torch.zeros((16, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(api.TQError, match="INVALID"):
        api.trellis_encode(x, 5)
    with pytest.raises(api.TQError, match="WORKSPACE"):
        api.trellis_encode(x, 2, ws=torch.empty(16, dtype=torch.uint8, device="cuda"))


def test_encode_full_projection_sampled_tiles(api):
    # the benchmark's size: one 1024x4096 projection (16,384 tiles) at K = 2; sampled tiles
    # are re-encoded by the oracle one by one, and every tile's stream must decode to a
    # cost equal to the one the kernel reports
    K, rows, cols = 2, 1024, 4096
    g = torch.Generator(device="cuda")
    g.manual_seed(2002)
    x = torch.randn((rows, cols), generator=g, device="cuda") * 100.0
    bits, cost = api.trellis_encode(x, K)
    codes = api.trellis_decode(bits, K, rows, cols).double()       # exact integer sums in fp64
    tau = torch.clamp(torch.round(4.0 * x), -1276, 1276).double()
    err = ((tau - 4.0 * codes) ** 2).reshape(rows // 16, 16, cols // 16, 16).sum(dim=(1, 3))
    np.testing.assert_array_equal(err.cpu().numpy().astype(np.int64),
                                  cost.cpu().numpy().view(np.uint32).astype(np.int64))
    xs = x.cpu().numpy()
    got = bits.cpu().numpy().view(np.uint32)
    for t in (0, 5000, 16383):
        i, j = divmod(t, cols // 16)
        words, c, _ = OE.encode_tile(xs[16 * i:16 * i + 16, 16 * j:16 * j + 16], K)
        np.testing.assert_array_equal(got[i, j], words)
