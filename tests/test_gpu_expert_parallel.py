"""Expert parallelism with the library's kernels: ExpertParallelMoE must give the same
bits as the single-GPU layer (api.moe_layer) on the same expert path, since every route
is computed from the same row and weights and combined on its token's rank in slot
order.  One rank over NCCL in this process (both expert paths), and two gloo ranks as
two processes sharing one GPU (their kernels never wait on each other: the exchanges
go through host memory)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from tests.conftest import ROOT

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(seed, T, layer):
    from trellis_quantized_moe_gemv_b200 import inputs
    rng = np.random.default_rng(seed)
    x = inputs.random_activations(rng, (T, layer.D), "bf16")
    logits = inputs.normal_logits(rng, T, layer.E)
    return torch.from_numpy(x).to(torch.bfloat16).cuda(), torch.from_numpy(logits).cuda()


def _single_gpu(layer, x, logits, k, path):
    from trellis_quantized_moe_gemv_b200 import api
    dl = api.DeviceLayer.from_synthetic(layer)
    out = api.moe_layer(dl, x, logits, k, path=path).clone()
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("path,T,signed", [("gemv", 24, False), ("gemm", 40, False), ("gemv", 10, True)])
def test_one_rank_nccl_bit_identical_to_single_gpu(path, T, signed):
    import torch.distributed as dist
    from trellis_quantized_moe_gemv_b200 import api, expert_parallel as EP, inputs
    import trellis_quantized_moe_gemv_b200.build as b
    b.build()
    layer = inputs.small_layer(610, E=12, D=512, F=256, split={2: 8, 3: 3, 4: 1})
    if signed:
        layer = inputs.with_signs(layer, 611)
    x, logits = _inputs(612, T, layer)
    k = 4
    ref = _single_gpu(layer, x, logits, k, path)
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % _free_port(), rank=0, world_size=1)
    try:
        moe = EP.ExpertParallelMoE(layer, k, path=path)
        got = moe.forward(x, logits)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(got, ref)
    assert api.device_status() == 0


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from trellis_quantized_moe_gemv_b200 import api, expert_parallel as EP, inputs
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    torch.cuda.set_device(0)
    layer = inputs.small_layer(620, E=12, D=512, F=256, split={2: 8, 3: 3, 4: 1})
    x, logits = _inputs(621 + rank, 6 + 5 * rank, layer)
    k = 4
    ref = _single_gpu(layer, x, logits, k, "gemv")
    moe = EP.ExpertParallelMoE(layer, k, path="gemv")
    for _ in range(2):                     # a second call reuses nothing stale
        got = moe.forward(x, logits)
    torch.cuda.synchronize()
    out[rank] = (bool(torch.equal(got, ref)), int(api.device_status()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_on_one_gpu_bit_identical_to_single_gpu():
    import trellis_quantized_moe_gemv_b200.build as b
    b.build()
    mgr = mp.get_context("spawn").Manager()   # no fork after CUDA is initialised
    out = mgr.dict()
    mp.spawn(_worker, args=(2, _free_port(), out), nprocs=2, join=True)
    for rank in range(2):
        assert out[rank] == (True, 0), (rank, out[rank])


def test_route_gather_rows_copies_bits_and_flags_bad_indices():
    from trellis_quantized_moe_gemv_b200 import api
    import trellis_quantized_moe_gemv_b200.build as b
    b.build()
    api.device_status(clear=True)
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    for dtype, cols in ((torch.float16, 256), (torch.bfloat16, 8), (torch.float32, 4), (torch.float32, 4096)):
        src = torch.randn((37, cols), generator=g, device="cuda").to(dtype)
        idx = torch.randint(0, 37 * 3, (101,), generator=g, device="cuda", dtype=torch.int32)
        got = api.route_gather_rows(src, idx, 3)
        assert torch.equal(got.view(torch.int16 if dtype != torch.float32 else torch.int32),
                           src[idx.long() // 3].view(torch.int16 if dtype != torch.float32 else torch.int32))
    assert api.device_status() == 0
    src = torch.ones((4, 8), dtype=torch.float32, device="cuda")
    idx = torch.tensor([0, 4, -1, 3], dtype=torch.int32, device="cuda")
    got = api.route_gather_rows(src, idx, 1)
    torch.cuda.synchronize()
    assert got[0].eq(1).all() and got[3].eq(1).all() and got[1].eq(0).all() and got[2].eq(0).all()
    assert api.device_status(clear=True) & 1
