"""Intermediate-unit tensor parallelism with the library's kernels: one NCCL rank is the
single-GPU layer bit for bit (its slice is the whole layer); two gloo ranks as two
processes on one GPU (all-reduce through host memory, no kernel waits on another
rank's) must match the oracle's full layer within its error bound, each rank having run
the GEMV or GEMM on its own units."""
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


def _case():
    from trellis_quantized_moe_gemv_b200 import inputs
    layer = inputs.small_layer(720, E=12, D=512, F=512, split={2: 8, 3: 3, 4: 1})
    rng = np.random.default_rng(721)
    x = inputs.random_activations(rng, (40, layer.D), "bf16")
    logits = inputs.normal_logits(rng, 40, layer.E)
    return layer, x, logits


def test_one_nccl_rank_bit_identical_to_single_gpu():
    import torch.distributed as dist
    import trellis_quantized_moe_gemv_b200.build as b
    b.build()
    from trellis_quantized_moe_gemv_b200 import api, unit_parallel as UP
    layer, x, logits = _case()
    xd = torch.from_numpy(x).to(torch.bfloat16).cuda()
    ld = torch.from_numpy(logits).cuda()
    dl = api.DeviceLayer.from_synthetic(layer)
    ref = api.moe_layer(dl, xd, ld, 4, path="gemv").clone()
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % _free_port(), rank=0, world_size=1)
    try:
        got = UP.UnitParallelMoE(layer, 4, path="gemv").forward(xd, ld)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(got, ref)


def _worker(rank, world, port, path, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from oracle import layer as OL
    from trellis_quantized_moe_gemv_b200 import api, unit_parallel as UP
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    torch.cuda.set_device(0)
    layer, x, logits = _case()
    xd = torch.from_numpy(x).to(torch.bfloat16).cuda()
    ld = torch.from_numpy(logits).cuda()
    moe = UP.UnitParallelMoE(layer, 4, layer_index=1, path=path)
    for _ in range(2):
        got = moe.forward(xd, ld)
    torch.cuda.synchronize()
    res = OL.moe_layer(layer, x, logits, 4)
    tol = res["bound"] + 1e-6 * np.abs(res["out"]) + 1e-12
    err = np.abs(got.cpu().numpy().astype(np.float64) - res["out"])
    out[rank] = (float((err / tol).max()), int(api.device_status()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("path", ["gemv", "gemm"])
def test_two_gloo_ranks_match_the_oracle(path):
    import trellis_quantized_moe_gemv_b200.build as b
    b.build()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, _free_port(), path, out), nprocs=2, join=True)
    for rank in range(2):
        ratio, status = out[rank]
        assert ratio <= 1.0 and status == 0, (rank, ratio, status)
