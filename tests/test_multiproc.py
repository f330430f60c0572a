"""Host logic of the multi-GPU path on CPU: `bench.py --gpus N` runs N independent
replicas (one process per GPU, no data-path collective) and reports all ranks' tokens
over the max-over-ranks time.  Checked here with world_size 2 on the gloo backend."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms_local = [40.0, 55.0][rank]
    ms_max, value = bench.aggregate_ranks(ms_local, tokens_per_rank=160, world=world, device="cpu")
    out[rank] = (ms_max, value)
    dist.barrier()
    dist.destroy_process_group()


def test_replicas_take_max_over_ranks_and_sum_tokens():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        ms_max, value = out[rank]
        assert ms_max == 55.0
        assert value == pytest.approx(2 * 160 / 0.055)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate_ranks(20.0, 100, 1) == (20.0, 100 / 0.020)


def test_reference_arm_prints_only_on_rank_zero():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
