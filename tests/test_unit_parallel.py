"""Intermediate-unit tensor parallelism on CPU: the ownership rule, the cut of every
expert's bit streams into rank slices (checked against the oracle's decode of the full
matrices), and UnitParallelMoE with gloo ranks (world size 2 and 4) whose per-rank layer
is the oracle's: the all-reduced output must equal the oracle's full layer."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_unit_owner_rule_partitions_units():
    from trellis_quantized_moe_gemv_b200 import unit_parallel as UP
    # closed form of the rule at a few points: (18 e + u + L) mod N
    assert UP.unit_owner(0, 0, 0, 8) == 0
    assert UP.unit_owner(1, 0, 0, 8) == 2
    assert UP.unit_owner(5, 7, 3, 8) == (90 + 7 + 3) % 8 == 4
    assert UP.unit_owner(383, 1, 42, 3) == (18 * 383 + 1 + 42) % 3
    for N in (1, 2, 4, 8):
        for e in (0, 1, 17, 383):
            for L in (0, 5):
                seen = sorted(u for r in range(N) for u in UP.owned_units(e, 8, r, N, L))
                assert seen == list(range(8))
                assert all(len(UP.owned_units(e, 8, r, N, L)) == 8 // N for r in range(N))


def test_slices_decode_to_the_owned_rows_and_columns():
    from oracle import layer as OL
    from trellis_quantized_moe_gemv_b200 import inputs, unit_parallel as UP
    layer = inputs.small_layer(700, E=6, D=256, F=512, split={2: 3, 3: 2, 4: 1})
    full = OL.ExpertWeights(layer)
    world, L = 4, 1
    for rank in range(world):
        sl = UP.unit_slice_layer(layer, rank, world, L)
        assert sl.F == 128
        part = OL.ExpertWeights(sl)
        for e in range(layer.E):
            units = UP.owned_units(e, 4, rank, world, L)
            chans = np.concatenate([np.arange(128 * u, 128 * u + 128) for u in units])
            np.testing.assert_array_equal(part.matrix(e, "gate"), full.matrix(e, "gate")[chans])
            np.testing.assert_array_equal(part.matrix(e, "up"), full.matrix(e, "up")[chans])
            np.testing.assert_array_equal(part.matrix(e, "down"), full.matrix(e, "down")[:, chans])


def test_slice_rejects_unsupported_layers():
    from trellis_quantized_moe_gemv_b200 import inputs, unit_parallel as UP
    layer = inputs.small_layer(701, E=4, D=256, F=256)
    with pytest.raises(ValueError):
        UP.unit_slice_layer(layer, 0, 4, 0)            # 2 units over 4 ranks
    with pytest.raises(ValueError):
        UP.unit_slice_layer(inputs.with_signs(layer, 702), 0, 2, 0)


def _oracle_compute(slice_layer, x, logits, k):
    from oracle import layer as OL
    return torch.from_numpy(OL.moe_layer(slice_layer, x.numpy(), logits.numpy(), k)["out"])


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from oracle import layer as OL
    from trellis_quantized_moe_gemv_b200 import inputs, unit_parallel as UP
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    layer = inputs.small_layer(710, E=6, D=256, F=512, split={2: 3, 3: 2, 4: 1})
    rng = np.random.default_rng(711)                  # every rank holds the same tokens
    x = inputs.random_activations(rng, (5, layer.D), "bf16")
    logits = inputs.normal_logits(rng, 5, layer.E)
    moe = UP.UnitParallelMoE(layer, 2, layer_index=2, compute=_oracle_compute)
    got = moe.forward(torch.from_numpy(np.asarray(x, dtype=np.float64)), torch.from_numpy(logits)).numpy()
    ref = OL.moe_layer(layer, x, logits, 2)["out"]
    out[rank] = (float(np.abs(got - ref).max()), float(np.abs(ref).max()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_all_reduced_slices_equal_the_full_layer(world):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        err, scale = out[rank]
        assert err <= 1e-12 * max(scale, 1.0), (rank, err, scale)
