"""Expert parallelism on CPU: ExpertParallelMoE's dispatch / combine with gloo ranks
(world size 2 and 3), its per-rank steps supplied by the oracle.  Every rank's output
must equal the oracle's single-process layer for that rank's tokens: the exchanges must
deliver each route's row to its expert's owner and bring each result back to the
sender's expert-grouped slot, including ranks that receive no rows at all."""
import os
import socket
import sys
from types import SimpleNamespace

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The per-rank steps in fp64 numpy (test stand-in for the GPU kernels)."""

    result_dtype = torch.float64

    def __init__(self, layer, lo, hi):
        from oracle import layer as OL
        self.OL, self.layer, self.lo, self.hi = OL, layer, lo, hi
        self.weights = OL.ExpertWeights(layer)
        self.signs = getattr(layer, "signs", None)
        self.expert_rows = 0

    def route(self, logits, k):
        ids, w = self.OL.route_topk(logits.numpy(), k)
        _, offsets, perm, inv = self.OL.route_permute(ids, self.layer.E)
        return torch.from_numpy(w), SimpleNamespace(offsets=torch.from_numpy(offsets),
                                                    perm=torch.from_numpy(perm), inv=torch.from_numpy(inv))

    def rotate(self, x):
        return torch.from_numpy(self.OL.rotate_in(x.numpy(), None if self.signs is None else self.signs["x"]))

    def gather(self, src, index, divisor):
        return src[index.long() // divisor].contiguous()

    def experts(self, rows, expert_ids, k, world):
        y = np.zeros((rows.shape[0], self.layer.D))
        for i, e in enumerate(expert_ids.tolist()):
            assert self.lo <= e < self.hi, "row sent to a rank that does not own its expert"
            y[i] = self.OL.expert_forward(self.weights, e, rows[i:i + 1].numpy(), signs=self.signs)["y"][0]
        self.expert_rows += rows.shape[0]
        return torch.from_numpy(y)

    def combine(self, y_perm, inv, w):
        return torch.from_numpy(self.OL.combine(y_perm.numpy(), inv.numpy(), w.numpy()))


def _case(rank, hot, empty_rank=-1):
    from trellis_quantized_moe_gemv_b200 import inputs
    layer = inputs.small_layer(321, E=6, D=256, F=128, split={2: 4, 3: 1, 4: 1})
    if hot:
        layer = inputs.with_signs(layer, 322)
    rng = np.random.default_rng(400 + rank)
    T = 0 if rank == empty_rank else 3 + 2 * rank     # ranks hold different token counts
    x = inputs.random_activations(rng, (T, layer.D), "bf16")
    logits = inputs.normal_logits(rng, T, layer.E)
    if hot:
        logits[:, :3] += 50.0                         # every route to experts 0..2
    return layer, x, logits


def _worker(rank, world, port, hot, out, empty_rank=-1):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from oracle import layer as OL
    from trellis_quantized_moe_gemv_b200 import expert_parallel as EP
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    layer, x, logits = _case(rank, hot, empty_rank)
    k = 2
    b = EP.expert_bounds(layer.E, world)
    ops = OracleOps(layer, b[rank], b[rank + 1])
    moe = EP.ExpertParallelMoE(layer, k, ops=ops)
    got = moe.forward(torch.from_numpy(np.asarray(x, dtype=np.float64)), torch.from_numpy(logits))
    ref = OL.moe_layer(layer, x, logits, k)["out"] if x.shape[0] else np.zeros((0, layer.D))
    assert got.shape == ref.shape
    out[rank] = (float(np.abs(got.numpy() - ref).max(initial=0.0)), float(np.abs(ref).max(initial=0.0)),
                 ops.expert_rows, int(x.shape[0]) * k)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,hot", [(2, False), (3, False), (2, True), (3, True)])
def test_dispatch_combine_matches_single_process_oracle(world, hot):
    mgr = mp.get_context("spawn").Manager()   # no fork after CUDA is initialised
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), hot, out), nprocs=world, join=True)
    total_routes = total_rows = 0
    for rank in range(world):
        err, scale, rows, routes = out[rank]
        assert err <= 1e-12 * max(scale, 1.0), (rank, err, scale)
        total_rows += rows
        total_routes += routes
    # every route computed exactly once, on its expert's owner
    assert total_rows == total_routes
    if hot:
        # routes to experts 0..2 only: the last rank owns none of them and receives nothing
        assert out[world - 1][2] == 0


def test_expert_bounds_cover_every_expert_once():
    from trellis_quantized_moe_gemv_b200 import expert_parallel as EP
    for E in (1, 6, 12, 384):
        for world in range(1, min(E, 9) + 1):
            b = EP.expert_bounds(E, world)
            assert b[0] == 0 and b[-1] == E
            sizes = np.diff(b)
            assert sizes.min() >= 1 and sizes.max() - sizes.min() <= 1
    with pytest.raises(ValueError):
        EP.expert_bounds(4, 5)


def test_owned_groups_keep_ids_and_arrays_together():
    from trellis_quantized_moe_gemv_b200 import expert_parallel as EP, inputs
    layer = inputs.small_layer(7, E=12, D=256, F=128, split={2: 8, 3: 3, 4: 1})
    seen = []
    for lo, hi in ((0, 4), (4, 8), (8, 12)):
        for g in EP.owned_groups(layer, lo, hi):
            src = next(s for s in layer.groups if s.K == g["K"])
            for i, e in enumerate(g["ids"]):
                assert lo <= e < hi
                j = int(np.nonzero(src.ids == e)[0][0])
                np.testing.assert_array_equal(g["gate"][i], src.gate[j])
                np.testing.assert_array_equal(g["s_down"][i], src.s_down[j])
                seen.append(int(e))
    assert sorted(seen) == list(range(12))


def test_rank_without_tokens_still_serves_its_experts():
    # rank 0 holds no tokens this step but owns experts that rank 1's tokens use
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, _free_port(), False, out, 0), nprocs=2, join=True)
    assert out[0][3] == 0 and out[0][2] > 0          # no routes of its own, rows served
    for rank in range(2):
        err, scale, rows, routes = out[rank]
        assert err <= 1e-12 * max(scale, 1.0), (rank, err, scale)
    assert out[0][2] + out[1][2] == out[1][3]
