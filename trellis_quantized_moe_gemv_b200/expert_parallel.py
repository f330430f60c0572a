"""Expert parallelism for the trellis-coded MoE layer: one process per GPU, each rank
owning a contiguous block of the layer's experts.

The pages run the layer on one GPU ("DeepSeek-V4.1-Flash-1017 · dsx T16" model card,
"How T16 works"); sharding its experts over ranks adds one exchange in each direction
around the unchanged expert computation:

1. every rank routes its own tokens (top-k, grouping by expert) and rotates them;
2. dispatch: the routes' rotated rows, laid out in expert-grouped order, go to the ranks
   that own their experts (one all-to-all; expert-grouped order is rank-grouped order
   because each rank owns a contiguous id range);
3. each rank runs the routed experts it owns on the rows it received (the trellis GEMV or
   GEMM with one route per row) and puts the results back into arrival order;
4. combine: the results return along the same paths (the reverse all-to-all), landing in
   the sender's expert-grouped route order -- the single-GPU y_perm -- and the sender
   adds its k routes per token in slot order.

Every per-route result is computed from the same row and the same expert weights as on
one GPU, and the combine runs on the token's own rank in the same slot order, so with
the same expert path the output is bit-identical to the single-GPU layer.

Row movement and the expert computation go through an ``ops`` object; the default,
``KernelOps``, runs the library's kernels on the rank's GPU.  The exchanges use
``torch.distributed`` collectives: NCCL moves device tensors directly; with a gloo
process group the rows are staged through host memory.
"""
from typing import List, Optional

import numpy as np
import torch
import torch.distributed as dist

from . import api


def expert_bounds(E: int, world: int) -> List[int]:
    """Rank r owns experts [b[r], b[r+1]) (contiguous, sizes differing by at most one)."""
    if not 1 <= world <= E:
        raise ValueError("expert parallelism needs 1 <= world size <= E")
    return [(r * E) // world for r in range(world + 1)]


def owned_groups(layer, lo: int, hi: int) -> List[dict]:
    """The width groups of a synthetic layer restricted to experts [lo, hi)."""
    out = []
    for g in layer.groups:
        sel = np.nonzero((g.ids >= lo) & (g.ids < hi))[0]
        if sel.size:
            out.append(dict(K=g.K, ids=g.ids[sel], gate=g.gate[sel], up=g.up[sel], down=g.down[sel],
                            s_gate=g.s_gate[sel], s_up=g.s_up[sel], s_down=g.s_down[sel]))
    return out


class KernelOps:
    """The expert-parallel steps on this rank's GPU, each one library call."""

    result_dtype = torch.float32      # dtype of experts() results (and of the combine's input)

    def __init__(self, layer, lo: int, hi: int, device="cuda", path: str = "auto"):
        groups = owned_groups(layer, lo, hi)
        if not groups:
            raise ValueError("rank owns no experts")
        self.dl = api.DeviceLayer(layer.E, layer.D, layer.F, groups, device, getattr(layer, "signs", None))
        self.E, self.D = layer.E, layer.D
        self.device = torch.device(device)
        self.path = path

    def route(self, logits: torch.Tensor, k: int):
        ids, w = api.route_topk(logits, k)
        return w, api.route_permute(ids, self.E)

    def rotate(self, x: torch.Tensor) -> torch.Tensor:
        if self.dl.signs is not None:
            return api.hadamard128_signed(x, self.dl.signs["x"])
        return api.hadamard128(x)

    def gather(self, src: torch.Tensor, index: torch.Tensor, divisor: int) -> torch.Tensor:
        return api.route_gather_rows(src, index, divisor)

    def experts(self, rows: torch.Tensor, expert_ids: torch.Tensor, k_global: int, world: int) -> torch.Tensor:
        """y [R, D] fp32 of rows [R, D] fp16, row i routed to expert_ids[i], in row order."""
        R = rows.shape[0]
        ids = expert_ids.to(device=self.device, dtype=torch.int32).reshape(R, 1).contiguous()
        routing = api.route_permute(ids, self.E)
        # the single-GPU switch point in routes per expert: T * k / E at T = GEMM_MIN_TOKENS
        use_gemm = self.path == "gemm" or (self.path == "auto" and R * world >= api.GEMM_MIN_TOKENS * k_global)
        fn = api.moe_trellis_gemm if use_gemm else api.moe_trellis_gemv
        y_perm = fn(self.dl, rows, routing, R, 1)
        return api.route_gather_rows(y_perm, routing.inv, 1)

    def combine(self, y_perm: torch.Tensor, inv: torch.Tensor, w: torch.Tensor) -> torch.Tensor:
        if self.dl.signs is not None:
            return api.route_unpermute_signed(y_perm, inv, w, self.dl.signs["y"])
        return api.route_unpermute(y_perm, inv, w)


class ExpertParallelMoE:
    """The routed experts of one MoE layer sharded by expert over a process group.

    layer: the host-side synthetic layer (every rank passes the same one; each keeps its
    own experts).  forward(x [T, D], logits [T, E]) -> out [T, D] fp32 for this rank's
    tokens; T may differ between ranks.  Every rank must call forward the same number
    of times (the exchanges are collectives)."""

    def __init__(self, layer, k: int, group=None, ops=None, device="cuda", path: str = "auto"):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.E, self.D, self.k = layer.E, layer.D, k
        self.bounds = expert_bounds(self.E, self.world)
        self.lo, self.hi = self.bounds[self.rank], self.bounds[self.rank + 1]
        self.ops = ops if ops is not None else KernelOps(layer, self.lo, self.hi, device, path)
        # gloo moves host tensors only
        self.host = dist.get_backend(group) == "gloo"

    def _all_to_all(self, t: torch.Tensor, out_rows: List[int], in_rows: List[int]) -> torch.Tensor:
        src = t.cpu() if self.host else t
        out = torch.empty((sum(out_rows),) + tuple(t.shape[1:]), dtype=t.dtype, device=src.device)
        dist.all_to_all_single(out, src.contiguous(), out_rows, in_rows, group=self.group)
        return out.to(t.device) if self.host else out

    def forward(self, x: torch.Tensor, logits: torch.Tensor) -> torch.Tensor:
        ops, k, b = self.ops, self.k, self.bounds
        w, routing = ops.route(logits, k)
        x_rot = ops.rotate(x)
        send = ops.gather(x_rot, routing.perm, k)          # [T*k, D], expert-grouped
        # routes per expert of every rank (one small host copy and one small collective)
        off = routing.offsets.to("cpu", torch.int64)
        counts = (off[1:] - off[:-1]).contiguous()
        if not self.host:
            counts = counts.to(x.device)
        gathered = [torch.empty_like(counts) for _ in range(self.world)]
        dist.all_gather(gathered, counts, group=self.group)
        gathered = [g.cpu() for g in gathered]
        send_rows = [int(off[b[r + 1]] - off[b[r]]) for r in range(self.world)]
        recv_rows = [int(g[self.lo:self.hi].sum()) for g in gathered]
        # rows arrive per source rank, each source's rows grouped by expert in id order
        mine = torch.arange(self.lo, self.hi, dtype=torch.int64)
        expert_ids = torch.cat([torch.repeat_interleave(mine, g[self.lo:self.hi]) for g in gathered])
        recv = self._all_to_all(send, recv_rows, send_rows)
        if recv.shape[0]:
            y_recv = ops.experts(recv, expert_ids, k, self.world)
        else:
            y_recv = torch.empty((0, self.D), dtype=ops.result_dtype, device=recv.device)
        y_perm = self._all_to_all(y_recv, send_rows, recv_rows)   # the sender's y_perm
        return ops.combine(y_perm, routing.inv, w)
