"""Intermediate-unit tensor parallelism for the trellis-coded MoE layer: every rank holds
a share of each expert's intermediate channels and the partial outputs are summed.

"DeepSeek-V4.1-Flash-1017 · dsx T16" model card, section "Layout": every expert
projection is cut into units of 128 intermediate channels, and at tensor-parallel size N
unit u of expert e in layer L belongs to rank (18·e + u + L) mod N.  A rank's slice of
an expert is then a smaller expert of the same form: its gate and up rows and its down
columns restricted to the owned units (whole 16-row strips of gate/up, whole 16-column
tile columns of down, so the bit streams are cut along tile boundaries and never
re-encoded).  The 128-wide rotation of h acts inside each unit, so it commutes with the
cut; SiLU·up is per channel; and the down projection is a sum over channels, so the
layer output is the sum over ranks of each rank's output on its slice (one all-reduce).

Limits of this reading: N must divide the number of units F/128 (each rank then owns
F/(128·N) units of every expert and every rank's slice has the same width), and the
layer must use the input-side rotation only -- the two-sided transform's sign vectors
for g, u and h are shared by all experts of a layer, while the owned channels differ
from expert to expert.
"""
from types import SimpleNamespace
from typing import List

import numpy as np
import torch
import torch.distributed as dist

from . import api

UNIT = 128      # intermediate channels per unit


def unit_owner(e: int, u: int, layer_index: int, world: int) -> int:
    """Rank owning unit u of expert e in layer `layer_index` at tensor-parallel size world."""
    return (18 * e + u + layer_index) % world


def owned_units(e: int, n_units: int, rank: int, world: int, layer_index: int = 0) -> List[int]:
    return [u for u in range(n_units) if unit_owner(e, u, layer_index, world) == rank]


def _rows_of(units, per_unit):
    return np.concatenate([np.arange(u * per_unit, (u + 1) * per_unit) for u in units])


def unit_slice_layer(layer, rank: int, world: int, layer_index: int = 0):
    """The experts of `layer` restricted to the units `rank` owns (a layer of width
    F / world with the same experts, widths and down scales)."""
    if getattr(layer, "signs", None) is not None:
        raise ValueError("unit parallelism needs the input-side-only layer (no shared g/u/h signs)")
    D, F = layer.D, layer.F
    n_units = F // UNIT
    if F % UNIT or n_units % world:
        raise ValueError("the number of 128-channel units must be a multiple of the world size")
    Fr = F // world
    groups = []
    for g in layer.groups:
        W = 8 * g.K                                   # words per 16x16 tile
        n = len(g.ids)
        gate = np.empty((n, (Fr // 16) * (D // 16) * W), dtype=np.uint32)
        up = np.empty_like(gate)
        down = np.empty((n, (D // 16) * (Fr // 16) * W), dtype=np.uint32)
        s_gate = np.empty((n, Fr), dtype=np.float16)
        s_up = np.empty_like(s_gate)
        for i, e in enumerate(np.asarray(g.ids).tolist()):
            units = owned_units(e, n_units, rank, world, layer_index)
            strips = _rows_of(units, UNIT // 16)          # 16-row strips of gate/up, tile columns of down
            chans = _rows_of(units, UNIT)
            gate[i] = np.asarray(g.gate[i]).reshape(F // 16, D // 16, W)[strips].reshape(-1)
            up[i] = np.asarray(g.up[i]).reshape(F // 16, D // 16, W)[strips].reshape(-1)
            down[i] = np.asarray(g.down[i]).reshape(D // 16, F // 16, W)[:, strips].reshape(-1)
            s_gate[i] = np.asarray(g.s_gate[i])[chans]
            s_up[i] = np.asarray(g.s_up[i])[chans]
        groups.append(SimpleNamespace(K=g.K, ids=np.asarray(g.ids), gate=gate, up=up, down=down,
                                      s_gate=s_gate, s_up=s_up, s_down=np.asarray(g.s_down)))
    return SimpleNamespace(E=layer.E, D=D, F=Fr, expert_bits=getattr(layer, "expert_bits", None),
                           groups=groups, signs=None)


class UnitParallelMoE:
    """The routed experts of one MoE layer with each expert's intermediate units spread
    over a process group.  Every rank passes the same layer and the same tokens;
    forward(x [T, D], logits [T, E]) returns the full out [T, D] fp32 on every rank."""

    def __init__(self, layer, k: int, group=None, layer_index: int = 0, device="cuda", path: str = "auto",
                 compute=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.k, self.path = k, path
        self.slice = unit_slice_layer(layer, self.rank, self.world, layer_index)
        # compute(slice, x, logits, k) -> this rank's partial out; default: the library's
        # layer on this rank's GPU
        self.compute = compute
        self.dl = None if compute is not None else api.DeviceLayer.from_synthetic(self.slice, device)
        self._bufs = {}
        self.host = dist.get_backend(group) == "gloo"    # gloo reduces host tensors only

    def _partial(self, x, logits):
        if self.compute is not None:
            return self.compute(self.slice, x, logits, self.k)
        T = x.shape[0]
        if T not in self._bufs:
            self._bufs[T] = api.MoeBuffers(self.dl, T, self.k)
        return api.moe_layer(self.dl, x, logits, self.k, bufs=self._bufs[T], path=self.path)

    def forward(self, x: torch.Tensor, logits: torch.Tensor) -> torch.Tensor:
        part = self._partial(x, logits)
        if self.host:
            buf = part.cpu()
            dist.all_reduce(buf, group=self.group)
            return buf.to(part.device)
        out = part.clone()
        dist.all_reduce(out, group=self.group)
        return out
