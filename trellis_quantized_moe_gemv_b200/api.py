"""Thin Python binding of the C-ABI library ``libtrellis_moe.so``.

Every function here only marshals arguments (torch tensors -> device pointers, the
current CUDA stream) and calls the entry point of the same name; every step of the
computation runs in the library's CUDA kernels.  There is no CPU fallback: if the
library is missing or a call fails, a ``TQError`` is raised.

Bit streams are int32 tensors holding the uint32 words bit for bit; fp16 tensors carry
the scales and rotated activations; routing tensors are int32.
"""
import ctypes
import os
from dataclasses import dataclass
from typing import List, Optional

import numpy as np
import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libtrellis_moe.so")

TQ_DTYPE = {torch.float16: 0, torch.bfloat16: 1, torch.float32: 2}


class TQError(RuntimeError):
    """A library entry point returned an error status (or the library is missing)."""


class TqWidthGroup(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int), ("n_experts", ctypes.c_int),
                ("expert_ids", ctypes.c_void_p), ("gate", ctypes.c_void_p),
                ("up", ctypes.c_void_p), ("down", ctypes.c_void_p),
                ("s_gate", ctypes.c_void_p), ("s_up", ctypes.c_void_p),
                ("s_down", ctypes.c_void_p)]


class TqMoeLayer(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int), ("D", ctypes.c_int), ("F", ctypes.c_int),
                ("n_groups", ctypes.c_int), ("groups", TqWidthGroup * 3),
                ("expert_slot", ctypes.c_void_p),
                ("sign_x", ctypes.c_void_p), ("sign_gu", ctypes.c_void_p),
                ("sign_h", ctypes.c_void_p), ("sign_y", ctypes.c_void_p),
                ("codebook", ctypes.c_int)]

CODEBOOKS = {"t16": 0, "pair_e4m3": 1}


_lib = None
_VP, _I, _I64, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t

# entry point -> (argtypes, restype); mirrors include/trellis_moe.h
SIGNATURES = {
    "tq_status_string": ([_I], ctypes.c_char_p),
    "tq_abi_version": ([], _I),
    "tq_last_error_string": ([], ctypes.c_char_p),
    "tq_device_status": ([_VP, _I], _I),
    "tq_launch_count": ([], ctypes.c_ulonglong),
    "tq_profile_enable": ([_I], _I),
    "tq_profile_stages": ([ctypes.c_uint32], _I),
    "tq_selftest_bounded_wait": ([ctypes.c_uint32, _VP], _I),
    "tq_profile_disable": ([], _I),
    "tq_profile_collect": ([_VP, _VP, _I], _I),
    "trellis_decode": ([_VP, _I, _I, _I, _VP, _VP], _I),
    "trellis_decode_e4m3": ([_VP, _I, _I, _I, _VP, _VP], _I),
    "trellis_encode_workspace_size": ([_I, _I, _I], _SZ),
    "trellis_encode": ([_VP, _I, _I, _I, _VP, _VP, _VP, _SZ, _VP], _I),
    "hadamard128": ([_VP, _I, _I64, _I64, _VP, _VP], _I),
    "hadamard128_signed": ([_VP, _I, _I64, _I64, _VP, _VP, _VP], _I),
    "trellis_gemv_workspace_size": ([_I, _I, _I], _SZ),
    "trellis_gemv": ([_VP, _VP, _I, _I, _I, _VP, _I, _VP, _VP, _SZ, _VP], _I),
    "route_topk": ([_VP, _I, _I, _I, _VP, _VP, _VP], _I),
    "route_permute": ([_VP, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP], _I),
    "route_unpermute": ([_VP, _VP, _VP, _I, _I, _I, _VP, _VP], _I),
    "route_gather_rows": ([_VP, _I, _I64, _I, _VP, _I, _I64, _VP, _VP], _I),
    "route_topk_permute": ([_VP, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP], _I),
    "route_unpermute_signed": ([_VP, _VP, _VP, _I, _I, _I, _VP, _VP, _VP], _I),
    "moe_trellis_workspace_size": ([ctypes.POINTER(TqMoeLayer), _I, _I], _SZ),
    "moe_trellis_gemv": ([ctypes.POINTER(TqMoeLayer), _VP, _VP, _VP, _VP, _VP, _I, _I, _VP, _VP,
                          _SZ, _VP], _I),
    "moe_trellis_gemm": ([ctypes.POINTER(TqMoeLayer), _VP, _VP, _VP, _VP, _VP, _I, _I, _VP, _VP,
                          _SZ, _VP], _I),
    "moe_trellis_gemv_noalloc": ([ctypes.POINTER(TqMoeLayer), _VP, _VP, _VP, _VP, _VP, _I, _I, _VP,
                                  _VP], _I),
}


def lib():
    """The loaded library (raises TQError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise TQError("libtrellis_moe.so is not built (run __graft_entry__.build() or "
                          "python trellis_quantized_moe_gemv_b200/build.py)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(L, name, None)
            if fn is None:
                continue
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _fn(name):
    fn = getattr(lib(), name, None)
    if fn is None:
        raise TQError("entry point %s is not in this build" % name)
    return fn


def _check(status, name):
    if status != 0:
        msg = _fn("tq_status_string")(status).decode()
        if status == 5:
            msg += " (%s)" % _fn("tq_last_error_string")().decode()
        raise TQError("%s failed: %s" % (name, msg))


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _require(t, dtype, name, device=True):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if device and not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


# ----------------------------------------------------------------------------- entry points

def abi_version() -> int:
    return _fn("tq_abi_version")()


def device_status(clear: bool = False) -> int:
    """Device anomaly flags (bit 0: bad id skipped, bit 1: bounded wait gave up)."""
    out = ctypes.c_int32(0)
    _check(_fn("tq_device_status")(ctypes.byref(out), int(clear)), "tq_device_status")
    return out.value


STAGES = ("route_topk", "route_permute", "rotate_x", "moe_gemv", "rotate_h", "gemv_down",
          "route_unpermute", "trellis_decode", "trellis_gemv", "gemm_gateup", "gemm_down", "gemm_prep",
          "gemv_quant", "trellis_encode", "route_gather")


def launch_count() -> int:
    """Kernel launches issued by the library since it was loaded."""
    return int(_fn("tq_launch_count")())


def profile_enable(max_launches: int = 65536):
    _check(_fn("tq_profile_enable")(max_launches), "tq_profile_enable")


def selftest_bounded_wait(limit_us: int, stream=None):
    """Run the library's bounded device wait on a barrier nothing arrives on (gives up
    after limit_us and raises device flag bit 1)."""
    _check(_fn("tq_selftest_bounded_wait")(limit_us, _stream(stream)), "tq_selftest_bounded_wait")


def profile_stages(names=None):
    """Record only the launches of the named stages (all stages when names is None)."""
    mask = 0xFFFFFFFF if names is None else sum(1 << STAGES.index(n) for n in names)
    _check(_fn("tq_profile_stages")(mask), "tq_profile_stages")


def profile_disable():
    _check(_fn("tq_profile_disable")(), "tq_profile_disable")


def profile_collect() -> dict:
    """{stage: (total_ms, launches)} of the launches recorded since the last collect."""
    n = len(STAGES)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int32 * n)()
    _check(_fn("tq_profile_collect")(ms, cnt, n), "tq_profile_collect")
    return {STAGES[i]: (ms[i], cnt[i]) for i in range(n)}


def trellis_decode(bits: torch.Tensor, K: int, rows: int, cols: int,
                   out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _require(bits, torch.int32, "bits")
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.float16, device=bits.device)
    _require(out, torch.float16, "out")
    _check(_fn("trellis_decode")(_p(bits), K, rows, cols, _p(out), _stream(stream)), "trellis_decode")
    return out


def trellis_decode_e4m3(bits: torch.Tensor, K: int, rows: int, cols: int,
                        out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Pair-trellis bit streams -> E4M3 codes [rows, cols] (torch.float8_e4m3fn)."""
    _require(bits, torch.int32, "bits")
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.float8_e4m3fn, device=bits.device)
    _require(out, torch.float8_e4m3fn, "out")
    _check(_fn("trellis_decode_e4m3")(_p(bits), K, rows, cols, _p(out), _stream(stream)), "trellis_decode_e4m3")
    return out


def trellis_encode(target: torch.Tensor, K: int, bits: Optional[torch.Tensor] = None,
                   cost: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                   stream=None):
    """T16 bit streams [R/16][C/16][8K] (int32 words) for fp32 targets [R][C] in code units,
    and each tile's squared error in quarter code units [R/16][C/16] (int32 holding uint32)."""
    _require(target, torch.float32, "target")
    rows, cols = target.shape
    tiles = (rows // 16, cols // 16)
    if bits is None:
        bits = torch.empty(tiles + (8 * K,), dtype=torch.int32, device=target.device)
    if cost is None:
        cost = torch.empty(tiles, dtype=torch.int32, device=target.device)
    _require(bits, torch.int32, "bits")
    _require(cost, torch.int32, "cost")
    if ws is None:
        need = _fn("trellis_encode_workspace_size")(K, rows, cols)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=target.device)
    _check(_fn("trellis_encode")(_p(target), K, rows, cols, _p(bits), _p(cost), _p(ws), ws.numel(),
                                 _stream(stream)), "trellis_encode")
    return bits, cost


def hadamard128(x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if x.dtype not in TQ_DTYPE:
        raise TypeError("hadamard128: x must be fp16, bf16 or fp32")
    _require(x, x.dtype, "x")
    rows, cols = (x.shape[0], x.shape[1]) if x.dim() == 2 else (1, x.shape[-1])
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.float16, device=x.device)
    _require(out, torch.float16, "out")
    _check(_fn("hadamard128")(_p(x), TQ_DTYPE[x.dtype], rows, cols, _p(out), _stream(stream)),
           "hadamard128")
    return out


def hadamard128_signed(x: torch.Tensor, signs: torch.Tensor, out: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
    """rotate(signs * x) on every 128-chunk (the input side of the two-sided transform)."""
    if x.dtype not in TQ_DTYPE:
        raise TypeError("hadamard128_signed: x must be fp16, bf16 or fp32")
    _require(x, x.dtype, "x")
    _require(signs, torch.int8, "signs")
    rows, cols = (x.shape[0], x.shape[1]) if x.dim() == 2 else (1, x.shape[-1])
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.float16, device=x.device)
    _require(out, torch.float16, "out")
    _check(_fn("hadamard128_signed")(_p(x), TQ_DTYPE[x.dtype], rows, cols, _p(signs), _p(out),
                                     _stream(stream)), "hadamard128_signed")
    return out


def trellis_gemv_workspace_size(rows: int, cols: int, batch: int) -> int:
    return int(_fn("trellis_gemv_workspace_size")(rows, cols, batch))


def trellis_gemv(bits: torch.Tensor, scales: torch.Tensor, K: int, rows: int, cols: int,
                 x_rot: torch.Tensor, out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    _require(bits, torch.int32, "bits")
    _require(scales, torch.float16, "scales")
    _require(x_rot, torch.float16, "x_rot")
    batch = x_rot.shape[0]
    if out is None:
        out = torch.empty((batch, rows), dtype=torch.float32, device=x_rot.device)
    _require(out, torch.float32, "out")
    if ws is None:
        ws = torch.empty(max(trellis_gemv_workspace_size(rows, cols, batch), 16), dtype=torch.uint8,
                         device=x_rot.device)
    _check(_fn("trellis_gemv")(_p(bits), _p(scales), K, rows, cols, _p(x_rot), batch, _p(out), _p(ws),
                               ws.numel() * ws.element_size(), _stream(stream)), "trellis_gemv")
    return out


def route_topk(logits: torch.Tensor, k: int, ids: Optional[torch.Tensor] = None,
               w: Optional[torch.Tensor] = None, stream=None):
    _require(logits, torch.float32, "logits")
    T, E = logits.shape
    if ids is None:
        ids = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    if w is None:
        w = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    _check(_fn("route_topk")(_p(logits), T, E, k, _p(ids), _p(w), _stream(stream)), "route_topk")
    return ids, w


@dataclass
class Routing:
    """Device routing tensors of route_permute (route index i = t*k + s)."""
    counts: torch.Tensor
    offsets: torch.Tensor
    perm: torch.Tensor
    inv: torch.Tensor
    active_ids: torch.Tensor
    n_active: torch.Tensor

    @staticmethod
    def empty(T: int, k: int, E: int, device) -> "Routing":
        z = lambda n: torch.empty(n, dtype=torch.int32, device=device)
        return Routing(z(E), z(E + 1), z(T * k), z(T * k), z(E), z(1))


def route_permute(topk_ids: torch.Tensor, E: int, out: Optional[Routing] = None, stream=None) -> Routing:
    _require(topk_ids, torch.int32, "topk_ids")
    T, k = topk_ids.shape
    r = out if out is not None else Routing.empty(T, k, E, topk_ids.device)
    _check(_fn("route_permute")(_p(topk_ids), T, k, E, _p(r.counts), _p(r.offsets), _p(r.perm),
                                _p(r.inv), _p(r.active_ids), _p(r.n_active), _stream(stream)),
           "route_permute")
    return r


def route_topk_permute(logits: torch.Tensor, k: int, E: int, ids: Optional[torch.Tensor] = None,
                       w: Optional[torch.Tensor] = None, out: Optional["Routing"] = None, stream=None):
    """route_topk then route_permute (one launch for up to 4096 routes): (ids, w, routing)."""
    _require(logits, torch.float32, "logits")
    T = logits.shape[0]
    if ids is None:
        ids = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    if w is None:
        w = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    r = out if out is not None else Routing.empty(T, k, E, logits.device)
    _check(_fn("route_topk_permute")(_p(logits), T, E, k, _p(ids), _p(w), _p(r.counts), _p(r.offsets),
                                     _p(r.perm), _p(r.inv), _p(r.active_ids), _p(r.n_active), _stream(stream)),
           "route_topk_permute")
    return ids, w, r


def route_gather_rows(src: torch.Tensor, index: torch.Tensor, divisor: int = 1,
                      out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out[j] = src[index[j] // divisor] (rows copied bit for bit; fp16, bf16 or fp32)."""
    if src.dtype not in TQ_DTYPE:
        raise TypeError("route_gather_rows: src must be fp16, bf16 or fp32")
    _require(src, src.dtype, "src")
    _require(index, torch.int32, "index")
    rows = index.numel()
    if out is None:
        out = torch.empty((rows, src.shape[1]), dtype=src.dtype, device=src.device)
    _require(out, src.dtype, "out")
    _check(_fn("route_gather_rows")(_p(src), TQ_DTYPE[src.dtype], src.shape[0], src.shape[1], _p(index), divisor,
                                    rows, _p(out), _stream(stream)), "route_gather_rows")
    return out


def route_unpermute(y_perm: torch.Tensor, inv: torch.Tensor, topk_w: torch.Tensor,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _require(y_perm, torch.float32, "y_perm")
    _require(inv, torch.int32, "inv")
    _require(topk_w, torch.float32, "topk_w")
    T, k = topk_w.shape
    D = y_perm.shape[1]
    if out is None:
        out = torch.empty((T, D), dtype=torch.float32, device=y_perm.device)
    _require(out, torch.float32, "out")
    _check(_fn("route_unpermute")(_p(y_perm), _p(inv), _p(topk_w), T, k, D, _p(out),
                                  _stream(stream)), "route_unpermute")
    return out


def route_unpermute_signed(y_perm: torch.Tensor, inv: torch.Tensor, topk_w: torch.Tensor, signs_y: torch.Tensor,
                           out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Combine, then the down projection's output side: signs_y * rotate(sum_s w * y)."""
    _require(y_perm, torch.float32, "y_perm")
    _require(inv, torch.int32, "inv")
    _require(topk_w, torch.float32, "topk_w")
    _require(signs_y, torch.int8, "signs_y")
    T, k = topk_w.shape
    D = y_perm.shape[1]
    if out is None:
        out = torch.empty((T, D), dtype=torch.float32, device=y_perm.device)
    _require(out, torch.float32, "out")
    _check(_fn("route_unpermute_signed")(_p(y_perm), _p(inv), _p(topk_w), T, k, D, _p(signs_y), _p(out),
                                         _stream(stream)), "route_unpermute_signed")
    return out


class DeviceLayer:
    """A trellis-coded MoE layer resident on the GPU, with its C-ABI descriptor.

    Built from per-width groups (K, ascending expert ids, bit streams and fp16 scales);
    `expert_slot[e] = (group << 16) | index` locates expert e.
    """

    def __init__(self, E: int, D: int, F: int, groups: List[dict], device="cuda", signs: Optional[dict] = None,
                 codebook: str = "t16"):
        self.E, self.D, self.F = E, D, F
        self.codebook = codebook
        self.device = torch.device(device)
        self.groups = []
        slot = np.full(E, -1, dtype=np.int32)
        st = TqMoeLayer()
        st.E, st.D, st.F, st.n_groups = E, D, F, len(groups)
        st.codebook = CODEBOOKS[codebook]
        if not 1 <= len(groups) <= 3:
            raise ValueError("1..3 width groups")
        for gi, g in enumerate(groups):
            t = {}
            for key in ("gate", "up", "down"):
                arr = g[key]
                if isinstance(arr, np.ndarray):
                    arr = torch.from_numpy(np.ascontiguousarray(arr).view(np.int32))
                t[key] = arr.to(self.device).contiguous()
            for key in ("s_gate", "s_up", "s_down"):
                arr = g[key]
                if isinstance(arr, np.ndarray):
                    arr = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float16))
                t[key] = arr.to(self.device).contiguous()
            ids = np.asarray(g["ids"], dtype=np.int32)
            t["ids"] = torch.from_numpy(ids).to(self.device)
            t["K"] = int(g["K"])
            slot[ids] = (gi << 16) | np.arange(ids.size, dtype=np.int32)
            w = st.groups[gi]
            w.K, w.n_experts = t["K"], int(ids.size)
            w.expert_ids = t["ids"].data_ptr()
            for key in ("gate", "up", "down", "s_gate", "s_up", "s_down"):
                setattr(w, key, t[key].data_ptr())
            self.groups.append(t)
        self.expert_slot = torch.from_numpy(slot).to(self.device)
        st.expert_slot = self.expert_slot.data_ptr()
        # layer sign vectors of the two-sided transform (int8 +1/-1): x, gu, h, y
        self.signs = None
        if signs is not None:
            self.signs = {key: torch.as_tensor(np.asarray(signs[key], dtype=np.int8)).to(self.device).contiguous()
                          for key in ("x", "gu", "h", "y")}
            st.sign_x, st.sign_gu = self.signs["x"].data_ptr(), self.signs["gu"].data_ptr()
            st.sign_h, st.sign_y = self.signs["h"].data_ptr(), self.signs["y"].data_ptr()
        self.struct = st

    @staticmethod
    def from_synthetic(layer, device="cuda") -> "DeviceLayer":
        groups = [dict(K=g.K, ids=g.ids, gate=g.gate, up=g.up, down=g.down,
                       s_gate=g.s_gate, s_up=g.s_up, s_down=g.s_down) for g in layer.groups]
        return DeviceLayer(layer.E, layer.D, layer.F, groups, device, getattr(layer, "signs", None),
                           getattr(layer, "codebook", "t16"))

    def compressed_bytes(self, experts) -> int:
        """Bit-stream + scale bytes of the given experts (all three projections)."""
        K_of = {}
        for g in self.groups:
            for e in g["ids"].tolist():
                K_of[e] = g["K"]
        n = 0
        for e in experts:
            n += 3 * self.D * self.F * K_of[int(e)] // 8 + 2 * (2 * self.F + self.D)
        return n


def moe_trellis_workspace_size(layer: DeviceLayer, T: int, k: int) -> int:
    return int(_fn("moe_trellis_workspace_size")(ctypes.byref(layer.struct), T, k))


def _moe_call(name, layer: DeviceLayer, x_rot, routing: Routing, T, k, y_perm=None, ws=None,
              stream=None):
    _require(x_rot, torch.float16, "x_rot")
    if y_perm is None:
        y_perm = torch.empty((T * k, layer.D), dtype=torch.float32, device=x_rot.device)
    need = moe_trellis_workspace_size(layer, T, k)
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=x_rot.device)
    _check(_fn(name)(ctypes.byref(layer.struct), _p(x_rot), _p(routing.offsets), _p(routing.perm),
                     _p(routing.active_ids), _p(routing.n_active), T, k, _p(y_perm), _p(ws),
                     ws.numel() * ws.element_size(), _stream(stream)), name)
    return y_perm


def moe_trellis_gemv(layer, x_rot, routing, T, k, y_perm=None, ws=None, stream=None):
    return _moe_call("moe_trellis_gemv", layer, x_rot, routing, T, k, y_perm, ws, stream)


def moe_trellis_gemv_noalloc(layer: DeviceLayer, x_rot: torch.Tensor, routing: Routing, T: int, k: int,
                             y_perm: torch.Tensor, stream=None) -> torch.Tensor:
    """moe_trellis_gemv with the library's own fixed 4 MiB scratch array instead of a
    workspace, for callers that cannot allocate device memory at call time.  y_perm
    ([T*k, D] fp32) must be provided; the call itself allocates nothing.  The call must
    fit the scratch: the GEMV workspace, moe_trellis_gemv's share of
    moe_trellis_workspace_size (include/trellis_moe.h gives the byte formula), at most
    4 MiB -- T <= 25 at k = 8, D = 4096, F = 1024.  Larger calls raise TQError
    (TQ_ERR_WORKSPACE)."""
    _require(x_rot, torch.float16, "x_rot")
    _require(y_perm, torch.float32, "y_perm")
    _check(_fn("moe_trellis_gemv_noalloc")(ctypes.byref(layer.struct), _p(x_rot), _p(routing.offsets),
                                           _p(routing.perm), _p(routing.active_ids),
                                           _p(routing.n_active), T, k, _p(y_perm), _stream(stream)),
           "moe_trellis_gemv_noalloc")
    return y_perm


def moe_trellis_gemm(layer, x_rot, routing, T, k, y_perm=None, ws=None, stream=None):
    return _moe_call("moe_trellis_gemm", layer, x_rot, routing, T, k, y_perm, ws, stream)


class MoeBuffers:
    """Preallocated device buffers of one MoE layer call (T tokens, top-k)."""

    def __init__(self, layer: DeviceLayer, T: int, k: int):
        dev = layer.device
        self.T, self.k = T, k
        self.ids = torch.empty((T, k), dtype=torch.int32, device=dev)
        self.w = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.routing = Routing.empty(T, k, layer.E, dev)
        self.x_rot = torch.empty((T, layer.D), dtype=torch.float16, device=dev)
        self.y_perm = torch.empty((T * k, layer.D), dtype=torch.float32, device=dev)
        self.out = torch.empty((T, layer.D), dtype=torch.float32, device=dev)
        self.ws = torch.empty(max(moe_trellis_workspace_size(layer, T, k), 1), dtype=torch.uint8,
                              device=dev)


GEMM_MIN_TOKENS = 340   # measured crossover of the two paths on the 384-expert decode layer


def moe_layer(layer: DeviceLayer, x: torch.Tensor, logits: torch.Tensor, k: int,
              bufs: Optional[MoeBuffers] = None, path: str = "auto", stream=None) -> torch.Tensor:
    """One MoE layer's routed experts: top-k routing, grouping, input rotation, the
    trellis GEMV (decode-sized T) or GEMM (prefill-sized T), and the combine.
    x: [T, D] bf16/fp16; logits: [T, E] fp32.  Returns out [T, D] fp32."""
    T = x.shape[0]
    bufs = bufs or MoeBuffers(layer, T, k)
    route_topk_permute(logits, k, layer.E, bufs.ids, bufs.w, bufs.routing, stream)
    if layer.signs is not None:
        hadamard128_signed(x, layer.signs["x"], bufs.x_rot, stream)
    else:
        hadamard128(x, bufs.x_rot, stream)
    use_gemm = (path == "gemm" or layer.codebook != "t16"      # the GEMV decodes T16 only
                or (path == "auto" and T >= GEMM_MIN_TOKENS))
    fn = moe_trellis_gemm if use_gemm else moe_trellis_gemv
    fn(layer, bufs.x_rot, bufs.routing, T, k, bufs.y_perm, bufs.ws, stream)
    if layer.signs is not None:
        route_unpermute_signed(bufs.y_perm, bufs.routing.inv, bufs.w, layer.signs["y"], bufs.out, stream)
    else:
        route_unpermute(bufs.y_perm, bufs.routing.inv, bufs.w, bufs.out, stream)
    return bufs.out


class MoeGraph:
    """One MoE layer call captured as a CUDA graph together with its host transfers.

    replay() copies x_host [T, D] (bf16/fp16) and logits_host [T, E] (fp32), both pinned,
    to the device, runs moe_layer (routing, rotation, expert path, combine) and copies the
    result into out_host [T, D] fp32 (pinned), all as one graph launch on `stream`.  The
    same host buffers are read and written on every replay: write the next step's inputs
    into x_host / logits_host, replay, read out_host after synchronising the stream.
    The first calls run eagerly (the library configures its kernels on first use, which
    must happen outside a capture)."""

    def __init__(self, layer: DeviceLayer, x_host: torch.Tensor, logits_host: torch.Tensor, k: int,
                 path: str = "auto", out_host: Optional[torch.Tensor] = None, stream=None, warmup: int = 2):
        for t, name in ((x_host, "x_host"), (logits_host, "logits_host")):
            if t.is_cuda or not t.is_pinned():
                raise ValueError("MoeGraph: %s must be pinned host memory" % name)
        T = x_host.shape[0]
        self.layer, self.k, self.path = layer, k, path
        self.x_host, self.logits_host = x_host, logits_host
        self.out_host = out_host if out_host is not None else \
            torch.empty((T, layer.D), dtype=torch.float32).pin_memory()
        self.x = torch.empty(x_host.shape, dtype=x_host.dtype, device="cuda")
        self.logits = torch.empty(logits_host.shape, dtype=logits_host.dtype, device="cuda")
        self.bufs = MoeBuffers(layer, T, k)
        self.stream = stream if stream is not None else torch.cuda.Stream()
        self.stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(self.stream):
            for _ in range(warmup):
                self._body()
            self.stream.synchronize()
            self.graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.graph, stream=self.stream):
                self._body()

    def _body(self):
        self.x.copy_(self.x_host, non_blocking=True)
        self.logits.copy_(self.logits_host, non_blocking=True)
        out = moe_layer(self.layer, self.x, self.logits, self.k, bufs=self.bufs, path=self.path)
        self.out_host.copy_(out, non_blocking=True)

    def replay(self) -> torch.Tensor:
        """Enqueue one layer call on the graph's stream; returns out_host (valid once the
        stream has been synchronised)."""
        self.graph.replay()
        return self.out_host
