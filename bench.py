"""Benchmark of the trellis-coded MoE routed-expert path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload moe_decode_t16]

A step is one pass of the whole hot path over one batch: route_topk -> route_permute ->
hadamard128 -> moe_trellis_gemv (gate/up+SiLU, rotation of h, down) -> route_unpermute,
for one 384-expert layer (D = 4096, F = 1024, mixed widths 368/15/1 experts at
K = 2/3/4) and 16 tokens with top-8 routing.  Four such layers (independent synthetic
weights and inputs) are cycled so that a weight byte is re-read only after ~1.4 GB of
other weights: every step reads its ~0.35 GB of touched bit streams from HBM, not L2.

Prints one JSON line (rank 0).  With N > 1 (torchrun) every rank runs an independent
replica (the path has no exchange step); value = all ranks' tokens / max-over-ranks time.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "routed-expert tok/s per MoE layer; GEMV HBM GB/s and GEMM tensor-pipe % of peak"
# what each expert path contracts (weights are exact integer codes on both)
DTYPE_LABEL = {
    "gemv": "gemv: activations as 16-bit fixed point (two words for rows with outliers), "
            "u8 x s8 IMMA, int32 sums; gemm: f16 operands, f32 accumulate",
    "gemm": "gemm: f16 operands (decoded codes exact), f32 accumulate in tensor memory",
    "gemm_fp8": "gemm: e4m3 weights (pair-trellis codes exact) and e4m3 activations with power-of-two row "
                "scales, f32 accumulate in tensor memory",
}
N_LAYER_COPIES = 4   # default of --layers
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None,
                   help="timed steps (default: 500 decode, 50 prefill: about 0.15-0.2 s timed)")
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--repeats", type=int, default=5,
                   help="the timed loop of --steps steps runs this many times; the median repeat is reported")
    p.add_argument("--no-prefill", action="store_true",
                   help="skip the prefill-layer (tensor-core GEMM) measurement of the default run")
    p.add_argument("--batch1", action="store_true",
                   help="decode GEMV at 1 and 16 tokens on single-width layers (K = 2, 3, 4), L2 flushed before "
                        "every step; kernel GB/s from the library's events")
    p.add_argument("--gemv-single", action="store_true",
                   help="trellis_gemv on 1024x4096 projections at batch 1 (K = 2, 3, 4), L2 flushed before "
                        "every call")
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="moe_decode_t16",
                   choices=["moe_decode_t16", "moe_prefill_t8192", "moe_prefill_t8192_fp8"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--layers", type=int, default=4,
                   help="synthetic layer copies cycled through (4 keep every step's weights out of L2)")
    p.add_argument("--eager", action="store_true", help="launch every step from the host instead of a CUDA graph")
    p.add_argument("--tokens", type=int, default=None, help="override the workload's token count (profiling runs)")
    p.add_argument("--experts", type=int, default=None, help="override the workload's expert count (profiling runs)")
    p.add_argument("--two-sided", action="store_true",
                   help="layers carry the two-sided transform (Hadamard on both sides, layer signs)")
    p.add_argument("--encode", action="store_true",
                   help="time trellis_encode (T16 tail-biting Viterbi) on 1024x4096 Gaussian targets, K = 2, 3, 4")
    p.add_argument("--sweep", action="store_true",
                   help="batch sweep of the mixed-width decode layer (T = 1 .. 16384, uniform top-8): "
                        "device time of the GEMV and the GEMM path at every T, one JSON line each")
    return p.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def aggregate_ranks(ms_local, tokens_per_rank, world, device=None):
    """Whole-job throughput of independent replicas: every rank's timed milliseconds are
    reduced with MAX over ranks (the job ends when its slowest replica ends) and the
    tokens of all ranks are divided by that time.  Returns (ms_max, tokens_per_s)."""
    ms_max = float(ms_local)
    if world > 1:
        import torch
        import torch.distributed as dist
        t = torch.tensor([ms_local], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_max = float(t.item())
    return ms_max, tokens_per_rank * world / (ms_max * 1e-3)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def csrc_digest(files=None):
    """Digest of the kernel sources a profile was taken on (all of csrc/ by default)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "trellis_quantized_moe_gemv_b200", "csrc")
    for f in sorted(files or os.listdir(d)):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def profile_traffic(name):
    """DRAM bytes per launch recorded by an ncu capture (profiles/<name>.txt), or None
    when missing or taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", name + ".txt")
    if not os.path.exists(path):
        return None
    kv = {}
    with open(path) as f:
        for line in f:
            if "=" in line and not line.lstrip().startswith("#"):
                k, v = line.split("=", 1)
                kv[k.strip()] = v.strip()
    files = kv.get("csrc_files", "").split() or None
    if kv.get("csrc_digest") != csrc_digest(files) or "dram_bytes_per_unit" not in kv:
        return None
    return kv


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every 2 ms."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index):
        self.samples = []
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.time(), mhz, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self, windows):
        """Median SM clock and the clock-event reasons seen in the timed windows
        [(t0, t1), ...] (the repeats of the timed loop)."""
        if not self.ok:
            return None
        inside = [s for s in self.samples if any(t0 <= s[0] <= t1 for t0, t1 in windows)]
        window = "timed (%d repeats)" % len(windows)
        if not inside:
            t0, t1 = windows[0][0], windows[-1][1]
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
            window = "nearest to the timed region (region shorter than the sampling period)"
        if not inside:
            return None
        reasons = set()
        for _, _, rs in inside:
            for bit, name in self.REASONS.items():
                if rs & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(inside), "window": window}


# ----------------------------------------------------------------------------- workload

def build_decode_workload(api, inputs, torch, device, rank, n_copies, two_sided=False, T=16):
    """Layer copy 0 from the seeded numpy generators (the copy the parity tests check);
    copies 1..3 with the same widths, their bit streams and scales drawn on the device
    from a seeded torch generator; every copy has its own tokens and logits (T tokens:
    16, or another count for profiling runs)."""
    w0 = inputs.moe_decode_t16(seed=1003 + 100 * rank, T=T)
    host_layer = w0["layer"]
    layers, xs, logits = [], [], []
    if two_sided:
        inputs.with_signs(host_layer, 8000 + 100 * rank)
    layers.append(api.DeviceLayer.from_synthetic(host_layer, device))
    gen = torch.Generator(device=device)
    for c in range(1, n_copies):
        gen.manual_seed(7000 + 100 * rank + c)
        groups = []
        for g in host_layer.groups:
            def rbits(shape):
                return torch.randint(-2 ** 31, 2 ** 31 - 1, shape, dtype=torch.int32, device=device,
                                     generator=gen)

            def rscale(shape):
                return (torch.rand(shape, device=device, generator=gen) + 0.5).to(torch.float16)
            groups.append(dict(K=g.K, ids=g.ids, gate=rbits(g.gate.shape), up=rbits(g.up.shape),
                               down=rbits(g.down.shape), s_gate=rscale(g.s_gate.shape),
                               s_up=rscale(g.s_up.shape), s_down=rscale(g.s_down.shape)))
        signs = None
        if two_sided:
            srng = np.random.default_rng(8000 + 100 * rank + c)
            signs = {key: inputs.random_signs(srng, n) for key, n in
                     (("x", host_layer.D), ("gu", host_layer.F), ("h", host_layer.F), ("y", host_layer.D))}
        layers.append(api.DeviceLayer(host_layer.E, host_layer.D, host_layer.F, groups, device, signs))
    for c in range(n_copies):
        rng = np.random.default_rng(9000 + 100 * rank + c)
        x = w0["x"] if c == 0 else inputs.random_activations(rng, (T, host_layer.D), "bf16")
        lg = w0["logits"] if c == 0 else inputs.normal_logits(rng, T, host_layer.E)
        xs.append((x, lg))
    return w0, layers, xs


def gemv_algorithmic_bytes(layer, counts):
    """Algorithmic bytes of one fused GEMV launch (gate/up, SwiGLU and down of every
    active expert): per expert with n routes, its gate, up and down bit streams (K/8 B per
    weight) and scales, its routes' rotated activations read (2 B per value), g and u
    written and read back (fp32), h' written and read (2 B per value) and y written
    (fp32)."""
    K_of = {}
    for g in layer.groups:
        for e in g["ids"].tolist():
            K_of[e] = g["K"]
    total = 0
    D, F = layer.D, layer.F
    for e, n in enumerate(counts):
        n = int(n)
        if n == 0:
            continue
        total += 3 * F * D * K_of[e] // 8 + (2 * F + D) * 2
        total += n * (D * 2 + 2 * F * 4 * 2 + F * 2 * 2 + D * 4)
    return total


def build_prefill_workload(api, inputs, device, rank, T=8192, E=384, two_sided=False, fp8=False):
    """The all-K=3 384-expert layer with 8192 Zipf(1.1)-routed tokens: one step touches
    every expert (1.8 GB of bit streams), far beyond L2, so one layer copy suffices.
    fp8: the same shape with pair-trellis (E4M3) streams."""
    if fp8:
        w0 = inputs.moe_prefill_t8192_fp8(seed=1006 + 100 * rank, T=T, E=E)
    else:
        w0 = inputs.moe_prefill_t8192(seed=1004 + 100 * rank, T=T, E=E)
    if two_sided:
        inputs.with_signs(w0["layer"], 8000 + 100 * rank)
    layers = [api.DeviceLayer.from_synthetic(w0["layer"], device)]
    return w0, layers, [(w0["x"], w0["logits"])]


def gateup_flops(layer, T, k):
    """Algorithmic FLOPs of one gate/up launch: 2 per weight per routed token, for the
    gate and up projections of every route."""
    return 2.0 * T * k * 2 * layer.F * layer.D


WORKLOADS = {
    "moe_decode_t16": dict(T=16, path="gemv", stage="moe_gemv",
                           kernel="moe_gemv_fused_kernel<1> (gate/up, SwiGLU and down GEMVs in one persistent launch, "
                                  "int8 tensor cores, 4 routes per pass)",
                           widths="368/15/1 experts at K=2/3/4", routing="top-8 of N(0,1) logits"),
    "moe_prefill_t8192": dict(T=8192, path="gemm", stage="gemm_gateup",
                              kernel="moe_gemm_kernel<1> (gate/up tcgen05 GEMM + SiLU)",
                              widths="all 384 experts at K=3",
                              routing="top-8 of log p + Gumbel, p ~ rank^-1.1 (Zipf)"),
    "moe_prefill_t8192_fp8": dict(T=8192, path="gemm", stage="gemm_gateup",
                                  kernel="moe_gemm_kernel<1, fp8> (gate/up tcgen05 kind::f8f6f4 GEMM + SiLU, "
                                         "pair-trellis E4M3 weights and activations)",
                                  widths="all 384 experts at K=3, pair-trellis (E4M3) codebook",
                                  routing="top-8 of log p + Gumbel, p ~ rank^-1.1 (Zipf)"),
}


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from trellis_quantized_moe_gemv_b200 import api, inputs
    from trellis_quantized_moe_gemv_b200 import build as tqbuild

    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if rank == 0:
        tqbuild.build()
    if world > 1:
        dist.barrier()
    api.lib()

    wl = WORKLOADS[args.workload]
    T, k = (args.tokens or wl["T"]), 8
    if args.workload == "moe_decode_t16":
        if args.experts:
            raise SystemExit("--experts applies to the prefill workload")
        NL = args.layers
        w0, layers, xs = build_decode_workload(api, inputs, torch, device, rank, NL, args.two_sided, T=T)
    else:
        NL = 1
        w0, layers, xs = build_prefill_workload(api, inputs, device, rank, T=T, E=args.experts or 384,
                                                two_sided=args.two_sided, fp8=args.workload.endswith("fp8"))
    E, D, F = layers[0].E, layers[0].D, layers[0].F
    bufs = [api.MoeBuffers(L, T, k) for L in layers]
    x_dev = [torch.from_numpy(x).to(torch.bfloat16).to(device) for x, _ in xs]
    l_dev = [torch.from_numpy(lg).to(device) for _, lg in xs]
    stream = torch.cuda.current_stream()

    def eager_step(i):
        c = i % NL
        api.moe_layer(layers[c], x_dev[c], l_dev[c], k, bufs=bufs[c], path=wl["path"])

    for i in range(args.warmup):
        eager_step(i)
    torch.cuda.synchronize()
    api.device_status(clear=True)

    # One CUDA graph per layer copy.  The library's profiling events are captured with
    # the kernels (every replay re-records them); the timed graphs carry the events of
    # the dominant kernel only, a second set of graphs, replayed after the timed region,
    # those of every stage.
    api.profile_enable(64 * NL)
    # the GEMV's stages: the fused launch, or (fewer than 32 routes) gate/up, h', down
    timed_stages = ["moe_gemv", "rotate_h", "gemv_down"] if wl["path"] == "gemv" else [wl["stage"]]
    api.profile_stages(timed_stages)
    api.profile_collect()
    launches0 = api.launch_count()

    def capture_graphs():
        out = []
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for c in range(NL):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=side):
                    eager_step(c)
                out.append(g)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        return out

    graphs = []
    if not args.eager:
        graphs = capture_graphs()
        launches_per_step = (api.launch_count() - launches0) // NL
        for i in range(args.warmup):
            graphs[i % NL].replay()
        torch.cuda.synchronize()

    def step(i):
        if args.eager:
            eager_step(i)
        else:
            graphs[i % NL].replay()

    # ---- device-timed region: R repeats of K steps, each bracketed by a barrier and a
    # synchronize on both sides; the median repeat is the result
    sampler = ClockSampler(local_rank)
    sampler.start()
    launches0 = api.launch_count()
    windows, rep_ms = [], []
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    for r in range(args.repeats):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t_wall0 = time.time()
        ev0.record(stream)
        for i in range(args.steps):
            step(i)
        ev1.record(stream)
        torch.cuda.synchronize()
        windows.append((t_wall0, time.time()))
        if world > 1:
            dist.barrier()
        rep_ms.append(ev0.elapsed_time(ev1))
    launches = (api.launch_count() - launches0) // args.repeats if args.eager else launches_per_step * args.steps
    stages = api.profile_collect()
    sampler.stop()
    # per-stage breakdown, outside the timed region
    api.profile_stages(None)
    if args.eager:
        for i in range(NL):
            eager_step(i)
    else:
        for g in capture_graphs():
            g.replay()
    torch.cuda.synchronize()
    stage_breakdown = api.profile_collect()
    api.profile_disable()
    ms_total = statistics.median(rep_ms)
    flags = api.device_status()
    if flags:
        raise RuntimeError("device anomaly flags %d during the timed region" % flags)

    ms_max, value = aggregate_ranks(ms_total, T * args.steps, world, device)

    # ---- the dominant kernel (gate/up) per launch: algorithmic bytes (decode GEMV,
    # HBM-bound) or FLOPs (prefill GEMM, tensor-bound) over its average duration; the
    # stage totals cover the last replay of each layer copy's graph (eager: every step)
    counts = [b.routing.counts.cpu().numpy() for b in bufs]
    split_gemv = wl["path"] == "gemv" and stages.get("gemv_down", (0.0, 0))[1] > 0
    g_n = stages[wl["stage"]][1]
    g_ms = sum(stages[n_][0] for n_ in timed_stages if n_ in stages) if split_gemv else stages[wl["stage"]][0]
    g_avg_ms = g_ms / max(g_n, 1)
    kernel_label = ("moe_gemv_items_kernel x 2 + quantize_rows_kernel (the split form below 32 routes)"
                    if split_gemv else wl["kernel"])
    stage_avg = {k_: v[0] / v[1] for k_, v in stage_breakdown.items() if v[1]}
    peaks, peak_src = load_peaks()
    if wl["path"] == "gemv":
        per_copy_bytes = [gemv_algorithmic_bytes(L, c) for L, c in zip(layers, counts)]
        if args.eager:
            unit_work = sum(per_copy_bytes[i % NL] for i in range(args.steps)) / max(args.steps, 1)
        else:
            unit_work = sum(per_copy_bytes) / NL
        achieved = unit_work / (g_avg_ms * 1e-3) / 1e9
        peak = float(peaks["hbm_gbs"])
        prof = profile_traffic("moe_gemv_fused_decode_t16")
        traffic = None
        if prof is not None:
            units = sum(int((c > 0).sum()) for c in counts) / NL
            traffic = float(prof["dram_bytes_per_unit"]) * units
        roofline = {"kernel": kernel_label, "bound": "hbm", "achieved": achieved, "peak": peak,
                    "unit": "GB/s", "frac": achieved / peak, "peak_source": peak_src + " (copy bandwidth)",
                    "bytes_per_launch": unit_work, "avg_launch_ms": g_avg_ms, "traffic": traffic}
    else:
        unit_work = gateup_flops(layers[0], T, k)
        E = layers[0].E
        achieved = unit_work / (g_avg_ms * 1e-3) / 1e12
        peak = float(peaks["bf16_tflops"])     # burst: the timed region is sub-second
        fp8 = args.workload.endswith("fp8")
        if fp8:
            peak *= 2.0                        # E4M3 dense rate: twice bf16 (4.5 vs 2.25 PF nominal)
        prof = profile_traffic("moe_gemm_gateup_prefill_t8192_fp8" if fp8 else "moe_gemm_gateup_prefill_t8192")
        traffic = None
        if prof is not None:
            traffic = float(prof["dram_bytes_per_unit"]) * float(prof.get("units", 1))
        roofline = {"kernel": wl["kernel"], "bound": "tensor", "achieved": achieved, "peak": peak,
                    "unit": "TFLOP/s", "frac": achieved / peak,
                    "peak_source": peak_src + (" (dense bf16 GEMM burst x 2, the nominal E4M3 / bf16 ratio)"
                                               if fp8 else " (dense bf16 GEMM, burst: the timed region is "
                                                           "sub-second; fp16 dense rate is the same)"),
                    "flops_per_launch": unit_work, "avg_launch_ms": g_avg_ms, "traffic": traffic}

    # ---- end to end through the public API with host buffers: api.MoeGraph, one per
    # layer copy, replays the pinned-host -> device copies of x and the logits, the layer
    # and the device -> pinned-host copy of the output as one graph launch
    pin_x = [torch.from_numpy(x).to(torch.bfloat16).pin_memory() for x, _ in xs]
    pin_l = [torch.from_numpy(lg).pin_memory() for _, lg in xs]
    pin_out = torch.empty((T, D), dtype=torch.float32).pin_memory()
    e2e_graphs = [api.MoeGraph(layers[c], pin_x[c], pin_l[c], k, path=wl["path"], out_host=pin_out)
                  for c in range(NL)]
    torch.cuda.synchronize()

    def e2e_step(i):
        e2e_graphs[i % NL].replay()

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_rep = []
    for r in range(args.repeats):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(args.steps):
            e2e_step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_rep.append(e0.elapsed_time(e1))
    e2e_ms, e2e_value = aggregate_ranks(statistics.median(e2e_rep), T * args.steps, world, device)
    h2d = T * D * 2 + T * E * 4
    d2h = T * D * 4

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w0, routes=16, name=args.workload)

    prefill = None
    if args.workload == "moe_decode_t16" and not args.no_prefill and not args.two_sided:
        del graphs, e2e_graphs
        prefill = measure_prefill(args, api, inputs, torch, device, rank, world, stream)

    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tok/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": DTYPE_LABEL["gemm_fp8" if args.workload.endswith("fp8") else wl["path"]],
        "data": "synthetic",
        "config": {
            "workload": args.workload, "experts": E, "hidden": D, "intermediate": F,
            "tokens": T, "top_k": k, "widths": wl["widths"], "routing": wl["routing"],
            "layer_copies_cycled": NL,
            "l2": ("inputs larger than L2: each step reads ~0.35 GB of bit streams; %d layers "
                   "(%.1f GB) cycled" % (NL, 1.23 * NL)) if wl["path"] == "gemv" else
                  "inputs larger than L2: each step reads all 1.8 GB of bit streams",
            "codebook": "pair_e4m3" if args.workload.endswith("fp8") else "t16",
            "path": wl["path"], "launch": "eager" if args.eager else "cuda-graph replay per step",
            "parallelism": "replicas" if world > 1 else "single-gpu",
            "transform": "two-sided (Hadamard on both sides, layer signs)" if args.two_sided
                         else "input-side Hadamard",
        },
        "roofline": roofline,
        "stage_avg_launch_ms": stage_avg,
        "gpu_launches": launches,
        "e2e": {"value": e2e_value, "unit": "tok/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "clocks": sampler.summary(windows),
        "cpu_baseline": cpu,
        "prefill": prefill,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def measure_prefill(args, api, inputs, torch, device, rank, world, stream, steps=20):
    """The prefill layer (384 experts all K = 3, 8192 Zipf-routed tokens, top-8) through the
    tcgen05 GEMM path: R repeats of `steps` CUDA-graph replays (each reads all 1.8 GB of bit
    streams, beyond L2), median repeat; the gate/up GEMM's average launch time from the
    library's events in the timed graph; tensor roofline against the burst bf16 peak (the
    timed region is well under a second)."""
    import torch.distributed as dist
    T, k = 8192, 8
    w0, layers, xs = build_prefill_workload(api, inputs, device, rank, T=T)
    L = layers[0]
    bufs = api.MoeBuffers(L, T, k)
    x = torch.from_numpy(xs[0][0]).to(torch.bfloat16).to(device)
    lg = torch.from_numpy(xs[0][1]).to(device)
    for _ in range(args.warmup):
        api.moe_layer(L, x, lg, k, bufs=bufs, path="gemm")
    torch.cuda.synchronize()
    api.profile_enable(64)
    api.profile_stages(["gemm_gateup", "gemm_down"])
    api.profile_collect()      # the graph's event nodes are re-recorded at every replay
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            api.moe_layer(L, x, lg, k, bufs=bufs, path="gemm")
    stream.wait_stream(side)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    rep_ms, windows = [], []
    for r in range(args.repeats):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = time.time()
        e0.record(stream)
        for i in range(steps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        windows.append((t0, time.time()))
        rep_ms.append(e0.elapsed_time(e1))
    sampler.stop()
    st = api.profile_collect()
    api.profile_disable()
    if api.device_status():
        raise RuntimeError("device anomaly flags during the prefill measurement")
    ms_max, tok_s = aggregate_ranks(statistics.median(rep_ms), T * steps, world, device)
    gu_ms = st["gemm_gateup"][0] / max(st["gemm_gateup"][1], 1)
    dn_ms = st["gemm_down"][0] / max(st["gemm_down"][1], 1)
    peaks, src = load_peaks()
    flops = gateup_flops(L, T, k)
    achieved = flops / (gu_ms * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    prof = profile_traffic("moe_gemm_gateup_prefill_t8192")
    del g
    return {
        "workload": "moe_prefill_t8192", "tokens": T, "steps": steps, "repeats": args.repeats,
        "ms_per_step": ms_max / steps, "value": tok_s, "unit": "tok/s", "dtype": DTYPE_LABEL["gemm"],
        "roofline": {"kernel": WORKLOADS["moe_prefill_t8192"]["kernel"], "bound": "tensor", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": src + " (dense bf16 GEMM, burst: the region is sub-second; fp16 dense "
                                          "rate is the same)",
                     "flops_per_launch": flops, "avg_launch_ms": gu_ms,
                     "traffic": (float(prof["dram_bytes_per_unit"]) * float(prof.get("units", 1)))
                     if prof is not None else None},
        "down_avg_launch_ms": dn_ms,
        "clocks": sampler.summary(windows),
    }


def cpu_baseline(w0, routes, name="moe_decode_t16"):
    """The fp64 CPU oracle, as it stands, on `routes` (token, expert) routes of layer
    copy 0 (single-threaded BLAS); reported in tok/s (k routes = one token)."""
    from oracle import layer as OL
    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(limits=1)
    except Exception:
        limiter = None
    layer, x, logits, k = w0["layer"], w0["x"], w0["logits"], w0["k"]
    ids, wts = OL.route_topk(logits, k)
    weights = OL.ExpertWeights(layer)
    t0 = time.time()
    done = 0
    for t in range(x.shape[0]):
        xr = OL.rotate(x[t:t + 1].astype(np.float64))
        for s in range(k):
            OL.expert_forward(weights, int(ids[t, s]), xr)
            done += 1
            if done >= routes:
                break
        if done >= routes:
            break
    dt = time.time() - t0
    if limiter is not None:
        limiter.unregister()
    return {"value": (done / k) / dt, "unit": "tok/s", "cores": 1, "kind": "oracle",
            "sample": "%d routes (= %d tokens x top-%d) of the %s layer, fp64 "
                      "scalar-C decode + numpy, %.1f s" % (done, done // k, k, name, dt)}


def run_reference(args, rank, world):
    """The oracle as the reference arm: each step is one (token, expert) route of the
    decode layer, decoded and computed in fp64 on the host; value in tok/s."""
    if rank != 0:
        return
    from oracle import layer as OL
    from trellis_quantized_moe_gemv_b200 import inputs
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=1)
    except Exception:
        pass
    w0 = inputs.moe_decode_t16() if args.workload == "moe_decode_t16" else inputs.moe_prefill_t8192()
    layer, x, logits, k = w0["layer"], w0["x"], w0["logits"], w0["k"]
    n_tok = min(x.shape[0], 64)
    ids, _ = OL.route_topk(logits[:n_tok], k)
    routes = [(t, s) for t in range(n_tok) for s in range(k)]

    def step(i):
        t, s = routes[i % len(routes)]
        weights = OL.ExpertWeights(layer)   # no decode reuse across steps
        OL.expert_forward(weights, int(ids[t, s]), OL.rotate(x[t:t + 1].astype(np.float64)))

    for i in range(args.warmup):
        step(i)
    t0 = time.time()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.time() - t0
    value = (args.steps / k) / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "experts": 384, "hidden": 4096,
                   "intermediate": 1024, "tokens": x.shape[0], "top_k": k,
                   "widths": WORKLOADS[args.workload]["widths"],
                   "routing": WORKLOADS[args.workload]["routing"]},
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": 1, "kind": "oracle",
                         "sample": "one (token, expert) route per step = 1/%d token" % k},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def device_layer(api, torch, device, K, seed, E=384, D=4096, F=1024):
    """A single-width layer (every expert at K bits per weight) with bit streams and
    U[0.5, 1.5] scales drawn on the device from a seeded generator."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)

    def rbits(n, rows, cols):
        return torch.randint(-2 ** 31, 2 ** 31 - 1, (n, (rows // 16) * (cols // 16) * 8 * K), dtype=torch.int32,
                             device=device, generator=gen)

    def rscale(shape):
        return (torch.rand(shape, device=device, generator=gen) + 0.5).to(torch.float16)
    g = dict(K=K, ids=np.arange(E, dtype=np.int32), gate=rbits(E, F, D), up=rbits(E, F, D), down=rbits(E, D, F),
             s_gate=rscale((E, F)), s_up=rscale((E, F)), s_down=rscale((E, D)))
    return api.DeviceLayer(E, D, F, [g], device)


def run_batch1(args, local_rank):
    """The decode GEMV at 1 and 16 tokens on single-width 384-expert layers (K = 2, 3, 4),
    top-8 of N(0,1) logits, a fresh token every step, L2 evicted (a 512 MB write) before
    every step.  The library's events give each GEMV launch's device time; the gate/up
    kernel's HBM rate is its algorithmic bytes (the touched experts' gate and up bit
    streams and scales, activations in, results out) over that time.  One JSON line per
    (K, tokens)."""
    import torch
    from trellis_quantized_moe_gemv_b200 import api, inputs
    from trellis_quantized_moe_gemv_b200 import build as tqbuild
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    tqbuild.build()
    api.lib()
    E, D, F, k = 384, 4096, 1024, 8
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    peaks, src = load_peaks()
    steps = max(args.steps, 8)
    for K in (2, 3, 4):
        L = device_layer(api, torch, device, K, 4000 + K)
        for T in (1, 16):
            rng = np.random.default_rng(4100 + 10 * K + T)
            bufs = api.MoeBuffers(L, T, k)
            data = [(torch.from_numpy(inputs.random_activations(rng, (T, D), "bf16")).to(torch.bfloat16).to(device),
                     torch.from_numpy(inputs.normal_logits(rng, T, E)).to(device)) for _ in range(16)]
            for i in range(args.warmup):
                api.moe_layer(L, data[i % 16][0], data[i % 16][1], k, bufs=bufs, path="gemv")
            torch.cuda.synchronize()
            api.profile_enable(64 * steps)
            api.profile_collect()
            gv_bytes = 0
            for i in range(steps):
                flush.zero_()
                api.moe_layer(L, data[i % 16][0], data[i % 16][1], k, bufs=bufs, path="gemv")
                counts = bufs.routing.counts.cpu().numpy()
                gv_bytes += gemv_algorithmic_bytes(L, counts)
            torch.cuda.synchronize()
            st = api.profile_collect()
            api.profile_disable()
            if api.device_status():
                raise RuntimeError("device anomaly flags during the batch-1 measurement")
            # the routed-expert GEMV: one fused launch, or (small batches) gate/up items, the
            # h' quantisation and down items
            split = st.get("gemv_down", (0.0, 0))[1] > 0
            gv_stages = ("moe_gemv", "rotate_h", "gemv_down") if split else ("moe_gemv",)
            gv_ms = sum(st[n][0] for n in gv_stages if n in st) / steps
            step_ms = sum(v[0] for v in st.values()) / steps
            hbm = float(peaks["hbm_gbs"])
            gv_gbs = gv_bytes / steps / (gv_ms * 1e-3) / 1e9
            print(json.dumps({
                "metric": "decode GEMV HBM GB/s on compressed bytes", "workload": "moe_gemv_single_width_K%d_t%d" % (K, T),
                "K": K, "tokens": T, "top_k": k, "steps": steps, "l2": "512 MB written before every step",
                "gemv": {"kernel": ("moe_gemv_items_kernel (gate/up) + quantize_rows_kernel (h') + moe_gemv_items_kernel "
                                    "(down)" if split else "moe_gemv_fused_kernel (gate/up, SwiGLU, down)"),
                         "avg_launch_ms": gv_ms,
                         "bytes_per_launch": gv_bytes / steps, "achieved_gbs": gv_gbs, "frac": gv_gbs / hbm},
                "layer_device_ms": step_ms, "layer_tok_s": T / (step_ms * 1e-3),
                "peak": hbm, "peak_source": src + " (copy bandwidth)"}), flush=True)
            del bufs, data
        del L
        torch.cuda.empty_cache()


def run_gemv_single(args, local_rank):
    """trellis_gemv on one 1024x4096 projection at batch 1 (K = 2, 3, 4): 16 projections
    drawn on the device, L2 evicted before every call, each call's device time (row
    quantisation, the GEMV and its finishing kernel) from the library's events.  A 1-2 MB
    projection is a few microseconds of HBM time, so this measures launch latency as much
    as bandwidth."""
    import torch
    from trellis_quantized_moe_gemv_b200 import api, inputs
    from trellis_quantized_moe_gemv_b200 import build as tqbuild
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    tqbuild.build()
    api.lib()
    rows, cols = 1024, 4096
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    peaks, src = load_peaks()
    steps = max(args.steps, 8)
    for K in (2, 3, 4):
        gen = torch.Generator(device=device)
        gen.manual_seed(4200 + K)
        mats = [torch.randint(-2 ** 31, 2 ** 31 - 1, ((rows // 16) * (cols // 16) * 8 * K,), dtype=torch.int32,
                              device=device, generator=gen) for _ in range(16)]
        scales = (torch.rand(rows, device=device, generator=gen) + 0.5).to(torch.float16)
        x = torch.randn((1, cols), device=device, generator=gen).to(torch.float16)
        y = torch.empty((1, rows), dtype=torch.float32, device=device)
        ws = torch.empty(api.trellis_gemv_workspace_size(rows, cols, 1), dtype=torch.uint8, device=device)
        for i in range(args.warmup):
            api.trellis_gemv(mats[i % 16], scales, K, rows, cols, x, y, ws)
        torch.cuda.synchronize()
        api.profile_enable(16 * steps)
        api.profile_collect()
        for i in range(steps):
            flush.zero_()
            api.trellis_gemv(mats[i % 16], scales, K, rows, cols, x, y, ws)
        torch.cuda.synchronize()
        st = api.profile_collect()
        api.profile_disable()
        call_ms = (st["trellis_gemv"][0] + st["gemv_quant"][0]) / steps
        gemv_ms = st["trellis_gemv"][0] / steps
        nbytes = rows * cols * K // 8 + rows * 2 + cols * 2 + rows * 4
        gbs = nbytes / (gemv_ms * 1e-3) / 1e9
        print(json.dumps({
            "metric": "single-projection GEMV HBM GB/s on compressed bytes", "workload": "proj_1024x4096_K%d_b1" % K,
            "K": K, "batch": 1, "steps": steps, "l2": "512 MB written before every call",
            "bytes_per_call": nbytes, "gemv_ms": gemv_ms, "call_device_ms": call_ms, "achieved_gbs": gbs,
            "frac": gbs / float(peaks["hbm_gbs"]), "peak_source": src + " (copy bandwidth)",
            "note": "gemv_ms covers the GEMV and its finishing kernel (two launches)"}), flush=True)


SWEEP_T = (1, 8, 64, 256, 384, 512, 1024, 2048, 16384)   # the configured sizes plus three near the crossover


def run_sweep(args, local_rank):
    """Both expert paths on the mixed-width 384-expert layer at every sweep size: CUDA-graph
    replays of the whole layer (routing to combine) cycled over 4 layer copies (4.9 GB of
    bit streams, beyond L2), timed with CUDA events after warm-up."""
    import torch
    from trellis_quantized_moe_gemv_b200 import api, inputs
    from trellis_quantized_moe_gemv_b200 import build as tqbuild
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    tqbuild.build()
    api.lib()
    # 12 layer copies: at 1 token a step touches ~26 MB of bit streams, so 4 copies would
    # stay in the 126 MB L2; from 8 tokens on, 4 copies are cycled
    w0, all_layers, _ = build_decode_workload(api, inputs, torch, device, 0, 12)
    host_layer, k = w0["layer"], 8
    stream = torch.cuda.current_stream()
    results = []
    for T in SWEEP_T:
        w = inputs.moe_sweep_tokens(T, layer=host_layer)
        x = torch.from_numpy(w["x"]).to(torch.bfloat16).to(device)
        lg = torch.from_numpy(w["logits"]).to(device)
        layers = all_layers if T == 1 else all_layers[:4]
        NC = len(layers)
        row = {"sweep": "moe_sweep_tokens", "tokens": T, "top_k": k, "routing": "top-8 of N(0,1) logits",
               "layer_copies_cycled": NC}
        for path in ("gemv", "gemm"):
            bufs = [api.MoeBuffers(L, T, k) for L in layers]
            for c, L in enumerate(layers):
                api.moe_layer(L, x, lg, k, bufs=bufs[c], path=path)
            torch.cuda.synchronize()
            graphs = []
            side = torch.cuda.Stream()
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                for c, L in enumerate(layers):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=side):
                        api.moe_layer(L, x, lg, k, bufs=bufs[c], path=path)
                    graphs.append(g)
            stream.wait_stream(side)
            for i in range(8):
                graphs[i % NC].replay()
            torch.cuda.synchronize()
            steps = max(8, min(400, int(4e5 / max(T, 1))))
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for i in range(steps):
                graphs[i % NC].replay()
            e1.record(stream)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / steps
            row[path + "_ms"] = ms
            row[path + "_tok_s"] = T / (ms * 1e-3)
            del graphs, bufs
            torch.cuda.empty_cache()
        row["faster"] = "gemv" if row["gemv_ms"] <= row["gemm_ms"] else "gemm"
        results.append(row)
        print(json.dumps(row), flush=True)
    cross = next((r["tokens"] for r in results if r["faster"] == "gemm"), None)
    print(json.dumps({"sweep": "moe_sweep_tokens", "gemm_faster_from_tokens": cross,
                      "library_switch_tokens": api.GEMM_MIN_TOKENS}), flush=True)


def run_encode(args, local_rank):
    """trellis_encode on a 1024x4096 target of N(0, 100^2) code units per width: device time
    (CUDA events, after a warm-up call), normalised squared error of the decoded codes
    against the Gaussian rate-distortion bound 2^(-2K), the least-squares gain that maps
    the codes back onto the targets, and the oracle's time for one tile on the host."""
    import torch
    import numpy as np
    from trellis_quantized_moe_gemv_b200 import api
    from trellis_quantized_moe_gemv_b200 import build as tqbuild
    torch.cuda.set_device(local_rank)
    tqbuild.build()
    api.lib()
    rows, cols, sigma = 1024, 4096, 100.0
    for K in (2, 3, 4):
        g = torch.Generator(device="cuda")
        g.manual_seed(2000 + K)
        x = torch.randn((rows, cols), generator=g, device="cuda") * sigma
        ws = torch.empty(api._fn("trellis_encode_workspace_size")(K, rows, cols), dtype=torch.uint8, device="cuda")
        for _ in range(args.warmup):
            api.trellis_encode(x[:64], K, ws=ws)
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        bits, cost = api.trellis_encode(x, K, ws=ws)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        codes = api.trellis_decode(bits, K, rows, cols).float()
        nmse = ((x - codes) ** 2).mean().item() / sigma ** 2
        gain = ((x * codes).sum() / (codes * codes).sum()).item()
        tile = x[:16, :16].cpu().numpy()
        from oracle import encode as OE
        OE.code_table()
        t0 = time.time()
        OE.encode_tile(tile, K)
        cpu_s = time.time() - t0
        print(json.dumps({
            "metric": "trellis_encode weights/s", "value": rows * cols / (ms * 1e-3), "unit": "weights/s",
            "n_gpus": 1, "ms": ms, "higher_is_better": True, "dtype": "int32", "data": "synthetic",
            "config": {"workload": "encode_gaussian_%dx%d_K%d" % (rows, cols, K), "K": K,
                       "targets": "N(0, %g^2) code units" % sigma, "tiles": rows * cols // 256},
            "nmse": nmse, "rate_distortion_bound": 2.0 ** (-2 * K), "gain": gain,
            "cpu_baseline": {"value": 256 / cpu_s, "unit": "weights/s", "cores": 1, "kind": "oracle",
                             "sample": "one 16x16 tile"}}), flush=True)


def main():
    args = parse_args()
    rank, world, local_rank = dist_env()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.steps is None:
        if args.impl == "reference":
            args.steps = 16
        else:
            args.steps = 500 if args.workload == "moe_decode_t16" else 50
    if args.encode:
        if rank == 0:
            run_encode(args, local_rank)
    elif args.batch1:
        if rank == 0:
            run_batch1(args, local_rank)
    elif args.gemv_single:
        if rank == 0:
            run_gemv_single(args, local_rank)
    elif args.sweep:
        if rank == 0:
            run_sweep(args, local_rank)
    elif args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
