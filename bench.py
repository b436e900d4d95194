#!/usr/bin/env python
"""Benchmark of the MXFP8 MoE expert-layer hot path on B200.

One step = one pass of the whole path over one synthetic routed batch of the
DeepSeek-V3-671B-like MoE layer (one GPU's share: 32 local experts, 16384
routed rows with Zipf(1.1)-skewed counts; gate/up N = 4096, K = 7168; down
N = 7168, K = 2048): for each of the two grouped linears, rowwise + colwise
MXFP8 quantisation of X, W and dY (one fused dual-layout kernel per tensor
by default; --quantiser separate runs the rowwise and colwise kernels),
then the forward, dgrad and wgrad grouped GEMMs.  The metric is algorithmic
GEMM TFLOP/s (3 passes x 2*M*N*K per linear over real tokens) per step.

The same JSON line also carries ``per_config``: every grouped GEMM pass of
the three MoE workloads (DeepSeek-V3-16B-like, DeepSeek-V3-671B-like,
Llama-4-Scout-like), each launch timed alone with L2 flushed before it, and
the dual quantiser on their X, W and dY.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

N > 1 (launched by torchrun): every rank runs its own copy of the layer on its
own GPU (experts are independent; no data-path collective), torch.distributed
is used only for the barrier and the max over ranks of the timings.
``--impl reference`` times the CPU oracle (bf16 inputs, fp32 accumulation)
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mxfp8_grouped_gemm_quantize_b200 import workloads as wl  # noqa: E402

METRIC = "MoE grouped-GEMM MXFP8 TFLOP/s (fwd+dgrad+wgrad) and % of B200 FP8 peak"
UNIT = "TFLOP/s"
WORKLOAD = "ds-v3-671b"
FP8_OVER_BF16 = 2.0   # nominal dense FP8 / BF16 tensor ratio (4.5 / 2.25 PFLOP/s)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quantiser", default="dual", choices=["dual", "separate"],
                    help="dual: one fused kernel writes both layouts of X, W and dY")
    # profiling aids (the headline line uses the defaults)
    ap.add_argument("--linears", default="all", help="comma-separated subset of the workload's linears")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the measurements outside the step (e2e, per-config passes, quantising epilogue, MoE "
                         "dispatch, NVFP4, quantiser sweep)")
    ap.add_argument("--per-config-iters", type=int, default=20)
    return ap.parse_args()


# DRAM traffic of one grouped_gemm_kernel launch from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum, mean over the fwd, dgrad and
# wgrad launches of the workload named below).  The figure belongs to the
# kernel sources it was taken on: when their hash differs the line reports
# null instead.
GEMM_TRAFFIC = {"bytes_per_launch": 1528028074, "workload": "the ds-v3-671b-like gate/up linear (N 4096, K 7168)",
                "sources_sha256": "b19e5160a346facb8e0a3c48976cebd46e5c39c213b4a01e7f673da3b597855e"}
GEMM_SOURCES = ("grouped_gemm.cu", "ptx.cuh", "codec.cuh", "launch.h", "tmap.cu")


def gemm_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, "mxfp8_grouped_gemm_quantize_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def step_peak(pk, timed_ms: float):
    """FP8 peak for kernels timed inside the step: the sustained figure once the
    timed region is a seconds-long loop (>= 0.5 s, where the power cap sets in),
    else the burst figure.  Returns (TFLOP/s, 'sustained' | 'burst')."""
    if timed_ms >= 500.0 and pk.get("bf16_sust"):
        return pk["bf16_sust"] * FP8_OVER_BF16, "sustained"
    return pk["bf16"] * FP8_OVER_BF16, "burst"


def gemm_traffic():
    """(bytes per GEMM launch, workload it was captured on), or (None, None)
    when no capture exists for the current kernel sources."""
    if GEMM_TRAFFIC["sources_sha256"] != gemm_sources_sha256():
        return None, None
    return GEMM_TRAFFIC["bytes_per_launch"], GEMM_TRAFFIC["workload"]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"], "bf16_sust": d.get("bf16_tflops_sustained"),
                "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sust": 1400.0, "src": "fallback"}


# ---------------------------------------------------------------- clocks (NVML reads only)
class ClockSampler:
    BAD = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}

    def __init__(self, device_index: int, period_s=0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self.stop_evt, self.thread = period_s, threading.Event(), None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _reason_names(self, mask):
        nv = self.nv
        names = {"hw_slowdown": getattr(nv, "nvmlClocksThrottleReasonHwSlowdown", 0x8),
                 "hw_thermal_slowdown": getattr(nv, "nvmlClocksThrottleReasonHwThermalSlowdown", 0x40),
                 "sw_thermal_slowdown": getattr(nv, "nvmlClocksThrottleReasonSwThermalSlowdown", 0x20),
                 "sw_power_cap": getattr(nv, "nvmlClocksThrottleReasonSwPowerCap", 0x4)}
        return {k for k, bit in names.items() if mask & bit}

    def _run(self):
        nv = self.nv
        while not self.stop_evt.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                self.reasons |= self._reason_names(fn(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        return self

    def __exit__(self, *a):
        if self.thread:
            self.stop_evt.set()
            self.thread.join()

    def summary(self):
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------- one grouped linear on the GPU
class Linear:
    """Device buffers and launches for one grouped linear (all three passes)."""

    def __init__(self, mx, w: wl.Workload, layer: wl.Layer, device, quantiser="dual"):
        self.mx = mx
        self.quantiser = quantiser
        self.name = layer.name
        self.M, self.N, self.K, self.E = w.M, layer.N, layer.K, w.E
        self.X, W, self.dY = wl.layer_tensors(w, layer, device=device)
        self.W2 = W.reshape(self.E * self.N, self.K)
        self.offs = torch.from_numpy(w.offsets).to(device)
        M, N, K, E = self.M, self.N, self.K, self.E
        u8 = lambda n: torch.empty(max(int(n), 16), dtype=torch.uint8, device=device)  # noqa: E731
        self.xq, self.xs = torch.empty((M, K), dtype=torch.uint8, device=device), u8(mx.mxfp8_rowwise_scale_bytes(M, K, E))
        self.wq, self.ws = torch.empty((E * N, K), dtype=torch.uint8, device=device), u8(mx.mxfp8_rowwise_scale_bytes(E * N, K, 1))
        self.dyq, self.dys = torch.empty((M, N), dtype=torch.uint8, device=device), u8(mx.mxfp8_rowwise_scale_bytes(M, N, E))
        self.wqT = torch.empty((K, mx.mxfp8_colwise_ld(E * N, 1)), dtype=torch.uint8, device=device)
        self.wsT = u8(mx.mxfp8_colwise_scale_bytes(E * N, K, 1))
        ldm = mx.mxfp8_colwise_ld(M, E)
        self.dyqT, self.dysT = torch.empty((N, ldm), dtype=torch.uint8, device=device), u8(mx.mxfp8_colwise_scale_bytes(M, N, E))
        self.xqT, self.xsT = torch.empty((K, ldm), dtype=torch.uint8, device=device), u8(mx.mxfp8_colwise_scale_bytes(M, K, E))
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        self.dx = torch.empty((M, K), dtype=torch.bfloat16, device=device)
        self.dw = torch.empty((E, N, K), dtype=torch.bfloat16, device=device)
        self.work = mx.new_workspace(E, M, N, K, device)

    def flops_per_pass(self):
        return 2 * self.M * self.N * self.K

    def quant_bytes(self):
        """Algorithmic bytes of quantising X, W and dY into both layouts: per
        element 2 B read per pass over the input and 1 + 1/32 B written per
        layout (dual: one read, separate: two reads)."""
        el = self.M * self.K + self.E * self.N * self.K + self.M * self.N
        reads = 1 if self.quantiser == "dual" else 2
        return el * (2 * reads + 2 * (1 + 1 / 32))

    def passes(self):
        """{pass: callable} for the three grouped GEMMs of this linear."""
        mx = self.mx
        return {
            "fwd": lambda: mx.mxfp8_grouped_gemm_fwd(self.xq, self.xs, self.wq, self.ws, self.offs, self.N,
                                                     out=self.y, work=self.work),
            "dgrad": lambda: mx.mxfp8_grouped_gemm_dgrad(self.dyq, self.dys, self.wqT, self.wsT, self.offs, self.K,
                                                         out=self.dx, work=self.work),
            "wgrad": lambda: mx.mxfp8_grouped_gemm_wgrad(self.dyqT, self.dysT, self.xqT, self.xsT, self.offs, self.M,
                                                         out=self.dw, work=self.work),
        }

    def dual_quantisations(self):
        """The three dual quantisations (X, W, dY: both layouts from one read)."""
        mx = self.mx
        return [
            lambda: mx.mxfp8_quantize_dual(self.X, self.offs, q=self.xq, scales=self.xs, qT=self.xqT,
                                           scalesT=self.xsT),
            lambda: mx.mxfp8_quantize_dual(self.W2, None, q=self.wq, scales=self.ws, qT=self.wqT, scalesT=self.wsT),
            lambda: mx.mxfp8_quantize_dual(self.dY, self.offs, q=self.dyq, scales=self.dys, qT=self.dyqT,
                                           scalesT=self.dysT),
        ]

    def launches(self):
        """(kind, callable) for one pass of the path; kind is 'quant' or 'gemm:<pass>'."""
        mx = self.mx
        g = self.passes()
        if self.quantiser == "dual":
            qx, qw, qdy = self.dual_quantisations()
            return [("quant", qx), ("quant", qw), ("gemm:fwd", g["fwd"]), ("quant", qdy),
                    ("gemm:dgrad", g["dgrad"]), ("gemm:wgrad", g["wgrad"])]
        return [
            ("quant", lambda: mx.mxfp8_quantize_rowwise(self.X, self.offs, q=self.xq, scales=self.xs)),
            ("quant", lambda: mx.mxfp8_quantize_rowwise(self.W2, None, q=self.wq, scales=self.ws)),
            ("gemm:fwd", g["fwd"]),
            ("quant", lambda: mx.mxfp8_quantize_rowwise(self.dY, self.offs, q=self.dyq, scales=self.dys)),
            ("quant", lambda: mx.mxfp8_quantize_colwise(self.W2, None, qT=self.wqT, scales=self.wsT)),
            ("gemm:dgrad", g["dgrad"]),
            ("quant", lambda: mx.mxfp8_quantize_colwise(self.dY, self.offs, qT=self.dyqT, scales=self.dysT)),
            ("quant", lambda: mx.mxfp8_quantize_colwise(self.X, self.offs, qT=self.xqT, scales=self.xsT)),
            ("gemm:wgrad", g["wgrad"]),
        ]


def system_info(device_index: int = 0) -> dict:
    """GPU name, driver, CUDA and torch versions and host cores, for the JSON
    line (reads only; every field is None when it cannot be read)."""
    info = {"gpu": None, "driver": None, "cuda": torch.version.cuda, "torch": torch.__version__,
            "host_cores": os.cpu_count()}
    try:
        info["gpu"] = torch.cuda.get_device_name(device_index)
    except Exception:
        pass
    try:
        import pynvml
        pynvml.nvmlInit()
        v = pynvml.nvmlSystemGetDriverVersion()
        info["driver"] = v.decode() if isinstance(v, bytes) else v
    except Exception:
        pass
    return info


ROUTING = {
    "tiny": "counts [0, 7, 21, 36]",
    "ds-v3-16b": "top-6 of 64 experts over 8192 tokens; N(0,1) logits + N(0,0.5) expert bias",
    "ds-v3-671b": "one GPU's share of top-8 of 256 experts over 16384 tokens: 32 local experts, 16384 rows, "
                  "Multinomial counts with Zipf(1.1) weights in a seeded order",
    "llama4-scout": "top-1 of 16 experts over 16384 tokens; N(0,1) logits",
}


def workload_config(w, quantiser: str, world: int) -> dict:
    """The `config` object of the JSON line, identical for both arms."""
    return {"workload": f"{w.name}-like MoE layer", "experts": w.E, "routed_rows": w.M,
            "layers": [{"name": L.name, "N": L.N, "K": L.K} for L in w.layers],
            "routing": ROUTING.get(w.name, w.name),
            "l2": "inputs larger than L2 (126 MB): the step's operands are several GB",
            "parallelism": f"replica x{world}", "quantiser": quantiser}


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest x over all ranks: a job's time is its slowest rank's."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: float, ms: float, world: int) -> float:
    """Throughput of the whole job: every rank's units over the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def run_ours(args, rank, world, local_rank):
    import mxfp8_grouped_gemm_quantize_b200 as mx
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if not mx.mxfp8_device_supported():
        raise SystemExit("bench: the current device is not sm_100")
    w = wl.WORKLOADS[args.workload]()
    chosen = w.layers if args.linears == "all" else [L for L in w.layers if L.name in args.linears.split(",")]
    if not chosen:
        raise SystemExit(f"bench: no linear named {args.linears!r} in {w.name}")
    layers = [Linear(mx, w, L, dev, args.quantiser) for L in chosen]
    calls = [c for L in layers for c in L.launches()]
    step_flops = 3 * sum(L.flops_per_pass() for L in layers)
    quant_bytes = sum(L.quant_bytes() for L in layers)
    stream = torch.cuda.current_stream()

    def step():
        for _, fn in calls:
            fn()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    for L in layers:
        st = mx.mxfp8_get_status(L.work)
        if st != 0:
            raise SystemExit(f"bench: device status {st} after warm-up")

    # per-launch events inside the timed region (same stream as the launches)
    K = args.steps
    n_calls = len(calls)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_calls + 1)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        start.record(stream)
        for s in range(K):
            e = ev[s]
            e[0].record(stream)
            for i, (_, fn) in enumerate(calls):
                fn()
                e[i + 1].record(stream)
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms_total = start.elapsed_time(end)
    per_kind = {}
    for s in range(K):
        for i, (kind, _) in enumerate(calls):
            per_kind.setdefault(kind, []).append(ev[s][i].elapsed_time(ev[s][i + 1]))
    ms_total = max_over_ranks(ms_total, world, dev)
    ms_step = ms_total / K
    value = whole_job_tflops(step_flops, ms_step, world)

    pk = peaks()
    fp8_peak = pk["bf16"] * FP8_OVER_BF16              # burst: kernels timed alone
    in_step_peak, peak_kind = step_peak(pk, ms_total)  # kernels timed inside the step loop
    traffic, traffic_wl = gemm_traffic()
    gemm_ms = sum(sum(v) for k, v in per_kind.items() if k.startswith("gemm")) / K
    gemm_launches = sum(len(v) for k, v in per_kind.items() if k.startswith("gemm"))
    gemm_tflops = step_flops / (gemm_ms * 1e-3) / 1e12
    quant_ms = sum(per_kind["quant"]) / K
    quant_gbs = quant_bytes / (quant_ms * 1e-3) / 1e9
    breakdown = {}
    for kind, v in per_kind.items():
        if kind.startswith("gemm"):
            p = kind.split(":")[1]
            breakdown[p] = {"ms_per_step": round(sum(v) / K, 4),
                            "tflops": round((step_flops / 3) / (sum(v) / K * 1e-3) / 1e12, 1)}
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": max(3, args.warmup), "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 (fp32 accumulate)", "data": "synthetic",
        "config": workload_config(w, args.quantiser, world),
        "fraction_of_fp8_peak": round(value / world / in_step_peak, 4),
        "roofline": {"kernel": "grouped_gemm_kernel (fwd+dgrad+wgrad launches)", "bound": "tensor",
                     "achieved": round(gemm_tflops, 1), "peak": round(in_step_peak, 1), "unit": "TFLOP/s",
                     "frac": round(gemm_tflops / in_step_peak, 4),
                     "frac_of_burst_peak": round(gemm_tflops / fp8_peak, 4), "traffic": traffic,
                     "traffic_source": (f"ncu dram__bytes_read.sum + dram__bytes_write.sum per launch, mean over the "
                                        f"fwd, dgrad and wgrad launches of {traffic_wl}" if traffic is not None else
                                        "no ncu capture of the current kernel sources"),
                     "peak_source": (f"{pk['src']} bf16 {peak_kind} x {FP8_OVER_BF16} (nominal FP8/BF16); "
                                     f"timed region {ms_total:.0f} ms"),
                     "launches_timed": gemm_launches},
        "quantiser": {"achieved_gbs": round(quant_gbs, 1), "peak_gbs": pk["hbm_gbs"],
                      "frac": round(quant_gbs / pk["hbm_gbs"], 4), "ms_per_step": round(quant_ms, 4)},
        "breakdown": breakdown,
        "gpu_launches": K * n_calls,
        "clocks": clk.summary(),
        "system": system_info(local_rank),
    }
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        out["cpu_baseline"] = cpu_baseline(w, budget_s=12.0)
    if args.linears != "all":
        out["config"]["linears_timed"] = [L.name for L in layers]
    if not args.no_extras:
        out["e2e"] = e2e(args, mx, w, layers, dev, world)
        out["per_config"] = per_config(mx, args, fp8_peak, pk["hbm_gbs"], dev, local_rank)
        c2 = out["per_config"].get("ds-v3-671b")
        if c2 is not None:
            out["fwd_frac"] = {"workload": "ds-v3-671b-like MoE layer, both linears, forward launches timed alone",
                               "tflops": c2["passes"]["fwd"]["tflops"], "frac": c2["passes"]["fwd"]["frac"],
                               "target": 0.60, "peak": round(fp8_peak, 1)}
        out["quantising_epilogue"] = quantising_epilogue(mx, layers[0])
        out["moe_dispatch"] = moe_dispatch(mx, args, pk["hbm_gbs"])
        out["ep_dispatch"] = ep_dispatch(mx, pk["hbm_gbs"])
        out["nvfp4"] = nvfp4_measure(mx, layers[0], fp8_peak, pk["hbm_gbs"])
        out["quantiser_sweep"] = quantiser_sweep(mx, pk["hbm_gbs"])
    return out


def timed_alone(fn, flush, iters, clean=False):
    """Median CUDA-event time (ms) of one launch with L2 flushed before it,
    after five warm-up launches.  The flush writes a buffer twice the size of
    L2; clean=True also reads it back, so L2 is left holding clean lines
    instead of up to a full L2 of dirty ones that the timed launch would have
    to write back to HBM on its first misses (which charges a bandwidth-bound
    kernel for traffic that is not its own)."""
    for _ in range(5):
        fn()
    ts = []
    for _ in range(iters):
        flush.zero_()
        if clean:
            flush.sum()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def per_config(mx, args, fp8_peak, hbm_gbs, dev, device_index):
    """Every grouped GEMM pass (fwd, dgrad, wgrad of both linears) of the three
    MoE workloads, each launch timed alone with L2 flushed before it (median
    of --per-config-iters), and the dual quantiser on each linear's X, W and
    dY timed the same way.  TFLOP/s are algorithmic (2*M*N*K over real
    tokens); fractions are of the FP8 peak of the roofline."""
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * max(l2, 64 << 20), dtype=torch.uint8, device=dev)
    it = max(3, args.per_config_iters)
    res = {}
    with ClockSampler(device_index) as clk:
        for name in ("ds-v3-16b", "ds-v3-671b", "llama4-scout"):
            w = wl.WORKLOADS[name]()
            cfg = {"routing": ROUTING[name], "experts": w.E, "routed_rows": w.M, "linears": {}}
            tot = {p: [0.0, 0.0] for p in ("fwd", "dgrad", "wgrad")}
            q_bytes, q_ms, q_ms_dirty = 0.0, 0.0, 0.0
            for layer in w.layers:
                L = Linear(mx, w, layer, dev, "dual")
                for fn in L.dual_quantisations():
                    fn()
                r = {"N": L.N, "K": L.K}
                for p, fn in L.passes().items():
                    ms = timed_alone(fn, flush, it)
                    fl = L.flops_per_pass()
                    tot[p][0] += fl
                    tot[p][1] += ms
                    r[p] = {"ms": round(ms, 4), "tflops": round(fl / (ms * 1e-3) / 1e12, 1),
                            "frac": round(fl / (ms * 1e-3) / 1e12 / fp8_peak, 4)}
                if mx.mxfp8_get_status(L.work) != 0:
                    raise SystemExit(f"bench: device status error in the {name} {layer.name} passes")
                for fn in L.dual_quantisations():
                    q_ms += timed_alone(fn, flush, it, clean=True)
                    q_ms_dirty += timed_alone(fn, flush, it)
                q_bytes += L.quant_bytes()
                cfg["linears"][layer.name] = r
                del L
                torch.cuda.empty_cache()
            cfg["passes"] = {p: {"tflops": round(f / (ms * 1e-3) / 1e12, 1),
                                 "frac": round(f / (ms * 1e-3) / 1e12 / fp8_peak, 4)} for p, (f, ms) in tot.items()}
            f_all, ms_all = sum(v[0] for v in tot.values()), sum(v[1] for v in tot.values())
            cfg["all_passes"] = {"tflops": round(f_all / (ms_all * 1e-3) / 1e12, 1),
                                 "frac": round(f_all / (ms_all * 1e-3) / 1e12 / fp8_peak, 4)}
            gbs = q_bytes / (q_ms * 1e-3) / 1e9
            gbs_dirty = q_bytes / (q_ms_dirty * 1e-3) / 1e9
            cfg["quantiser"] = {"kernel": "quantize_dual_kernel (X, W, dY of both linears)", "ms": round(q_ms, 4),
                                "gbs": round(gbs, 1), "frac": round(gbs / hbm_gbs, 4),
                                "flush": "written, then read back (L2 left clean)",
                                "write_only_flush": {"ms": round(q_ms_dirty, 4), "gbs": round(gbs_dirty, 1),
                                                     "frac": round(gbs_dirty / hbm_gbs, 4)}}
            res[name] = cfg
    del flush
    torch.cuda.empty_cache()
    res["method"] = (f"each launch alone, L2 flushed before it ({2 * max(l2, 64 << 20) >> 20} MiB written; the "
                     f"quantisers' flush also reads it back), five warm-ups, median of {it}")
    res["clocks"] = clk.summary()
    return res


def e2e(args, mx, w, layers, dev, world):
    """Same metric through the public API with host buffers: every step copies
    the bf16 inputs (X, W, dY of both linears) and the offsets from pinned host
    memory, runs the path and copies Y, dX and dW back to pinned host memory.
    Steps are pipelined the way a training loop prefetches its next batch:
    host-to-device copies on one stream, the path on the current stream and
    device-to-host copies on a third, with two device buffer sets, so step
    k+1's inputs and step k-1's outputs cross PCIe (one direction each) while
    step k computes.  The timed region spans all K steps' copies and compute."""
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    in_names, out_names = ("X", "W2", "dY", "offs"), ("y", "dx", "dw")
    sets = []   # per buffer set: {layer index: {name: device tensor}}
    for b in range(2):
        sets.append([{n: (getattr(L, n) if b == 0 else torch.empty_like(getattr(L, n)))
                      for n in in_names + out_names} for L in layers])
    host_in = [{n: getattr(L, n).cpu().pin_memory() for n in in_names} for L in layers]
    host_out = [{n: torch.empty_like(getattr(L, n), device="cpu").pin_memory() for n in out_names} for L in layers]
    calls = [fn for L in layers for _, fn in L.launches()]
    h2d = sum(h.numel() * h.element_size() for d in host_in for h in d.values())
    d2h = sum(h.numel() * h.element_size() for d in host_out for h in d.values())
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "comp", "out")}
    used = [False, False]

    def step(k):
        b = k % 2
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(ev["comp"][b])      # set b's inputs were read by step k-2
            for i, d in enumerate(host_in):
                for n, h in d.items():
                    sets[b][i][n].copy_(h, non_blocking=True)
            ev["in"][b].record(s_in)
        comp.wait_event(ev["in"][b])
        if used[b]:
            comp.wait_event(ev["out"][b])           # set b's outputs were copied out by step k-2
        for i, L in enumerate(layers):
            for n in in_names + out_names:
                setattr(L, n, sets[b][i][n])
        for fn in calls:
            fn()
        ev["comp"][b].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["comp"][b])
            for i, d in enumerate(host_out):
                for n, h in d.items():
                    h.copy_(sets[b][i][n], non_blocking=True)
            ev["out"][b].record(s_out)
        used[b] = True

    for k in range(2):
        step(k)
    torch.cuda.synchronize()
    K = max(1, args.e2e_steps)
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    a.record(comp)
    s_in.wait_event(a)
    s_out.wait_event(a)
    for k in range(K):
        step(k)
    comp.wait_event(ev["out"][(K - 1) % 2])
    z.record(comp)
    torch.cuda.synchronize()
    ms = a.elapsed_time(z) / K
    for i, L in enumerate(layers):
        for n in in_names + out_names:
            setattr(L, n, sets[0][i][n])
    ms = max_over_ranks(ms, world, dev)
    flops = 3 * sum(L.flops_per_pass() for L in layers)
    return {"value": round(whole_job_tflops(flops, ms, world), 2), "unit": UNIT, "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": K,
            "pipelined": "h2d / compute / d2h on three streams, two device buffer sets"}


def quantising_epilogue(mx, L: Linear, iters=20):
    """The quantising epilogue (the GEMM writes its output as MXFP8 too)
    against the GEMM followed by the dual quantiser on its bf16 output, for
    fwd and dgrad of one linear.  Not part of the step above; reported as
    its own measurement."""
    dev = L.y.device
    M, E = L.M, L.E
    ld = mx.mxfp8_colwise_ld(M, E)
    res = {"linear": L.name}
    for mode, C in (("fwd", L.N), ("dgrad", L.K)):
        out = L.y if mode == "fwd" else L.dx
        row = (torch.empty((M, C), dtype=torch.uint8, device=dev),
               torch.empty(mx.mxfp8_rowwise_scale_bytes(M, C, E), dtype=torch.uint8, device=dev))
        col = (torch.empty((C, ld), dtype=torch.uint8, device=dev),
               torch.empty(mx.mxfp8_colwise_scale_bytes(M, C, E), dtype=torch.uint8, device=dev))
        if mode == "fwd":
            plain = lambda: mx.mxfp8_grouped_gemm_fwd(L.xq, L.xs, L.wq, L.ws, L.offs, L.N, out=out, work=L.work)  # noqa: E731
            fused = lambda o: mx.mxfp8_grouped_gemm_fwd_quant(L.xq, L.xs, L.wq, L.ws, L.offs, L.N, out=o,  # noqa: E731
                                                              rowwise=row, colwise=col, work=L.work)
        else:
            plain = lambda: mx.mxfp8_grouped_gemm_dgrad(L.dyq, L.dys, L.wqT, L.wsT, L.offs, L.K, out=out,  # noqa: E731
                                                        work=L.work)
            fused = lambda o: mx.mxfp8_grouped_gemm_dgrad_quant(L.dyq, L.dys, L.wqT, L.wsT, L.offs, L.K, out=o,  # noqa: E731
                                                                rowwise=row, colwise=col, work=L.work)
        quant = lambda: mx.mxfp8_quantize_dual(out, L.offs, q=row[0], scales=row[1], qT=col[0], scalesT=col[1])  # noqa: E731
        variants = {"gemm_then_dual_quantiser": lambda: (plain(), quant()),
                    "quantising_epilogue": lambda: fused(out),
                    "quantising_epilogue_no_bf16": lambda: fused(None)}
        r = {}
        for name, fn in variants.items():
            for _ in range(3):
                fn()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record()
            for _ in range(iters):
                fn()
            b.record()
            torch.cuda.synchronize()
            r[name + "_ms"] = round(a.elapsed_time(b) / iters, 4)
        st = mx.mxfp8_get_status(L.work)
        if st != 0:
            raise SystemExit(f"bench: device status {st} in the quantising-epilogue measurement")
        r["tflops"] = round(L.flops_per_pass() / (r["quantising_epilogue_ms"] * 1e-3) / 1e12, 1)
        res[mode] = r
    if L.N % 256 == 0:
        # gate/up forward fused with SwiGLU and MXFP8 of h [M, N/2] (both
        # layouts, no bf16 h), against the unfused path's lower bound: the
        # GEMM writing bf16 Y [M, N], then the dual quantiser on an h-sized
        # tensor (the elementwise SwiGLU pass itself is not counted)
        I = L.N // 2
        h = torch.empty((M, I), dtype=torch.bfloat16, device=dev)
        row = (torch.empty((M, I), dtype=torch.uint8, device=dev),
               torch.empty(mx.mxfp8_rowwise_scale_bytes(M, I, E), dtype=torch.uint8, device=dev))
        col = (torch.empty((I, ld), dtype=torch.uint8, device=dev),
               torch.empty(mx.mxfp8_colwise_scale_bytes(M, I, E), dtype=torch.uint8, device=dev))
        variants = {
            "gemm_then_dual_quantiser_ms": lambda: (
                mx.mxfp8_grouped_gemm_fwd(L.xq, L.xs, L.wq, L.ws, L.offs, L.N, out=L.y, work=L.work),
                mx.mxfp8_quantize_dual(h, L.offs, q=row[0], scales=row[1], qT=col[0], scalesT=col[1])),
            "fused_swiglu_ms": lambda: mx.mxfp8_grouped_gemm_fwd_swiglu(L.xq, L.xs, L.wq, L.ws, L.offs, L.N, out=None,
                                                                      rowwise=row, colwise=col, work=L.work),
            "fused_swiglu_with_bf16_h_ms": lambda: mx.mxfp8_grouped_gemm_fwd_swiglu(
                L.xq, L.xs, L.wq, L.ws, L.offs, L.N, out=h, rowwise=row, colwise=col, work=L.work),
        }
        r = {}
        for name, fn in variants.items():
            for _ in range(3):
                fn()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record()
            for _ in range(iters):
                fn()
            b.record()
            torch.cuda.synchronize()
            r[name] = round(a.elapsed_time(b) / iters, 4)
        if mx.mxfp8_get_status(L.work) != 0:
            raise SystemExit("bench: device status error in the SwiGLU measurement")
        r["tflops"] = round(L.flops_per_pass() / (r["fused_swiglu_ms"] * 1e-3) / 1e12, 1)
        r["unfused_note"] = "lower bound of the unfused path: GEMM to bf16 Y, then the dual quantiser on an [M, N/2] tensor"
        res["swiglu_fwd"] = r
        del h, row, col
    return res


def moe_dispatch(mx, args, hbm_gbs, iters=20):
    """The steps around the GEMMs on the DeepSeek-V3-16B-like routing (8192
    tokens, top-6 of 64 experts, hidden 2048): the dispatch plan, the token
    permute fused with dual MXFP8 quantisation, and the weighted combine of
    the down projection's outputs.  Timed on their own, not in the step."""
    r = wl.routing("ds-v3-16b")
    dev = torch.device("cuda", torch.cuda.current_device())
    idx = torch.from_numpy(r.idx).to(dev)
    w = torch.from_numpy(r.w).to(dev)
    x = wl.normal_bf16((r.T, r.K), 1.0, 101, device=dev)
    offs, perm, inv, work = mx.mxfp8_moe_plan(idx, r.E)
    R = perm.numel()
    q, s, qT, sT = mx.mxfp8_permute_quantize_dual(x, perm, offs)
    yp = wl.normal_bf16((R, r.K), 1.0, 102, device=dev)
    y = torch.empty((r.T, r.K), dtype=torch.bfloat16, device=dev)

    def t(fn):
        for _ in range(3):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for _ in range(iters):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / iters

    plan_ms = t(lambda: mx.mxfp8_moe_plan(idx, r.E, work=work))
    pq_ms = t(lambda: mx.mxfp8_permute_quantize_dual(x, perm, offs, q, s, qT, sT))
    cb_ms = t(lambda: mx.mxfp8_moe_combine(yp, inv, w, out=y))
    if mx.mxfp8_get_status(work) != 0:
        raise SystemExit("bench: dispatch plan reported a bad routing")
    pq_bytes = R * r.K * (2 + 2 * (1 + 1 / 32))          # gathered bf16 read, both MXFP8 layouts written
    cb_bytes = R * r.K * 2 + r.T * r.K * 2               # expert outputs read, token outputs written
    return {"routing": f"{r.T} tokens, top-{r.k} of {r.E}, hidden {r.K}", "plan_ms": round(plan_ms, 4),
            "permute_quantize_ms": round(pq_ms, 4),
            "permute_quantize_gbs": round(pq_bytes / (pq_ms * 1e-3) / 1e9, 1),
            "permute_quantize_frac": round(pq_bytes / (pq_ms * 1e-3) / 1e9 / hbm_gbs, 4),
            "combine_ms": round(cb_ms, 4), "combine_gbs": round(cb_bytes / (cb_ms * 1e-3) / 1e9, 1),
            "combine_frac": round(cb_bytes / (cb_ms * 1e-3) / 1e9 / hbm_gbs, 4)}


def ep_dispatch(mx, hbm_gbs, iters=20):
    """The expert-parallel exchange's device work for a DeepSeek-V3-671B-like
    layer split over 8 ranks (16384 tokens, 2048 per rank, hidden 7168, top-8
    of 256 experts with N(0,1) logits + N(0,0.5) expert bias, 32 experts per
    rank), on one GPU: one source's plan and quantise-and-pack, one
    receiver's unpack of what the 8 sources send it (assembled here as the
    all-to-all delivers it), and the return gather of its expert outputs.
    The transfer itself is not timed (one GPU per run)."""
    from mxfp8_grouped_gemm_quantize_b200 import ep
    P, Tr, k, E, C = 8, 2048, 8, 256, 7168
    epr = E // P
    dev = torch.device("cuda", torch.cuda.current_device())
    rng = np.random.default_rng(4242)
    bias = rng.normal(0.0, 0.5, E)
    srcs = []
    for q in range(P):
        logits = rng.standard_normal((Tr, E)) + bias[None, :]
        idx = torch.from_numpy(np.argsort(-logits, axis=1, kind="stable")[:, :k].astype(np.int32)).to(dev)
        x = wl.normal_bf16((Tr, C), 1.0, 300 + q, device=dev)
        counts, rec_token, pe, prc, ret_pos, work = mx.mxfp8_ep_plan(idx, E, P)
        cnt = counts.tolist()
        R, S = sum(cnt[:P]), sum(cnt[P:])
        srcs.append((idx, x, cnt, rec_token[:R], pe[:S], prc[:S], work, mx.mxfp8_ep_pack(x, rec_token[:R])))

    def t(fn):
        for _ in range(3):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for _ in range(iters):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / iters

    idx0, x0, cnt0, rt0, _, _, work0, recs0 = srcs[0]
    plan_ms = t(lambda: mx.mxfp8_ep_plan(idx0, E, P, work=work0))
    pack_ms = t(lambda: mx.mxfp8_ep_pack(x0, rt0, out=recs0))
    stride = mx.mxfp8_ep_record_bytes(C)
    R0, S0 = sum(cnt0[:P]), sum(cnt0[P:])

    def block(c, p):
        return slice(sum(c[:p]), sum(c[:p + 1]))
    recs = torch.cat([s[7][block(s[2][:P], 0)] for s in srcs])
    pe = torch.cat([s[4][block(s[2][P:], 0)] for s in srcs])
    prc = torch.cat([s[5][block(s[2][P:], 0)] for s in srcs])
    rc = [s[2][0] for s in srcs] + [s[2][P] for s in srcs]
    d = ep.Dispatch(recs, pe, prc, rc, cnt0, C)
    offs, perm, inv, q, sf = ep.receive(d, epr)
    src_base = torch.tensor(ep.source_bases(rc), dtype=torch.int32, device=dev)
    unpack_ms = t(lambda: mx.mxfp8_ep_unpack(recs, C, prc, src_base, perm, offs, q, sf))
    rows = perm.numel()
    y = wl.normal_bf16((rows, C), 1.0, 333, device=dev)
    y_ret = torch.empty_like(y)
    inv_flat = inv.view(-1).contiguous()
    gather_ms = t(lambda: mx.mxfp8_gather_rows(y, inv_flat, out=y_ret))
    pack_bytes = R0 * (2 * C + stride)
    unpack_bytes = rows * 2 * (C + C // 32)
    gather_bytes = rows * C * 2 * 2
    wire = R0 * stride + S0 * 8
    return {"layout": f"{P} ranks x {Tr} tokens, hidden {C}, top-{k} of {E} experts ({epr} per rank)",
            "records_sent": R0, "pairs_sent": S0,
            "dispatch_bytes": wire, "dispatch_bytes_bf16_rows": S0 * 2 * C,
            "dispatch_bytes_ratio": round(wire / (S0 * 2 * C), 4),
            "plan_ms": round(plan_ms, 4),
            "pack_ms": round(pack_ms, 4), "pack_gbs": round(pack_bytes / (pack_ms * 1e-3) / 1e9, 1),
            "pack_frac": round(pack_bytes / (pack_ms * 1e-3) / 1e9 / hbm_gbs, 4),
            "receiver_rows": rows,
            "unpack_ms": round(unpack_ms, 4), "unpack_gbs": round(unpack_bytes / (unpack_ms * 1e-3) / 1e9, 1),
            "unpack_frac": round(unpack_bytes / (unpack_ms * 1e-3) / 1e9 / hbm_gbs, 4),
            "return_gather_ms": round(gather_ms, 4),
            "return_gather_gbs": round(gather_bytes / (gather_ms * 1e-3) / 1e9, 1),
            "note": "device work only; the all-to-all transfer is not measured (one GPU per run)"}


def nvfp4_measure(mx, L: Linear, fp8_peak, hbm_gbs, iters=20):
    """The NVFP4 variant of one linear (same shapes and routing): tensor amax,
    the rowwise / colwise quantisers of X, W and dY, and the three grouped
    GEMMs on E2M1 x E2M1 block-scaled MMAs.  Timed on its own; the FP4 dense
    peak is twice the FP8 one (nominal ratio 9 / 4.5 PFLOP/s)."""
    X, W2, dY, od = L.X, L.W2, L.dY, L.offs

    def t(fn):
        for _ in range(3):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for _ in range(iters):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / iters

    ax, aw, ady = mx.mxfp8_nvfp4_amax(X), mx.mxfp8_nvfp4_amax(W2), mx.mxfp8_nvfp4_amax(dY)
    xq, xs = mx.mxfp8_nvfp4_quantize_rowwise(X, ax, od)
    wq, ws = mx.mxfp8_nvfp4_quantize_rowwise(W2, aw)
    dyq, dys = mx.mxfp8_nvfp4_quantize_rowwise(dY, ady, od)
    wqT, wsT = mx.mxfp8_nvfp4_quantize_colwise(W2, aw)
    dyqT, dysT = mx.mxfp8_nvfp4_quantize_colwise(dY, ady, od)
    xqT, xsT = mx.mxfp8_nvfp4_quantize_colwise(X, ax, od)
    quant = [lambda: mx.mxfp8_nvfp4_amax(X, ax), lambda: mx.mxfp8_nvfp4_amax(W2, aw),
             lambda: mx.mxfp8_nvfp4_amax(dY, ady),
             lambda: mx.mxfp8_nvfp4_quantize_rowwise(X, ax, od, xq, xs),
             lambda: mx.mxfp8_nvfp4_quantize_rowwise(W2, aw, None, wq, ws),
             lambda: mx.mxfp8_nvfp4_quantize_rowwise(dY, ady, od, dyq, dys),
             lambda: mx.mxfp8_nvfp4_quantize_colwise(W2, aw, None, wqT, wsT),
             lambda: mx.mxfp8_nvfp4_quantize_colwise(dY, ady, od, dyqT, dysT),
             lambda: mx.mxfp8_nvfp4_quantize_colwise(X, ax, od, xqT, xsT)]
    q_ms = t(lambda: [f() for f in quant])
    el = L.X.numel() + L.W2.numel() + L.dY.numel()
    q_bytes = el * 2 + 2 * el * (2 + 0.5 + 1 / 16)        # amax reads, then two quantisations each
    fl = L.flops_per_pass()
    r = {"linear": L.name, "peak_tflops": round(2 * fp8_peak, 1)}
    for name, fn in (("fwd", lambda: mx.mxfp8_nvfp4_grouped_gemm_fwd(xq, xs, ax, wq, ws, aw, od, L.N, out=L.y,
                                                                       work=L.work)),
                     ("dgrad", lambda: mx.mxfp8_nvfp4_grouped_gemm_dgrad(dyq, dys, ady, wqT, wsT, aw, od, L.K,
                                                                         out=L.dx, work=L.work)),
                     ("wgrad", lambda: mx.mxfp8_nvfp4_grouped_gemm_wgrad(dyqT, dysT, ady, xqT, xsT, ax, od, L.M,
                                                                         out=L.dw, work=L.work))):
        ms = t(fn)
        r[name] = {"ms": round(ms, 4), "tflops": round(fl / (ms * 1e-3) / 1e12, 1),
                   "frac": round(fl / (ms * 1e-3) / 1e12 / (2 * fp8_peak), 4)}
    if mx.mxfp8_get_status(L.work) != 0:
        raise SystemExit("bench: NVFP4 GEMM reported a device error")
    r["quantisers"] = {"ms": round(q_ms, 4), "gbs": round(q_bytes / (q_ms * 1e-3) / 1e9, 1),
                       "frac": round(q_bytes / (q_ms * 1e-3) / 1e9 / hbm_gbs, 4)}
    return r


# ---------------------------------------------------------------- CPU oracle baseline / reference arm
def _cpu_sample(w: wl.Workload, budget_s: float):
    """Times the oracle's bf16-input fp32-accumulate fwd, dgrad and wgrad on
    a bounded sample of the first linear (rows / output rows chosen so the
    sample takes about budget_s); returns (flops, seconds, description)."""
    import oracle
    layer = w.layers[0]
    X, W, dY = wl.layer_tensors(w, layer)
    W2 = W.reshape(w.E * layer.N, layer.K)
    offs = w.offsets
    N, K, M = layer.N, layer.K, w.M
    cal = min(M, 512)
    oracle.baseline_fwd_f32(X, W2, offs, N, 0, 16)                    # thread start-up
    t0 = time.perf_counter()
    oracle.baseline_fwd_f32(X, W2, offs, N, 0, cal)
    rate = 2 * cal * N * K / max(time.perf_counter() - t0, 1e-6)      # FLOP/s estimate
    rows = int(max(1, min(M, budget_s / 3 * rate / (2 * N * K))))
    # wgrad sample: output rows n in [0, nr) for every expert (work 2*M*nr*K)
    nr = int(max(1, min(N, budget_s / 3 * rate / (2 * M * K))))
    Y = np.zeros((M, N), dtype=np.float32)
    dX = np.zeros((M, K), dtype=np.float32)
    dW = np.zeros((w.E, N, K), dtype=np.float32)
    t0 = time.perf_counter()
    oracle.baseline_fwd_f32(X, W2, offs, N, 0, rows, out=Y)
    oracle.baseline_dgrad_f32(dY, W2, offs, K, 0, rows, out=dX)
    oracle.baseline_wgrad_f32(dY, X, offs, 0, nr, out=dW)
    secs = time.perf_counter() - t0
    flops = 2 * rows * N * K * 2 + 2 * M * nr * K
    desc = (f"{layer.name} linear of {w.name}: fwd+dgrad on rows 0..{rows - 1} of {M}, "
            f"wgrad on output rows 0..{nr - 1} of {N} for all {w.E} experts")
    return flops, secs, desc


def quantiser_sweep(mx, hbm_gbs, iters=20):
    """The quantiser sweep: M in {4096, 16384, 65536} x K in {2048, 5120, 7168},
    one group, N(0,1) with 0.1 % outliers x1000 and 1 % of aligned 32x32 tiles
    zeroed.  Rowwise, colwise and dual kernels, each launch timed alone with L2
    flushed before it; GB/s of algorithmic bytes (rowwise / colwise:
    2 + 1 + 1/32 B per element, dual: 2 + 2 (1 + 1/32))."""
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device="cuda")

    def t(fn, clean=True):
        return timed_alone(fn, flush, iters, clean)

    rows = []
    for M, K in wl.quantiser_sweep():
        x = wl.sweep_tensor(M, K, device="cuda")
        q, sf = mx.mxfp8_quantize_rowwise(x)
        qT, sfT = mx.mxfp8_quantize_colwise(x)
        r = {"M": M, "K": K}
        for name, fn, bpe in (("rowwise", lambda: mx.mxfp8_quantize_rowwise(x, None, q=q, scales=sf), 3.03125),
                              ("colwise", lambda: mx.mxfp8_quantize_colwise(x, None, qT=qT, scales=sfT), 3.03125),
                              ("dual", lambda: mx.mxfp8_quantize_dual(x, None, q=q, scales=sf, qT=qT, scalesT=sfT),
                               4.0625)):
            ms, ms_dirty = t(fn), t(fn, clean=False)
            gbs, gbs_dirty = M * K * bpe / (ms * 1e-3) / 1e9, M * K * bpe / (ms_dirty * 1e-3) / 1e9
            r[name] = {"us": round(ms * 1e3, 1), "gbs": round(gbs, 1), "frac": round(gbs / hbm_gbs, 4),
                       "write_only_flush": {"us": round(ms_dirty * 1e3, 1), "frac": round(gbs_dirty / hbm_gbs, 4)}}
        rows.append(r)
        del x, q, sf, qT, sfT
    torch.cuda.empty_cache()
    return {"input": "N(0,1), 0.1 % outliers x1000, 1 % of aligned 32x32 tiles zeroed; one group",
            "method": (f"each launch alone, L2 flushed before it (a 256 MiB buffer written, then read back, so L2 "
                       f"holds clean lines; write_only_flush: written only), five warm-ups, median of {iters}"),
            "peak_gbs": hbm_gbs, "sizes": rows}


def _cpu_quantiser(budget_s=2.0):
    """The oracle's rowwise quantiser on the smallest sweep size (4096 x 2048):
    GB/s of the same algorithmic bytes as the GPU sweep."""
    import oracle
    x = wl.sweep_tensor(4096, 2048)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.quantize_rowwise(x)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    secs = (time.perf_counter() - t0) / n
    return {"gbs": round(4096 * 2048 * 3.03125 / secs / 1e9, 3), "kernel": "rowwise", "M": 4096, "K": 2048,
            "seconds_per_call": round(secs, 4)}


CPU_BUILD = ("oracle/baseline_f32.c: bf16 inputs, fp32 accumulation, OpenMP over experts x 8-row blocks, "
             "gcc -O3 -march=x86-64-v3 -ffp-contract=fast")


def cpu_baseline(w, budget_s=12.0):
    import oracle
    flops, secs, desc = _cpu_sample(w, budget_s)
    return {"value": round(flops / secs / 1e12, 5), "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "sample": desc, "seconds": round(secs, 2), "build": CPU_BUILD, "quantiser": _cpu_quantiser()}


def run_reference(args):
    import oracle
    w = wl.WORKLOADS[args.workload]()
    steps, warm = max(1, args.steps), max(0, args.warmup)
    per_step = max(0.05, min(2.0, 120.0 / (steps + warm)))
    for _ in range(warm):
        _cpu_sample(w, per_step)
    tot_f, tot_s, desc = 0, 0.0, ""
    for _ in range(steps):
        f, s, desc = _cpu_sample(w, per_step)
        tot_f += f
        tot_s += s
    value = tot_f / tot_s / 1e12
    return {"metric": METRIC, "value": round(value, 5), "unit": UNIT, "n_gpus": args.gpus, "steps": steps,
            "warmup": warm, "ms_per_step": round(1e3 * tot_s / steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32 (bf16 inputs)", "data": "synthetic",
            "impl": "reference",
            "config": workload_config(w, args.quantiser, args.gpus),
            "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
                             "sample": desc + f"; {per_step:.2f} s per step", "build": CPU_BUILD},
            "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
