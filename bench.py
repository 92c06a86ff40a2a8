"""Benchmark of the VDN-H3 hybrid attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 768p_bf16] [--impl ours|reference]

A step is one whole hybrid-attention call (staging when needed, state build,
sparse softmax with the forward/backward scan in the same kernel, readout +
merge) on one batch of seeded synthetic inputs already resident in HBM.  Each step's kernels are launched through the
library's per-step C-ABI entry points with a CUDA event after each one, on the
launching stream, so the dominant kernel's time is measured live.  The inputs
of one call (1.9 GB at 768p) are larger than L2, so no flush is needed.

Multi-GPU: the path runs on one GPU; under torchrun every rank runs an
independent replica of the same workload (no data-path collective) and the
timing is the max over ranks.

``--impl reference`` times the fp64 CPU oracle (the method's definition) on
the host cores: each step is one pass over a bounded sample of one call of the
same workload (the whole call for the small workloads), and the value is the
sample's algorithmic FLOPs over its measured time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from video_diffusion_hybrid_sparse_b200.workloads import BY_NAME, make_inputs  # noqa: E402

METRIC = "hybrid-attn ms/call & TFLOP/s at 768p-shaped latent, 1×B200, % of roofline"
SPEC_TFLOPS, SPEC_GBS = 2250.0, 8000.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Steps timed separately (CUDA events between them), with the Steps method
# that runs each.  The forward/backward scan runs inside the softmax kernel
# (its otherwise idle warps) on both paths; the readout and merge run in a
# kernel of their own (separate) or in the softmax kernel's epilogue (fused).
KERNELS = [("stage", "stage"), ("state_build", "state_build"), ("sparse_softmax", "softmax_and_scan"),
           ("readout_merge", "readout_merge")]
KERNELS_FUSED = [("stage", "stage"), ("state_build", "state_build"), ("sparse_softmax", "softmax_merge")]


# ---------------------------------------------------------------- algorithmic work


def softmax_key_frames(c, F, C):
    n_chunks = F // C
    win = set(range(max(0, c - 1) * C, (min(n_chunks - 1, c + 1) + 1) * C))
    return win | {0, F - 1}


def work(w, fp8: bool = False, fused: bool = False):
    """Algorithmic FLOPs and bytes per call (counts only what the method must do);
    fp8: the e4m3 softmax path (its softmax kernel does not apply the gate);
    fused: the readout and merge run in the softmax kernel (k3f_bytes)."""
    e = 2 if w.dtype == "bf16" else 4
    n_chunks, anchors = w.F // w.C, len({0, w.F - 1})
    pairs = sum(w.C * w.P * (w.P * len(softmax_key_frames(c, w.F, w.C)) + w.T) for c in range(n_chunks))
    softmax_flops = 4.0 * w.d * w.H * w.B * pairs
    linear_flops = 2.0 * w.d * (w.d + 1) * w.H * w.B * (w.P * (w.F - anchors) + w.T + w.N)
    state = w.B * w.H * w.d * (w.d + 1) * 4
    k1 = 2 * (w.P * (w.F - anchors) + w.T) * w.B * w.H * w.d * e + (w.F - anchors + 1) * state
    k2 = (w.F - anchors + 1) * state + n_chunks * state
    # on the bf16 path with head_dim 64 or 128 the softmax kernel applies the
    # softmax branch's gate: it reads g_s, and the readout reads q, the gated
    # term and g_l and writes out (four tensors instead of five)
    gated = w.dtype == "bf16" and w.d in (64, 128) and not fp8
    k4 = (4 if gated else 5) * w.B * w.N * w.H * w.d * e + n_chunks * state
    k3_bytes = ((3 + (1 if gated else 0)) * w.B * w.N + 2 * w.B * w.T) * w.H * w.d * e + w.B * w.N * w.H * w.d * 2
    # fused: q, k, v, text, g_s and g_l read, M_c read once per (batch,
    # chunk, head), out written, and the scan that runs inside
    k3f_bytes = ((5 * w.B * w.N + 2 * w.B * w.T) * w.H * w.d + w.B * w.N * w.H * w.d) * e + n_chunks * state + k2
    if fused:
        return dict(softmax_flops=softmax_flops, linear_flops=linear_flops, k1_bytes=k1, k2_bytes=k2, k4_bytes=0,
                    k3_bytes=k3f_bytes, linear_bytes=k1 + (k3f_bytes - k3_bytes))
    return dict(softmax_flops=softmax_flops, linear_flops=linear_flops, k1_bytes=k1, k2_bytes=k2, k4_bytes=k4,
                k3_bytes=k3_bytes, linear_bytes=k1 + k2 + k4)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return p, "measured"
    return FALLBACK, "fallback"


# ---------------------------------------------------------------- clocks


class ClockSampler:
    """SM clock and clock-event reasons sampled every 10 ms while the timed
    region runs (NVML, read-only queries), so that a region of a few hundred
    milliseconds still yields dozens of samples.  Falls back to nvidia-smi at
    its 200-ms floor when NVML cannot be loaded."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}
    SMI_FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
                  "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
                  "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id: str, period_s: float = 0.01):
        self.gpu_id, self.period = gpu_id, period_s
        self.samples, self.max_mhz, self.source = [], None, None
        self.proc = self.thread = None

    def _nvml_handle(self):
        import pynvml

        pynvml.nvmlInit()
        if self.gpu_id.isdigit():
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(int(self.gpu_id))
        return pynvml, pynvml.nvmlDeviceGetHandleByUUID(self.gpu_id)

    def __enter__(self):
        import threading

        try:
            nv, h = self._nvml_handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.stop = threading.Event()

            def loop():
                while not self.stop.is_set():
                    try:
                        self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)), int(get_reasons(h))))
                    except Exception:  # noqa: BLE001 - a failed read only loses a sample
                        pass
                    self.stop.wait(self.period)

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            self.source = "nvml, 10 ms"
        except Exception:  # noqa: BLE001 - NVML missing: nvidia-smi instead
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + ",".join(self.SMI_FIELDS),
                     "--format=csv,noheader,nounits", "-lms", "200"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.source = "nvidia-smi, 200 ms"
            except OSError:
                self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            for ln in out.splitlines():
                f = [x.strip() for x in ln.split(",")]
                if len(f) < 9:
                    continue
                try:
                    mhz, self.max_mhz = float(f[1]), float(f[2])
                except ValueError:
                    continue
                mask = 0
                for (_, bit), val in zip(self.REASONS.items(), f[5:9]):
                    if val.lower().startswith("active"):
                        mask |= bit
                self.samples.append((mhz, mask))

    def summary(self):
        sms = [m for m, _ in self.samples]
        reasons = sorted({nm for _, mask in self.samples for nm, bit in self.REASONS.items() if mask & bit})
        return {"sm_mhz": statistics.median(sms) if sms else None, "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(sms), "sampler": self.source}


def gpu_id_for(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ---------------------------------------------------------------- ncu traffic record


def _code_only(text: str) -> str:
    """C/C++/CUDA source without comments and blank space (what the compiler
    sees; a comment edit does not change the kernel)."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(name: str) -> str:
    """sha1 of the code (comments and blank space removed) of the kernel's
    source file and of the headers it is compiled with."""
    k3 = ["k3_sparse_softmax.cu", "k3_common.cuh", "phi.cuh", "scan.cuh", "sm100.cuh", "plan.h", "kernels.h"]
    files = {"sparse_softmax": k3, "sparse_softmax_fused": k3,
             "state_scan": ["k2_state_scan.cu", "scan.cuh", "sm100.cuh", "plan.h", "kernels.h"],
             "state_build": ["k1_state_build.cu", "phi.cuh", "sm100.cuh", "plan.h", "kernels.h"],
             "readout_merge": ["k4_merge_tma.cu", "k4_common.cuh", "phi.cuh", "sm100.cuh", "plan.h", "kernels.h"]}
    h = hashlib.sha1()
    for f in files[name]:
        with open(os.path.join(ROOT, "video_diffusion_hybrid_sparse_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:12]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel (lines: kernel workload bytes source_hash)."""
    path = os.path.join(ROOT, "profiles", "ncu_dram_traffic.txt")
    if not os.path.exists(path):
        return None
    cur = kernel_source_hash(kernel)
    with open(path) as fh:
        for ln in fh:
            f = ln.split()
            if len(f) >= 4 and not ln.startswith("#") and f[0] == kernel and f[1] == workload and f[3] == cur:
                return float(f[2])
    return None


# ---------------------------------------------------------------- CPU baseline (oracle)

# Workloads small enough for the whole oracle call to be the sample (under a
# second on the host): their CPU baseline is a full, exactly timed call.
FULL_CALL_TOKENS = 15 * 256 * 8


def sample_flops(w, heads: int, frames, with_states: bool) -> float:
    """Algorithmic FLOPs of the sampled work: for each sampled head, the frame
    and text states (if built) and, per sampled query frame, its softmax pairs
    and its linear readout -- the same counting as :func:`work`."""
    anchors = len({0, w.F - 1})
    per_head = 0.0
    if with_states:
        per_head += 2.0 * w.d * (w.d + 1) * (w.P * (w.F - anchors) + w.T)
    for f in frames:
        keys = w.P * len(softmax_key_frames(f // w.C, w.F, w.C)) + w.T
        per_head += 4.0 * w.d * w.P * keys + 2.0 * w.d * (w.d + 1) * w.P
    return per_head * heads * w.B


class OracleSample:
    """The fp64 oracle, as it stands, timed on a bounded sample of one call of
    the workload.  Small workloads: the sample is the whole call (all batches,
    heads and frames).  Large ones: batch 0, head 0 -- its frame and text
    states and the query rows of its first, middle and last frames (softmax
    rows, readout, RMSNorm, merge), about 1-3 s of host time at 768p.  The
    value is the sample's algorithmic FLOPs over its measured time; nothing
    is extrapolated into it."""

    def __init__(self, w, inputs):
        from oracle import hybrid_attn as O  # only the CPU-baseline legs import the oracle

        self.O, self.w = O, w
        self.cores = len(os.sched_getaffinity(0))
        self.full = w.N * w.H * w.B <= FULL_CALL_TOKENS
        if self.full:
            self.x = {k: t.to(torch.float64).numpy() for k, t in inputs.items()}
            self.prob = O.Problem(B=w.B, F=w.F, P=w.P, H=w.H, d=w.d, T=w.T, C=w.C)
            self.frames = list(range(w.F))
            self.flops = work(w)["softmax_flops"] + work(w)["linear_flops"]
            self.desc = "fp64 oracle, the whole call (all %d heads, all %d frames)" % (w.H, w.F)
        else:
            self.x = {k: t[0:1, :, 0:1, :].to(torch.float64).numpy() for k, t in inputs.items()}
            self.prob = O.Problem(B=1, F=w.F, P=w.P, H=1, d=w.d, T=w.T, C=w.C)
            self.frames = sorted({0, (w.F // w.C // 2) * w.C, w.F - 1})
            self.rows = np.concatenate([np.arange(f * w.P, (f + 1) * w.P) for f in self.frames])
            self.flops = sample_flops(w, 1, self.frames, True) / w.B
            self.desc = ("fp64 oracle, batch 0 head 0 of %d: frame and text states plus the query rows of frames "
                         "%s (softmax, readout, RMSNorm, merge)" % (w.H, self.frames))

    def run(self) -> float:
        """Seconds for one pass over the sample."""
        x, O = self.x, self.O
        t0 = time.perf_counter()
        if self.full:
            O.hybrid_attn(x["q"], x["k"], x["v"], x["text_k"], x["text_v"], x["gate_s"], x["gate_l"], self.prob)
        else:
            O.hybrid_attn_rows(x["q"], x["k"], x["v"], x["text_k"], x["text_v"], x["gate_s"], x["gate_l"],
                               self.prob, 0, 0, self.rows)
        return time.perf_counter() - t0

    def record(self, secs: float) -> dict:
        call = work(self.w)["softmax_flops"] + work(self.w)["linear_flops"]
        value = self.flops / secs / 1e12
        return {"value": value, "unit": "TFLOP/s", "cores": self.cores, "kind": "oracle", "sample": self.desc,
                "sample_s": secs, "sample_tflop": self.flops / 1e12,
                "ms_per_call_extrapolated": None if self.full else call / (value * 1e12) * 1e3}


def full_oracle_calls(names=("tiny_fp32", "small_bf16")) -> dict:
    """Whole oracle calls of the small workloads, each timed exactly (ms)."""
    out = {}
    for name in names:
        w = BY_NAME[name]
        s = OracleSample(w, make_inputs(w))
        out[name] = s.run() * 1e3
    return out


# ---------------------------------------------------------------- main


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank time over all ranks (NCCL on GPU, gloo on CPU)."""
    if world == 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def run_reference(args, w, world, rank):
    if rank != 0:
        return
    cb = OracleSample(w, make_inputs(w))
    secs = []
    for i in range(args.warmup + args.steps):
        t = cb.run()
        if i >= args.warmup:
            secs.append(t)
    med = statistics.median(secs)
    rec = cb.record(med)
    value = rec["value"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": med * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, world, args.precision),
        "step": "one pass of the oracle over the sample below (a bounded part of one call of the workload)",
        "cpu_baseline": rec,
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(w, world, precision="bf16"):
    c = {"workload": w.name, "B": w.B, "F": w.F, "P": w.P, "H": w.H, "d": w.d, "T": w.T, "C": w.C,
         "dtype": w.dtype, "l2": "inputs larger than L2 (no flush)", "parallelism": f"replicas x{world}"}
    if precision != "bf16":
        c["softmax_precision"] = precision
    return c


def bench_line(args, w, world, wk, per_kernel, ms, e2e_ms, h2d, d2h, launches_per_step, clocks):
    """The JSON line of our arm from the measured times (ms per call, per
    kernel, end to end)."""
    fp8 = args.precision == "fp8"
    fused = args.readout == "fused"
    flops_call = wk["softmax_flops"] + wk["linear_flops"]
    value = flops_call * world / (ms * 1e-3) / 1e12
    pk, src = peaks()
    # an e4m3 contraction takes the bf16 measured peak x the nominal fp8 / bf16 ratio (4.5 / 2.25)
    ratio = 2.0 if fp8 else 1.0
    tc_peak, hbm = pk["bf16_tflops"] * ratio, pk["hbm_gbs"]
    k3_ms = per_kernel["sparse_softmax"]
    achieved = wk["softmax_flops"] / (k3_ms * 1e-3) / 1e12
    k3_key = "sparse_softmax_fused" if fused else "sparse_softmax"
    traffic = recorded_traffic(k3_key, w.name)
    kern = {}
    hbm_steps = (("state_build", wk["k1_bytes"], "hbm"),) if fused else \
        (("state_build", wk["k1_bytes"], "hbm"), ("readout_merge", wk["k4_bytes"], "hbm"))
    for n, amount, bound in hbm_steps + (("sparse_softmax", wk["softmax_flops"], "tensor"),):
        t = per_kernel[n] * 1e-3
        if bound == "hbm":
            a = amount / t / 1e9 if t > 0 else None
            kern[n] = {"ms": per_kernel[n], "bound": "hbm", "achieved_gbs": a, "frac": a / hbm if a else None,
                       "bytes": amount, "traffic": None if fp8 else recorded_traffic(n, w.name)}
        else:
            a = amount / t / 1e12
            kern[n] = {"ms": per_kernel[n], "bound": "tensor", "achieved_tflops": a, "frac": a / tc_peak}
    kern["stage"] = {"ms": per_kernel["stage"]}
    if fused:
        kern["sparse_softmax"]["includes"] = "readout, RMSNorm and gated merge (fused epilogue)"
        kern["sparse_softmax"]["bytes"] = wk["k3_bytes"]
    kern["state_scan"] = {"ms": None, "in": "sparse_softmax (warps 2-3)", "bytes": wk["k2_bytes"]}
    roof_s = wk["softmax_flops"] / (tc_peak * 1e12) + wk["linear_bytes"] / (hbm * 1e9)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8 (e4m3 softmax operands)" if fp8 else "bf16", "data": "synthetic",
        "config": config_of(w, world, args.precision),
        "readout": args.readout,
        "roofline": {"bound": "tensor", "kernel": "sparse_softmax" + (" (incl. e4m3 quantisation)" if fp8 else "")
                     + (" (readout and merge fused)" if fused else ""),
                     "achieved": achieved, "peak": tc_peak,
                     "unit": "TFLOP/s", "frac": achieved / tc_peak, "traffic": None if fp8 else traffic,
                     "peak_source": (f"{src} bf16 burst (MEASURED_PEAKS.json)" if src == "measured" else "fallback")
                     + (" x 2 (nominal fp8 / bf16)" if fp8 else ""),
                     "frac_of_sustained": achieved / (pk.get("bf16_tflops_sustained", tc_peak) * ratio),
                     "frac_of_spec": achieved / (SPEC_TFLOPS * ratio)},
        "call_roofline": {"roofline_ms": roof_s * 1e3, "frac": roof_s * 1e3 / ms},
        "kernels": kern,
        "e2e": {"value": flops_call * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "calls_in_flight": 2, "readout": "separate",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    return line


def run_ours(args, w, world, rank, local):
    from video_diffusion_hybrid_sparse_b200 import binding as vb

    dev_t = make_inputs(w)
    dev = {k: t.cuda() for k, t in dev_t.items()}
    out = torch.empty_like(dev["q"])
    fp8 = args.precision == "fp8"
    if args.readout == "fused" and (fp8 or w.dtype != "bf16" or w.d != 128):
        args.readout = "separate"  # the fused readout is built for bf16, head_dim 128
    fused = args.readout == "fused"
    prec = vb.PREC_FP8 if fp8 else vb.PREC_BF16
    mode = vb.READOUT_FUSED if fused else vb.READOUT_SEPARATE
    steps = vb.Steps(dev["q"], dev["k"], dev["v"], dev["text_k"], dev["text_v"], dev["gate_s"], dev["gate_l"], out,
                     frames=w.F, chunk_frames=w.C, softmax_precision=prec, readout_mode=mode)
    stream = torch.cuda.current_stream()
    wk = work(w, fp8, fused)
    staged = w.dtype == "fp32" or w.d == 32
    # state build, softmax (+ scan), readout; the fused readout has no readout launch
    launches_per_step = (2 if fused else 3) + (5 if staged else 0) + (4 if fp8 and w.T > 0 else 3 if fp8 else 0)
    seq = KERNELS_FUSED if fused else KERNELS

    def one_call():
        for _, method in seq:
            getattr(steps, method)()

    for _ in range(args.warmup):
        one_call()
    torch.cuda.synchronize()

    # ------------------------------------------------ device-resident timing
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(seq) + 1)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(gpu_id_for(local)) as clk:
        for s in range(args.steps):
            ev[s][0].record(stream)
            for i, (_, method) in enumerate(seq):
                getattr(steps, method)()
                ev[s][i + 1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    per_kernel = {n: 0.0 for n, _ in seq}
    total_ms = 0.0
    for s in range(args.steps):
        total_ms += ev[s][0].elapsed_time(ev[s][-1])
        for i, (n, _) in enumerate(seq):
            per_kernel[n] += ev[s][i].elapsed_time(ev[s][i + 1]) / args.steps
    total_ms = max_over_ranks(total_ms, world)
    ms = total_ms / args.steps

    # ------------------------------------------------ end to end from pinned host memory
    host = {k: t.pin_memory() for k, t in dev_t.items()}
    host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = host_out.numel() * host_out.element_size()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(4, args.steps // 4)
    # The host calls use the separate readout whatever --readout says: there
    # the softmax kernel runs while the gates are still being copied in,
    # which the fused kernel (it reads the gates) cannot.  Two calls in flight, as a server streaming
    # requests would run them: call i on stream i % 2 with its own staging
    # buffer, workspace and host output, so the copy-out of one call overlaps
    # the copy-in of the next (the two PCIe directions); the library's copy
    # stream still takes the copies-in one call after the other.
    streams = [stream, torch.cuda.Stream()]
    stagings = [vb.new_staging(steps.s, dev["q"].device) for _ in range(2)]
    wss = [steps.ws, vb.new_workspace(steps.s, dev["q"].device, prec)]
    host_outs = [host_out, torch.empty(out.shape, dtype=out.dtype, pin_memory=True)]
    # one untimed host call first (under --readout fused, the separate
    # readout's kernels are loaded then)
    vb.hybrid_attn_fwd_host(host["q"], host["k"], host["v"], host["text_k"], host["text_v"], host["gate_s"],
                            host["gate_l"], frames=w.F, chunk_frames=w.C, out=host_outs[0], workspace=wss[0],
                            staging=stagings[0], stream=streams[0], softmax_precision=prec,
                            readout_mode=vb.READOUT_SEPARATE)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    streams[1].wait_event(e0)
    for i in range(n_e2e):
        # the C-ABI call on host tensors: copies in (overlapped with the
        # kernels that do not need them), the whole call, copy out
        k = i % 2
        vb.hybrid_attn_fwd_host(host["q"], host["k"], host["v"], host["text_k"], host["text_v"], host["gate_s"],
                                host["gate_l"], frames=w.F, chunk_frames=w.C, out=host_outs[k], workspace=wss[k],
                                staging=stagings[k], stream=streams[k], softmax_precision=prec,
                                readout_mode=vb.READOUT_SEPARATE)
    joined = torch.cuda.Event()
    joined.record(streams[1])
    stream.wait_event(joined)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / n_e2e
    del stagings, wss

    line = bench_line(args, w, world, wk, per_kernel, ms, e2e_ms, h2d, d2h, launches_per_step, clk.summary())
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = OracleSample(w, dev_t)
        rec = cb.record(min(cb.run() for _ in range(3 if cb.full else 1)))
        rec["full_call_ms"] = full_oracle_calls()
        line["cpu_baseline"] = rec
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="768p_bf16", choices=sorted(BY_NAME))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--readout", default="separate", choices=["separate", "fused"],
                    help="readout and merge in a kernel of their own, or in the softmax kernel's epilogue "
                         "(bf16, head_dim 128; separate elsewhere)")
    ap.add_argument("--precision", default="bf16", choices=["bf16", "fp8"],
                    help="operand precision of the softmax branch (bf16 is the headline)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = BY_NAME[args.workload]
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, w, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        run_ours(args, w, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
