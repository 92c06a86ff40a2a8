"""Host-side checks of bench.py: work accounting, the multi-rank timing
reduction (world_size 2 over gloo, on CPU) and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import hybrid_attn as O
from video_diffusion_hybrid_sparse_b200.workloads import BY_NAME, WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("w", WORKLOADS, ids=[w.name for w in WORKLOADS])
def test_softmax_flops_match_oracle_pair_count(w):
    prob = O.Problem(B=w.B, F=w.F, P=w.P, H=w.H, d=w.d, T=w.T, C=w.C)
    assert bench.work(w)["softmax_flops"] == 4.0 * w.d * w.H * w.B * O.softmax_pairs(prob)


def test_768p_work_figures():
    wk = bench.work(BY_NAME["768p_bf16"])
    assert abs(wk["softmax_flops"] / 1e12 - 14.164) < 0.01
    # the readout's bytes at 768p: q, sigmoid(g_s) * o_s (the softmax kernel
    # applies that gate on the bf16 path), g_l read and out written (4 x 0.3716
    # GB) plus the readout operands M_c (15 chunks x 24 heads x 128 x 129 fp32)
    assert abs(wk["k4_bytes"] / 1e9 - (4 * 0.37159 + 0.02378)) < 0.002
    # where the readout applies both gates (fp32 I/O): five tensors
    tiny = bench.work(BY_NAME["tiny_fp32"])
    w = BY_NAME["tiny_fp32"]
    assert tiny["k4_bytes"] == 5 * w.N * w.H * w.d * 4 + w.F // w.C * w.H * w.d * (w.d + 1) * 4


def test_fused_work_figures():
    """With the readout fused into the softmax kernel there is no readout
    kernel: the softmax kernel reads q, k, v, text, both gates and M_c,
    writes out (five video tensors read, one written) and runs the scan."""
    w = BY_NAME["768p_bf16"]
    sep, fus = bench.work(w), bench.work(w, fused=True)
    assert fus["k4_bytes"] == 0 and fus["softmax_flops"] == sep["softmax_flops"]
    video = w.N * w.H * w.d * 2
    assert fus["k3_bytes"] == (6 * video + 2 * w.T * w.H * w.d * 2 + 15 * w.H * w.d * (w.d + 1) * 4
                               + sep["k2_bytes"])


@pytest.mark.parametrize("name", sorted({n for n, _ in bench.KERNELS + bench.KERNELS_FUSED} - {"stage"}
                                        | {"sparse_softmax_fused"}))
def test_every_timed_kernel_has_a_source_hash(name):
    """bench.py looks up a DRAM-traffic record for every timed kernel by the
    hash of its sources; each step name must map to its files, and each
    Steps method named in the sequences must exist."""
    assert len(bench.kernel_source_hash(name)) == 12
    bench.recorded_traffic(name, "768p_bf16")
    from video_diffusion_hybrid_sparse_b200 import binding as vb
    for _, method in bench.KERNELS + bench.KERNELS_FUSED:
        assert callable(getattr(vb.Steps, method))


@pytest.mark.parametrize("readout,precision", [("separate", "bf16"), ("fused", "bf16"), ("separate", "fp8")])
def test_bench_line_from_fake_times(readout, precision):
    """The JSON line our arm prints, built from made-up kernel times: the
    contract keys, per-kernel entries of the sequence that ran, and the
    roofline of the softmax kernel (no GPU needed)."""
    import argparse
    args = argparse.Namespace(steps=20, warmup=5, precision=precision, readout=readout)
    w = BY_NAME["768p_bf16"]
    fused = readout == "fused"
    seq = bench.KERNELS_FUSED if fused else bench.KERNELS
    per_kernel = {n: {"stage": 0.005, "state_build": 0.13, "state_scan": 0.03, "sparse_softmax": 13.0,
                      "readout_merge": 0.31}[n] for n, _ in seq}
    ms = sum(per_kernel.values())
    wk = bench.work(w, precision == "fp8", fused)
    line = bench.bench_line(args, w, 1, wk, per_kernel, ms, 35.0, 10, 2, 3, {"sm_mhz": 1700.0})
    json.dumps(line)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in line
    assert set(line["kernels"]) >= {n for n, _ in seq}
    assert abs(line["roofline"]["achieved"] - 14.164e12 / 13e-3 / 1e12) < 1.0
    assert line["readout"] == readout and "readout" not in line["config"]


def _worker(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = bench.max_over_ranks(times[rank], world)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, [3.5, 7.25], out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == 7.25


def test_reference_arm_prints_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_fp32", "--steps", "3", "--warmup", "3"], capture_output=True, text=True, timeout=300,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_do_nothing():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_fp32", "--steps", "3", "--warmup", "3"], capture_output=True, text=True, timeout=120,
                       cwd=ROOT, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""
