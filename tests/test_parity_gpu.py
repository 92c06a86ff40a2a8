"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (stated for the merged output): max-abs 2e-2 and relative L2
1e-2; membership tables bit-exact.  Branch outputs read through the debug
modes use the same relative-L2 bound and a max-abs bound scaled by the
branch's own magnitude.  Exported forward/backward states: relative L2
1e-2 (phi(k) is rounded to bf16 for the tensor cores, a relative error of
2^-9 per term).

Small shapes are checked element by element over the whole output; the
workload shapes too large for the host oracle are checked on sampled rows
(chunk edges, ragged tile tails, random rows) of sampled heads, computed by
the oracle one row set at a time.
"""
import numpy as np
import pytest
import torch

from oracle import hybrid_attn as O
from video_diffusion_hybrid_sparse_b200 import binding as vb
from video_diffusion_hybrid_sparse_b200.workloads import BY_NAME, Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL_ABS, TOL_REL = 2e-2, 1e-2
NAMES = ["q", "k", "v", "text_k", "text_v", "gate_s", "gate_l"]


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def assert_close(got, ref, what, abs_tol=TOL_ABS, rel_tol=TOL_REL):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    i = np.unravel_index(np.argmax(err), err.shape)
    r = rel_l2(got, ref)
    # one line per comparison (shown with pytest -s): the accuracy record
    print(f"ACCURACY {what}: max-abs {err[i]:.2e} at {tuple(int(x) for x in i)}, rel-L2 {r:.2e}, "
          f"max|ref| {np.abs(ref).max():.3g}")
    assert err[i] <= abs_tol, f"{what}: max-abs {err[i]:.3e} at {i} (got {got[i]}, ref {ref[i]})"
    assert r <= rel_tol, f"{what}: rel-L2 {r:.3e}"


def to_dev(inputs):
    return {k: t.cuda() for k, t in inputs.items()}


def run(w: Workload, dev, **kw):
    out = vb.hybrid_attn_fwd(dev["q"], dev["k"], dev["v"], dev["text_k"], dev["text_v"], dev["gate_s"],
                             dev["gate_l"], frames=w.F, chunk_frames=w.C, **kw)
    torch.cuda.synchronize()
    return out


def np64(t):
    return t.to(torch.float64).cpu().numpy()


def oracle_full(w: Workload, inputs, gamma=None, mode="local"):
    x = {k: np64(t) for k, t in inputs.items()}
    prob = O.Problem(B=w.B, F=w.F, P=w.P, H=w.H, d=w.d, T=w.T, C=w.C, anchor_query_mode=mode)
    return O.hybrid_attn(x["q"], x["k"], x["v"], x["text_k"], x["text_v"], x["gate_s"], x["gate_l"], prob,
                         gamma=gamma)


# ----------------------------------------------------------------- membership


@pytest.mark.parametrize("F,C,P,T", [(15, 1, 16, 8), (45, 5, 4, 3), (60, 5, 3, 0), (1, 1, 5, 2), (2, 1, 5, 2),
                                     (3, 1, 5, 0), (6, 6, 2, 1), (12, 3, 2, 2), (96, 1, 1, 1)])
def test_device_membership_matches_oracle(F, C, P, T):
    np.testing.assert_array_equal(vb.membership_device(F, C, P, T), O.membership_table(F, C))


# ----------------------------------------------------------------- whole outputs, small shapes


SMALL = [
    BY_NAME["tiny_fp32"],
    BY_NAME["small_bf16"],
    # ragged frames (P not a multiple of 128), two batches, text not a multiple of 128
    Workload("ragged", 2, 15, 200, 2, 128, 70, 1, "bf16", "normal", 11),
    Workload("c5_ragged", 1, 10, 130, 2, 128, 40, 5, "bf16", "half", 12),
    Workload("one_frame", 1, 1, 150, 2, 64, 20, 1, "bf16", "normal", 13),
    Workload("two_frames", 1, 2, 100, 2, 64, 9, 1, "bf16", "normal", 14),
    Workload("three_frames_no_text", 1, 3, 90, 2, 128, 0, 1, "bf16", "normal", 15),
    Workload("one_chunk", 1, 6, 64, 2, 128, 33, 6, "bf16", "normal", 16),
    Workload("two_chunks_no_text", 1, 4, 64, 1, 64, 0, 2, "bf16", "normal", 17),
    Workload("d32_bf16", 1, 15, 40, 3, 32, 5, 1, "bf16", "normal", 18),
    Workload("d64_fp32", 1, 9, 50, 2, 64, 7, 3, "fp32", "normal", 19),
    Workload("d128_fp32", 1, 5, 300, 1, 128, 130, 1, "fp32", "rms", 20),
    Workload("tiny_tokens", 1, 7, 1, 2, 64, 1, 1, "bf16", "normal", 21),
    # the most chunks the scan keeps on chip (96), one-frame chunks
    Workload("max_chunks", 1, 96, 4, 1, 64, 3, 1, "bf16", "normal", 23),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_full_output_matches_oracle(w):
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    ref = oracle_full(w, inputs)
    out = run(w, dev)
    assert_close(out.float().cpu().numpy(), ref["out"], f"{w.name} out")


@pytest.mark.parametrize("w", SMALL[:4], ids=[w.name for w in SMALL[:4]])
def test_branches_match_oracle(w):
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    ref = oracle_full(w, inputs)
    o_s = run(w, dev, debug_flags=vb.OUT_SOFTMAX_ONLY).float().cpu().numpy()
    assert_close(o_s, ref["o_s"], f"{w.name} o_s")
    r = run(w, dev, debug_flags=vb.OUT_LINEAR_ONLY).float().cpu().numpy()
    assert_close(r, ref["r"], f"{w.name} r", abs_tol=3e-2)
    o_l = run(w, dev, debug_flags=vb.OUT_LINEAR_RAW).float().cpu().numpy()
    scale = np.abs(ref["o_l"]).max()
    assert_close(o_l, ref["o_l"], f"{w.name} o_l", abs_tol=TOL_ABS * scale)


# ----------------------------------------------------------------- GLOBAL anchor queries, SPLIT output


GLOBAL_CASES = [SMALL[i] for i in (0, 2, 3, 4, 5, 7, 9, 10, 12, 13)] + [
    Workload("global_b2_c3", 2, 12, 100, 2, 128, 20, 3, "bf16", "normal", 22)]


@pytest.mark.parametrize("F,C,P,T", [(15, 1, 16, 8), (45, 5, 4, 3), (1, 1, 5, 2), (2, 1, 5, 2), (6, 6, 2, 1),
                                     (12, 3, 2, 2)])
def test_device_membership_global_matches_oracle(F, C, P, T):
    np.testing.assert_array_equal(vb.membership_device(F, C, P, T, anchor_query_mode=vb.ANCHOR_GLOBAL),
                                  O.membership_table(F, C, "global"))


@pytest.mark.parametrize("w", GLOBAL_CASES, ids=[w.name for w in GLOBAL_CASES])
def test_global_anchor_mode_matches_oracle(w):
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    ref = oracle_full(w, inputs, mode="global")
    out = run(w, dev, anchor_query_mode=vb.ANCHOR_GLOBAL)
    assert_close(out.float().cpu().numpy(), ref["out"], f"{w.name} out (GLOBAL)")
    o_s = run(w, dev, anchor_query_mode=vb.ANCHOR_GLOBAL, debug_flags=vb.OUT_SOFTMAX_ONLY)
    assert_close(o_s.float().cpu().numpy(), ref["o_s"], f"{w.name} o_s (GLOBAL)")


@pytest.mark.parametrize("w", [SMALL[0], SMALL[1], SMALL[3], SMALL[9]], ids=["tiny", "small", "c5_ragged", "d32"])
def test_split_output_matches_oracle(w):
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    ref = oracle_full(w, inputs)
    out_lin = torch.empty_like(dev["q"])
    out = run(w, dev, out_linear=out_lin)
    assert_close(out.float().cpu().numpy(), ref["out_s"], f"{w.name} sigmoid(g_s) o_s")
    assert_close(out_lin.float().cpu().numpy(), ref["out_l"], f"{w.name} sigmoid(g_l) r")
    merged = run(w, dev).float()
    # the two stored terms add up to the merged output up to one rounding of each
    assert_close((out.float() + out_lin.float()).cpu().numpy(), merged.cpu().numpy(), f"{w.name} split sum")


@pytest.mark.parametrize("w,mode,split", [(SMALL[0], 0, False), (SMALL[1], 0, False), (SMALL[3], 1, False),
                                          (SMALL[2], 0, True), (SMALL[2], 0, False)],
                         ids=["tiny", "small", "c5_global", "ragged_split", "ragged"])
def test_host_tensor_call_matches_device_call_and_oracle(w, mode, split):
    """vdn_hybrid_attn_fwd_host (pinned host tensors, copies overlapped with
    the kernels) against the oracle at the parity tolerance, and against the
    device call.  The two calls differ only in where the softmax branch's gate
    is applied (the host call leaves it to the readout, so that the softmax
    kernel runs while the gates are still being copied): one bf16 rounding of
    the gated term, so the outputs agree within two bf16 steps.  The second
    output of SPLIT (the linear term) is the same bit for bit."""
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    ref_lin = torch.empty_like(dev["q"]) if split else None
    ref = run(w, dev, anchor_query_mode=mode, out_linear=ref_lin)
    host = {k: t.pin_memory() for k, t in inputs.items()}
    out_lin = torch.empty(host["q"].shape, dtype=host["q"].dtype, pin_memory=True) if split else None
    out = vb.hybrid_attn_fwd_host(host["q"], host["k"], host["v"], host["text_k"], host["text_v"], host["gate_s"],
                                  host["gate_l"], frames=w.F, chunk_frames=w.C, anchor_query_mode=mode,
                                  out_linear=out_lin)
    torch.cuda.synchronize()
    orc = oracle_full(w, inputs, mode="global" if mode else "local")
    assert_close(out.float().numpy(), orc["out_s"] if split else orc["out"], f"{w.name} host call")
    # the two differ by one more bf16 rounding (relative 2^-9) of sigmoid(g_s) * o_s,
    # |o_s| <= max |v|, and by the output's own rounding: at most three half-steps
    # relative to the value (2^-7 in rel-L2), plus that absolute bound for values
    # that cancel
    assert_close(out.float().numpy(), ref.cpu().float().numpy(), f"{w.name} host vs device call",
                 abs_tol=2.0 ** -9 * 2 * float(inputs["v"].float().abs().max()) + 2.0 ** -8 * 8, rel_tol=2.0 ** -7)
    if split:
        assert torch.equal(out_lin, ref_lin.cpu())


def test_host_calls_in_flight_on_two_streams():
    """Host-tensor calls with two in flight, as bench.py's end-to-end number
    runs them: call i on stream i % 2 with its own staging buffer, workspace
    and host output, all enqueued before any synchronisation.  Each call's
    output must equal the same call made alone, bit for bit, whatever the
    overlap of one call's copies and kernels with the other's."""
    calls = [BY_NAME["small_bf16"], SMALL[2], BY_NAME["small_bf16"], SMALL[2]]
    hosts, alone = [], []
    for w in calls:
        inputs = make_inputs(w)
        host = {k: t.pin_memory() for k, t in inputs.items()}
        hosts.append(host)
        ref = vb.hybrid_attn_fwd_host(host["q"], host["k"], host["v"], host["text_k"], host["text_v"],
                                      host["gate_s"], host["gate_l"], frames=w.F, chunk_frames=w.C)
        torch.cuda.synchronize()
        alone.append(ref.clone())
    streams = [torch.cuda.current_stream(), torch.cuda.Stream()]
    outs = []
    for i, (w, host) in enumerate(zip(calls, hosts)):
        s = vb.shape_of(host["q"], host["text_k"], w.F, w.C)
        stg, ws = vb.new_staging(s, "cuda"), vb.new_workspace(s, "cuda")
        out = torch.empty(host["q"].shape, dtype=host["q"].dtype, pin_memory=True)
        vb.hybrid_attn_fwd_host(host["q"], host["k"], host["v"], host["text_k"], host["text_v"], host["gate_s"],
                                host["gate_l"], frames=w.F, chunk_frames=w.C, out=out, workspace=ws, staging=stg,
                                stream=streams[i % 2])
        outs.append((out, stg, ws))
    torch.cuda.synchronize()
    for i, (out, _, _) in enumerate(outs):
        assert torch.equal(out, alone[i]), f"call {i}"


# Exported forward/backward states against the oracle's, relative L2.  The
# states are fp32 sums of phi(k) v^T with phi(k) rounded to bf16 for the
# tensor cores (relative rounding <= 2^-9, about 1.1e-3 RMS per term,
# unbiased, independent across terms), so the relative error of a state
# whose terms have random signs is about 1.1e-3, and states of few tokens
# scatter around that: measured up to 1.3e-3 on the frame states and up to
# 2.1e-3 on the 40- to 70-token text states of the bf16 shapes; bound 3e-3.
# fp32 inputs are first rounded to bf16 themselves (k and v), three
# roundings per term, about 1.9e-3 RMS: measured 2.6e-3 on the 8-token text
# state of the fp32 shape; bound 4e-3.
STATE_TOL = 3e-3
STATE_TOL_FP32 = 4e-3


@pytest.mark.parametrize("w", [SMALL[0], SMALL[2], SMALL[3], SMALL[1]], ids=["tiny", "ragged", "c5_ragged", "small"])
def test_exported_states_match_oracle(w):
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    ref = oracle_full(w, inputs)
    nc = w.F // w.C
    fwd = torch.zeros((w.B, nc, w.H, w.d + 1, w.d), dtype=torch.float32, device="cuda")
    bwd = torch.zeros_like(fwd)
    run(w, dev, debug_flags=vb.EXPORT_STATES, export=(fwd, bwd))
    fwd, bwd = fwd.cpu().numpy(), bwd.cpu().numpy()
    tol = STATE_TOL_FP32 if w.dtype == "fp32" else STATE_TOL
    worst = 0.0
    for b in range(w.B):
        for h in range(w.H):
            st = ref["states"][(b, h)]
            # exported layout: row a' < d holds S[:, a'] (value column a'), row d holds z
            ref_f = np.concatenate([st["SF"].transpose(0, 2, 1), st["zF"][:, None, :]], axis=1)
            ref_b = np.concatenate([st["SB"].transpose(0, 2, 1), st["zB"][:, None, :]], axis=1)
            ef, eb = rel_l2(fwd[b, :, h], ref_f), rel_l2(bwd[b, :, h], ref_b)
            worst = max(worst, ef, eb)
            assert ef <= tol and eb <= tol, (b, h, ef, eb)
            if w.T > 0:  # chunk 0's forward state holds nothing but half of the text state
                et = rel_l2(fwd[b, 0, h, :w.d, :], 0.5 * st["S_t"].T)
                worst = max(worst, et)
                assert et <= tol, (b, h, et)
            # the states that hold no video frame are the same half text state, bit for bit:
            # forward of chunks 0 and 1, backward of the last two chunks
            half_t = fwd[b, 0, h]
            for c in range(min(2, nc)):
                assert np.array_equal(fwd[b, c, h], half_t), f"forward state of chunk {c} holds video"
                assert np.array_equal(bwd[b, nc - 1 - c, h], half_t), f"backward state of chunk {nc - 1 - c} holds video"
    print(f"{w.name}: worst state rel-L2 {worst:.2e}")


def test_rms_weight_gamma():
    w = SMALL[2]
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    gamma = torch.rand((w.H, w.d), generator=torch.Generator("cpu").manual_seed(5)) + 0.5
    ref = oracle_full(w, inputs, gamma=gamma.double().numpy())
    out = run(w, dev, rms_weight=gamma.cuda())
    assert_close(out.float().cpu().numpy(), ref["out"], "gamma out")


def test_steps_equal_whole_call_and_deterministic():
    w = BY_NAME["small_bf16"]
    dev = to_dev(make_inputs(w))
    a = run(w, dev).clone()
    b = run(w, dev).clone()
    assert torch.equal(a, b), "two calls differ"
    out = torch.empty_like(dev["q"])
    steps = vb.Steps(dev["q"], dev["k"], dev["v"], dev["text_k"], dev["text_v"], dev["gate_s"], dev["gate_l"], out,
                     frames=w.F, chunk_frames=w.C)
    steps.all()
    torch.cuda.synchronize()
    assert torch.equal(out, a)


@pytest.mark.parametrize("w,mode", [(BY_NAME["small_bf16"], 0), (SMALL[3], 0), (SMALL[3], 1), (SMALL[0], 0),
                                    (SMALL[9], 0)], ids=["small", "c5_ragged", "c5_ragged_global", "tiny_fp32", "d32"])
def test_scan_inside_softmax_equals_separate_scan(w, mode):
    """The forward/backward scan run by the softmax kernel's idle warps and the
    scan launched on its own write the same readout operands: the outputs of
    the two step sequences are bit-identical."""
    dev = to_dev(make_inputs(w))
    outs = []
    for seq in ("fused_scan", "all_separate"):
        out = torch.full_like(dev["q"], float("nan"))
        steps = vb.Steps(dev["q"], dev["k"], dev["v"], dev["text_k"], dev["text_v"], dev["gate_s"], dev["gate_l"],
                         out, frames=w.F, chunk_frames=w.C, anchor_query_mode=mode,
                         workspace=torch.empty(vb.workspace_bytes(vb.shape_of(dev["q"], dev["text_k"], w.F, w.C)),
                                               dtype=torch.uint8, device="cuda"))
        if seq == "fused_scan":  # the softmax leaves o_s ungated, as vdn_sparse_softmax does
            steps.stage()
            steps.state_build()
            steps.softmax_and_scan(gate=False)
            steps.readout_merge()
        else:
            steps.all_separate()
        torch.cuda.synchronize()
        outs.append(out)
    word = torch.int32 if outs[0].dtype == torch.float32 else torch.int16
    assert torch.equal(outs[0].view(word), outs[1].view(word))


def test_status_word_stays_clear():
    w = SMALL[2]
    dev = to_dev(make_inputs(w))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    run(w, dev, status=status)
    assert int(status.item()) == 0


# ----------------------------------------------------------------- workload shapes, sampled rows


def sample_rows(w: Workload, rng, n_random=24):
    rpc = w.C * w.P
    rows = set()
    for c in range(w.F // w.C):
        base = c * rpc
        rows.update({base, base + rpc - 1})
        last_tile = (rpc - 1) // 128 * 128
        rows.update({base + last_tile, base + min(rpc - 1, last_tile + 1)})
    rows.update(rng.integers(0, w.N, n_random).tolist())
    return np.array(sorted(rows))


@pytest.mark.parametrize("name,heads", [("chunk5_bf16", [0, 7, 15]), ("768p_bf16", [0, 4, 9, 14, 19, 23]),
                                        ("768p_long_bf16", [0, 7, 23])])
def test_workload_sampled_rows(name, heads):
    w = BY_NAME[name]
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    ws = vb.workspace_for(vb.shape_of(dev["q"], dev["text_k"], w.F, w.C), dev["q"].device)
    vb.clear_timeout_record(ws)
    status1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run(w, dev, status=status1, workspace=ws)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out2 = run(w, dev, status=status, workspace=ws)
    assert int(status1.item()) == 0 and int(status.item()) == 0, \
        f"a bounded wait ran out: statuses {int(status1.item())}, {int(status.item())}; {vb.timeout_record(ws)}"
    same = out.view(torch.int16) == out2.view(torch.int16)
    if not bool(same.all()):
        bad = (~same).nonzero()
        f1, f2 = out.float(), out2.float()
        raise AssertionError(
            f"{name}: two calls differ in {bad.shape[0]} elements (first at {bad[0].tolist()}: "
            f"{f1[tuple(bad[0])].item()} vs {f2[tuple(bad[0])].item()}; rows {bad[:, 1].unique().numel()}, "
            f"heads {bad[:, 2].unique().tolist()[:8]}; non-finite {int((~torch.isfinite(f1)).sum())} / "
            f"{int((~torch.isfinite(f2)).sum())})")
    del dev
    rng = np.random.default_rng(7)
    rows = sample_rows(w, rng)
    prob = O.Problem(B=1, F=w.F, P=w.P, H=1, d=w.d, T=w.T, C=w.C)
    for h in heads:
        x = {k: np64(t[:, :, h:h + 1, :]) for k, t in inputs.items()}
        ref = O.hybrid_attn_rows(x["q"], x["k"], x["v"], x["text_k"], x["text_v"], x["gate_s"], x["gate_l"],
                                 prob, 0, 0, rows)
        got = out[0, torch.from_numpy(rows).cuda(), h, :].float().cpu().numpy()
        assert_close(got, ref["out"], f"{name} head {h}")


def test_global_anchor_mode_sampled_rows_768p():
    """GLOBAL at the 768p shape: anchor rows attend to all 60,480 video keys
    plus text; sampled rows of both anchor frames and of inner frames."""
    w = BY_NAME["768p_bf16"]
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    out = run(w, dev, anchor_query_mode=vb.ANCHOR_GLOBAL)
    del dev
    rng = np.random.default_rng(11)
    last = (w.F - 1) * w.P
    rows = np.unique(np.concatenate([[0, 127, 128, 4031, last, last + 127, last + 128, w.N - 1],
                                     rng.integers(0, w.P, 6), last + rng.integers(0, w.P, 6),
                                     rng.integers(w.P, last, 6)]))
    prob = O.Problem(B=1, F=w.F, P=w.P, H=1, d=w.d, T=w.T, C=w.C, anchor_query_mode="global")
    for h in (0, 17):
        x = {k: np64(t[:, :, h:h + 1, :]) for k, t in inputs.items()}
        ref = O.hybrid_attn_rows(x["q"], x["k"], x["v"], x["text_k"], x["text_v"], x["gate_s"], x["gate_l"],
                                 prob, 0, 0, rows)
        got = out[0, torch.from_numpy(rows).cuda(), h, :].float().cpu().numpy()
        assert_close(got, ref["out"], f"768p GLOBAL head {h}")


# ----------------------------------------------------------------- failure path


@pytest.mark.parametrize("w", [SMALL[0], Workload("inject_8tiles", 1, 6, 1024, 1, 64, 8, 1, "bf16", "normal", 24)],
                         ids=["tiny", "eight_tiles"])
def test_injected_timeout_reports_status_and_context_survives(w):
    """A wait that nothing completes (VDN_INJECT_TIMEOUT: one CTA of the
    state build, 10-ms limit) ends with VDN_ERR_TIMEOUT in the status word
    instead of a hang or a fault, the timeout record names that wait, and the
    next call is correct."""
    import time
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    ws = vb.workspace_for(vb.shape_of(dev["q"], dev["text_k"], w.F, w.C), dev["q"].device)
    vb.clear_timeout_record(ws)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    run(w, dev, debug_flags=vb.INJECT_TIMEOUT, status=status, workspace=ws)
    assert time.time() - t0 < 30
    assert int(status.item()) == 6
    rec = vb.timeout_record(ws)
    assert rec["timeouts"] >= 1 and rec["kernel"] == 1 and rec["block"] == 0, rec
    assert 10_000_000 <= rec["ns"] < 1_000_000_000, rec
    vb.clear_timeout_record(ws)
    status.zero_()
    out = run(w, dev, status=status)
    assert int(status.item()) == 0
    assert_close(out.float().cpu().numpy(), oracle_full(w, inputs)["out"], f"{w.name} after the injected timeout")


# The readout's MMA thread held up at every readout-operand change: the other
# warps run as far ahead as the barrier protocol allows (in the TMA-fed
# readout they once completed two phases of the phi-ready barrier before the
# MMA thread waited on the first, which then waited on a third for good).
# 37 heads put four CTAs on each head; with eight 128-row tiles per chunk each
# CTA takes two tiles of every (batch, chunk), so the MMA thread stalls at the
# first while the loads of the second need no new operand.  Outputs must be
# bit-identical to an unstalled call.
STALL_CASES = [Workload("stall_bf16", 1, 4, 1024, 37, 128, 16, 1, "bf16", "normal", 28),
               Workload("stall_fp32", 1, 4, 1024, 37, 32, 16, 1, "fp32", "normal", 29)]


@pytest.mark.parametrize("w", STALL_CASES, ids=[w.name for w in STALL_CASES])
def test_readout_protocol_survives_stalled_mma_thread(w):
    dev = to_dev(make_inputs(w))
    ws = vb.workspace_for(vb.shape_of(dev["q"], dev["text_k"], w.F, w.C), dev["q"].device)
    vb.clear_timeout_record(ws)
    st0 = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = run(w, dev, status=st0, workspace=ws)
    st1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run(w, dev, status=st1, workspace=ws, debug_flags=vb.STALL_READOUT_MMA)
    assert int(st0.item()) == 0 and int(st1.item()) == 0, vb.timeout_record(ws)
    assert torch.equal(ref.view(torch.int16) if ref.dtype == torch.bfloat16 else ref.view(torch.int32),
                       out.view(torch.int16) if out.dtype == torch.bfloat16 else out.view(torch.int32))


# ----------------------------------------------------------------- fp8 softmax branch
#
# Tolerance for softmax_precision = FP8, derived from e4m3: three mantissa
# bits, so a rounded operand is off by at most 2^-4 of its value (RMS
# 2^-4 / sqrt(3) ~ 3.6 %).  Each term of o_s = sum p v / sum p carries the
# rounding of v, of p, and the perturbation of p by the rounding of q and k in
# the logit (~5 % RMS for unit-RMS rows at head_dim 128): ~7 % RMS per term,
# independent across keys, so o_s keeps a relative error of that order:
# rel-L2 <= 0.1 for o_s.  The merged output is dominated by the linear branch
# and the gates: rel-L2 <= 1e-2 as for bf16, and max-abs <= 4e-2 (the bf16
# output rounding, up to 1.6e-2, plus sigmoid(g_s) times the o_s error).

FP8_CASES = [Workload("fp8_rms", 1, 6, 256, 2, 128, 32, 1, "bf16", "rms", 25),
             Workload("fp8_c3", 1, 9, 96, 2, 128, 40, 3, "bf16", "normal", 26),
             Workload("fp8_b2_no_text", 2, 4, 128, 1, 128, 0, 1, "bf16", "half", 27)]


@pytest.mark.parametrize("w", FP8_CASES, ids=[w.name for w in FP8_CASES])
def test_fp8_softmax_matches_oracle(w):
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    ref = oracle_full(w, inputs)
    out = run(w, dev, softmax_precision=vb.PREC_FP8)
    assert_close(out.float().cpu().numpy(), ref["out"], f"{w.name} out (fp8)", abs_tol=4e-2, rel_tol=1e-2)
    o_s = run(w, dev, softmax_precision=vb.PREC_FP8, debug_flags=vb.OUT_SOFTMAX_ONLY)
    scale = np.abs(ref["o_s"]).max()
    assert_close(o_s.float().cpu().numpy(), ref["o_s"], f"{w.name} o_s (fp8)", abs_tol=0.25 * scale, rel_tol=0.1)
    again = run(w, dev, softmax_precision=vb.PREC_FP8)
    assert torch.equal(out, again)


def test_fp8_global_anchor_mode():
    w = FP8_CASES[1]
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    ref = oracle_full(w, inputs, mode="global")
    out = run(w, dev, softmax_precision=vb.PREC_FP8, anchor_query_mode=vb.ANCHOR_GLOBAL)
    assert_close(out.float().cpu().numpy(), ref["out"], f"{w.name} out (fp8, GLOBAL)", abs_tol=4e-2, rel_tol=1e-2)


def test_fp8_rejects_unsupported_shapes():
    w = SMALL[3]  # c5_ragged: 130 tokens per frame, not a multiple of 16
    dev = to_dev(make_inputs(w))
    with pytest.raises(vb.VdnError) as e:
        run(w, dev, softmax_precision=vb.PREC_FP8)
    assert e.value.code == 2


def test_fp8_768p_sampled_rows():
    w = BY_NAME["768p_bf16"]
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    out = run(w, dev, softmax_precision=vb.PREC_FP8)
    del dev
    rows = sample_rows(w, np.random.default_rng(7))
    prob = O.Problem(B=1, F=w.F, P=w.P, H=1, d=w.d, T=w.T, C=w.C)
    for h in (0, 23):
        x = {k: np64(t[:, :, h:h + 1, :]) for k, t in inputs.items()}
        ref = O.hybrid_attn_rows(x["q"], x["k"], x["v"], x["text_k"], x["text_v"], x["gate_s"], x["gate_l"],
                                 prob, 0, 0, rows)
        got = out[0, torch.from_numpy(rows).cuda(), h, :].float().cpu().numpy()
        assert_close(got, ref["out"], f"768p fp8 head {h}", abs_tol=4e-2, rel_tol=1e-2)


# ----------------------------------------------------------------- workspace poison, state export after a call
#
# VDN_POISON_WS fills the workspace past its status slot with 0xFF (NaN in
# bf16 and fp32) before the call: an output that differs from an unpoisoned
# call on the same workspace would mean that some kernel read scratch the call
# had not written.


@pytest.mark.parametrize("w,prec", [(SMALL[0], vb.PREC_BF16), (SMALL[2], vb.PREC_BF16), (SMALL[3], vb.PREC_BF16),
                                    (FP8_CASES[0], vb.PREC_FP8), (FP8_CASES[2], vb.PREC_FP8)],
                         ids=["tiny_fp32", "ragged_b2", "c5_ragged", "fp8_rms", "fp8_b2_no_text"])
def test_poisoned_workspace_changes_nothing(w, prec):
    dev = to_dev(make_inputs(w))
    ws = vb.workspace_for(vb.shape_of(dev["q"], dev["text_k"], w.F, w.C), dev["q"].device, prec)
    st0 = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = run(w, dev, status=st0, workspace=ws, softmax_precision=prec)
    st1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run(w, dev, status=st1, workspace=ws, softmax_precision=prec, debug_flags=vb.POISON_WS)
    assert int(st0.item()) == 0 and int(st1.item()) == 0
    word = torch.int32 if out.dtype == torch.float32 else torch.int16
    assert torch.equal(ref.view(word), out.view(word))


@pytest.mark.parametrize("w", [SMALL[0], SMALL[3]], ids=["tiny", "c5_ragged"])
def test_export_states_after_a_call_equals_export_during_it(w):
    dev = to_dev(make_inputs(w))
    ws = vb.workspace_for(vb.shape_of(dev["q"], dev["text_k"], w.F, w.C), dev["q"].device)
    nc = w.F // w.C
    fwd = torch.zeros((w.B, nc, w.H, w.d + 1, w.d), dtype=torch.float32, device="cuda")
    bwd = torch.zeros_like(fwd)
    run(w, dev, workspace=ws, debug_flags=vb.EXPORT_STATES, export=(fwd, bwd))
    run(w, dev, workspace=ws)
    fwd2, bwd2 = torch.full_like(fwd, float("nan")), torch.full_like(bwd, float("nan"))
    vb.export_states(vb.shape_of(dev["q"], dev["text_k"], w.F, w.C), ws, fwd2, bwd2)
    torch.cuda.synchronize()
    assert torch.equal(fwd, fwd2) and torch.equal(bwd, bwd2)
