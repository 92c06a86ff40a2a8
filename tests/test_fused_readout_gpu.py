"""GPU parity of the fused readout (VDN_READOUT_FUSED): the softmax kernel
runs the linear read, the RMSNorm and the gated merge in its item epilogue.

Same bar as the separate path (max-abs 2e-2, relative L2 1e-2 on the merged
output, against the fp64 oracle), plus: two fused calls are bit-identical,
the step-by-step and host-tensor forms equal the whole device call bit for
bit, and the fused and separate outputs differ by no more than the bf16
rounding of o_s that only the separate path makes.
"""
import numpy as np
import pytest
import torch

from oracle import hybrid_attn as O
from video_diffusion_hybrid_sparse_b200 import binding as vb
from video_diffusion_hybrid_sparse_b200.workloads import BY_NAME, Workload, make_inputs

from test_parity_gpu import assert_close, np64, oracle_full, run, sample_rows, to_dev

pytestmark = pytest.mark.gpu

FUSED = vb.READOUT_FUSED

CASES = [
    # ragged frames (P not a multiple of 128), two batches, text not a multiple of 128
    Workload("ragged", 2, 15, 200, 2, 128, 70, 1, "bf16", "normal", 11),
    # chunks of five frames, a ragged last tile per chunk
    Workload("c5_ragged", 1, 10, 130, 2, 128, 40, 5, "bf16", "half", 12),
    # the window covers everything and there is no text: o_l = 0 exactly
    Workload("three_frames_no_text", 1, 3, 90, 2, 128, 0, 1, "bf16", "normal", 15),
    # one chunk: no state at all besides the text
    Workload("one_chunk", 1, 6, 64, 2, 128, 33, 6, "bf16", "normal", 16),
    # 480 items (several per CTA), items of two and of one query tile mixed
    Workload("many_items", 1, 15, 300, 16, 128, 64, 1, "bf16", "rms", 31),
    # one frame: both anchors are frame 0
    Workload("one_frame_d128", 1, 1, 150, 2, 128, 20, 1, "bf16", "normal", 32),
    # the most chunks the scan keeps on chip (96): 96 readout operands per
    # head, every item a single tile with 4 valid rows
    Workload("max_chunks_d128", 1, 96, 4, 1, 128, 3, 1, "bf16", "normal", 33),
    # one token per frame, one text token
    Workload("tiny_tokens_d128", 1, 7, 1, 2, 128, 1, 1, "bf16", "normal", 34),
]


def fused(w, dev, **kw):
    return run(w, dev, readout_mode=FUSED, **kw)


def assert_one_rounding_apart(a, b, what, extra=4e-3):
    """|a - b| <= one bf16 ulp of the larger magnitude + extra, element by
    element: each path rounds the output to bf16 once, and the separate path
    also rounds sigmoid(g_s) o_s (a relative 2^-9, at most a few 1e-3 here)."""
    a, b = a.float(), b.float()
    m = torch.maximum(a.abs(), b.abs()).clamp_min(2.0 ** -126)
    ulp = torch.exp2(torch.floor(torch.log2(m)) - 7)
    excess = (a - b).abs() - ulp - extra
    worst = excess.max().item()
    assert worst <= 0, f"{what}: fused and separate outputs differ by {worst:.3e} past one rounding"


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_fused_output_matches_oracle(w):
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    ref = oracle_full(w, inputs)
    out = fused(w, dev).clone()
    assert_close(out.float().cpu().numpy(), ref["out"], f"{w.name} fused out")
    again = fused(w, dev)
    assert torch.equal(out, again), "two fused calls differ"
    # the separate path rounds sigmoid(g_s) o_s to bf16 before the merge; the
    # fused one keeps it in fp32
    assert_one_rounding_apart(out, run(w, dev), w.name)


@pytest.mark.parametrize("w", [CASES[0], CASES[1], CASES[4], CASES[5]], ids=["ragged", "c5_ragged", "many_items",
                                                                            "one_frame"])
def test_fused_global_anchor_mode_matches_oracle(w):
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    ref = oracle_full(w, inputs, mode="global")
    out = fused(w, dev, anchor_query_mode=vb.ANCHOR_GLOBAL)
    assert_close(out.float().cpu().numpy(), ref["out"], f"{w.name} fused GLOBAL out")


def test_fused_rms_weight_gamma():
    w = CASES[4]
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    gamma = torch.rand((w.H, w.d), generator=torch.Generator("cpu").manual_seed(6)) + 0.5
    ref = oracle_full(w, inputs, gamma=gamma.double().numpy())
    out = fused(w, dev, rms_weight=gamma.cuda())
    assert_close(out.float().cpu().numpy(), ref["out"], "fused gamma out")


def test_fused_steps_and_host_call_equal_the_device_call():
    w = CASES[4]
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    ref = fused(w, dev).clone()
    out = torch.empty_like(dev["q"])
    steps = vb.Steps(dev["q"], dev["k"], dev["v"], dev["text_k"], dev["text_v"], dev["gate_s"], dev["gate_l"], out,
                     frames=w.F, chunk_frames=w.C, readout_mode=FUSED)
    steps.all_fused()
    torch.cuda.synchronize()
    assert torch.equal(out, ref), "fused steps differ from the fused call"
    host = {k: t.pin_memory() for k, t in inputs.items()}
    hout = vb.hybrid_attn_fwd_host(host["q"], host["k"], host["v"], host["text_k"], host["text_v"], host["gate_s"],
                                   host["gate_l"], frames=w.F, chunk_frames=w.C, readout_mode=FUSED)
    torch.cuda.synchronize()
    assert torch.equal(hout, ref.cpu()), "fused host call differs from the fused device call"


def test_fused_poisoned_workspace_changes_nothing():
    """With the workspace filled with NaN first, the fused call reads no
    scratch it has not written (the o_s area is never touched)."""
    w = CASES[0]
    dev = to_dev(make_inputs(w))
    a = fused(w, dev).clone()
    b = fused(w, dev, debug_flags=vb.POISON_WS)
    assert torch.equal(a, b)


def test_fused_exported_states_equal_separate():
    """The fused call runs the scan as a kernel of its own; the states it
    exports are those of the separate path's in-kernel scan."""
    w = CASES[1]
    dev = to_dev(make_inputs(w))
    s = vb.shape_of(dev["q"], dev["text_k"], w.F, w.C)
    shape = (w.B, w.F // w.C, w.H, w.d + 1, w.d)
    ex = [torch.empty(shape, dtype=torch.float32, device="cuda") for _ in range(4)]
    ws = vb.new_workspace(s, "cuda")
    fused(w, dev, workspace=ws, debug_flags=vb.EXPORT_STATES, export=(ex[0], ex[1]))
    run(w, dev, workspace=ws, debug_flags=vb.EXPORT_STATES, export=(ex[2], ex[3]))
    assert torch.equal(ex[0], ex[2]) and torch.equal(ex[1], ex[3])


@pytest.mark.parametrize("name,heads", [("768p_bf16", [0, 9, 23]), ("chunk5_bf16", [0, 15]),
                                        ("768p_long_bf16", [0, 23])])
def test_fused_workload_sampled_rows(name, heads):
    w = BY_NAME[name]
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    ws = vb.workspace_for(vb.shape_of(dev["q"], dev["text_k"], w.F, w.C), dev["q"].device)
    vb.clear_timeout_record(ws)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = fused(w, dev, status=status, workspace=ws)
    out2 = fused(w, dev, workspace=ws)
    assert int(status.item()) == 0, f"a bounded wait ran out: {vb.timeout_record(ws)}"
    assert torch.equal(out, out2), f"{name}: two fused calls differ"
    sep = run(w, dev, workspace=ws)
    del dev
    rng = np.random.default_rng(8)
    rows = sample_rows(w, rng)
    prob = O.Problem(B=1, F=w.F, P=w.P, H=1, d=w.d, T=w.T, C=w.C)
    for h in heads:
        x = {k: np64(t[:, :, h:h + 1, :]) for k, t in inputs.items()}
        ref = O.hybrid_attn_rows(x["q"], x["k"], x["v"], x["text_k"], x["text_v"], x["gate_s"], x["gate_l"],
                                 prob, 0, 0, rows)
        idx = torch.from_numpy(rows).cuda()
        assert_close(out[0, idx, h, :].float().cpu().numpy(), ref["out"], f"{name} fused head {h}")
        assert_one_rounding_apart(out[0, idx, h, :], sep[0, idx, h, :], f"{name} head {h}")


def test_fused_rejects_unsupported_configurations():
    w = BY_NAME["small_bf16"]  # head_dim 64
    dev = to_dev(make_inputs(w))
    with pytest.raises(vb.VdnError, match="unsupported"):
        fused(w, dev)


def test_injected_scan_count_timeout_reports_status_and_context_survives():
    """The fused readout's wait for the in-kernel scan's count
    (VDN_INJECT_TIMEOUT_SCAN: CTA 0's producer asks for one unit more than its
    (batch, head) has, 10-ms limit) ends with VDN_ERR_TIMEOUT in the status
    word instead of a hang or a fault; the timeout record names that wait
    (softmax kernel, block 0, warp 0, barrier offset 0 and parity 2: a counter
    wait), and the next call is correct."""
    import time
    w = CASES[4]
    inputs = make_inputs(w)
    dev = to_dev(inputs)
    ws = vb.workspace_for(vb.shape_of(dev["q"], dev["text_k"], w.F, w.C), dev["q"].device)
    vb.clear_timeout_record(ws)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    fused(w, dev, debug_flags=vb.INJECT_TIMEOUT_SCAN, status=status, workspace=ws)
    assert time.time() - t0 < 30
    assert int(status.item()) == 6
    rec = vb.timeout_record(ws)
    assert rec["timeouts"] >= 1 and rec["kernel"] == 3 and rec["block"] == 0 and rec["warp"] == 0, rec
    assert rec["bar_off"] == 0 and rec["parity"] == 2, rec
    assert 10_000_000 <= rec["ns"] < 1_000_000_000, rec
    vb.clear_timeout_record(ws)
    status.zero_()
    out = fused(w, dev, status=status, workspace=ws)
    assert int(status.item()) == 0
    assert_close(out.float().cpu().numpy(), oracle_full(w, inputs)["out"], f"{w.name} after the injected timeout")
