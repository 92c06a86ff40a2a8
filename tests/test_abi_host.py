"""Host-only checks of the C ABI (no GPU needed, no kernel launched).

* the shared library loads and exports every function include/vdnattn.h declares;
* argument validation returns the documented status codes before any CUDA call;
* the host membership table equals the oracle's, bit for bit, on the workload
  shapes and on edge cases (one to three frames, one chunk, many chunks);
* the binding reads the kernels' timeout record where and as they write it.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

from oracle import hybrid_attn as O
from video_diffusion_hybrid_sparse_b200 import binding as vb
from video_diffusion_hybrid_sparse_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vdnattn.h")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"VDN_API\s+[\w\s\*]+?\b(vdn_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    lib = vb.library()
    names = declared_functions()
    assert len(names) >= 12
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(vb.EXPORTED)


def test_version_and_status_strings():
    lib = vb.library()
    assert lib.vdn_version() >> 16 == 1
    for code, text in vb.STATUS.items():
        assert lib.vdn_status_string(code).decode() == text


def shape(**kw):
    base = dict(B=1, F=15, P=16, H=2, d=64, T=8, C=1, fp32=False)
    base.update(kw)
    return vb.Shape(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(), 0),
    (dict(F=16, C=5), 1),          # frames not a whole number of chunks
    (dict(d=48), 2),               # unsupported head_dim
    (dict(d=256), 2),
    (dict(T=-1), 1),
    (dict(B=0), 1),
    (dict(P=0), 1),
    (dict(F=200, C=1), 0),         # 200 chunks: within the 256 the kernel parameters carry
    (dict(F=257, C=1), 2),         # more chunks than the kernel parameters carry
    (dict(d=32, fp32=True), 0),
    (dict(d=128, F=60, C=5, P=4032, H=24, T=512), 0),
])
def test_validate_codes(kw, code):
    assert vb.validate(shape(**kw)) == code


def test_validate_rejects_unknown_dtype_and_flags():
    lib = vb.library()
    cfg = vb.make_cfg(shape())
    cfg.dtype = 7
    assert lib.vdn_validate(ctypes.byref(cfg)) == 2
    cfg = vb.make_cfg(shape(), debug_flags=256)
    assert lib.vdn_validate(ctypes.byref(cfg)) == 1
    for flag in (vb.INJECT_TIMEOUT, vb.STALL_READOUT_MMA, vb.POISON_WS, vb.INJECT_TIMEOUT_SCAN):
        cfg = vb.make_cfg(shape(), debug_flags=flag)
        assert lib.vdn_validate(ctypes.byref(cfg)) == 0
    cfg = vb.make_cfg(shape())
    cfg.softmax_precision = 3
    assert lib.vdn_validate(ctypes.byref(cfg)) == 1
    # fp8 softmax: head_dim 128, bf16, tokens per frame a multiple of 16
    assert vb.validate(shape(d=128, P=32), softmax_precision=vb.PREC_FP8) == 0
    assert vb.validate(shape(d=64, P=32), softmax_precision=vb.PREC_FP8) == 2
    assert vb.validate(shape(d=128, P=30), softmax_precision=vb.PREC_FP8) == 2
    assert vb.validate(shape(d=128, P=32, fp32=True), softmax_precision=vb.PREC_FP8) == 2
    s8 = shape(d=128, P=32)
    assert vb.workspace_bytes(s8, vb.PREC_FP8) > vb.workspace_bytes(s8)
    for mode in (2, -1):
        cfg = vb.make_cfg(shape())
        cfg.anchor_query_mode = mode
        assert lib.vdn_validate(ctypes.byref(cfg)) == 1
        cfg = vb.make_cfg(shape())
        cfg.output_mode = mode
        assert lib.vdn_validate(ctypes.byref(cfg)) == 1
    cfg = vb.make_cfg(shape(), anchor_query_mode=vb.ANCHOR_GLOBAL)
    assert lib.vdn_validate(ctypes.byref(cfg)) == 0
    # SPLIT excludes the debug outputs
    cfg = vb.make_cfg(shape(), debug_flags=vb.OUT_SOFTMAX_ONLY)
    cfg.output_mode = vb.OUTPUT_SPLIT
    assert lib.vdn_validate(ctypes.byref(cfg)) == 1
    assert lib.vdn_validate(None) == 1


def test_cfg_struct_layout_matches_header(tmp_path):
    """The ctypes mirror of vdn_cfg has the C layout: every field's offset
    and the size, as a C compiler lays out the header's struct."""
    fields = [f[0] for f in vb.VdnCfg._fields_]
    src = tmp_path / "layout.c"
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "vdnattn.h"', "int main(void) {"]
    lines += [f'  printf("%zu\\n", offsetof(vdn_cfg, {f}));' for f in fields]
    lines += ['  printf("%zu\\n", sizeof(vdn_cfg));', "  return 0;", "}"]
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    assert got[:-1] == [getattr(vb.VdnCfg, f).offset for f in fields]
    assert got[-1] == ctypes.sizeof(vb.VdnCfg)


def test_readout_mode_validation():
    """VDN_READOUT_FUSED: bf16, head_dim 128, bf16 softmax operands and the
    merged output without debug outputs; anything else is unsupported, and an
    unknown mode is an invalid argument."""
    lib = vb.library()
    ok = vb.Shape(1, 15, 256, 2, 128, 64, 1)
    assert lib.vdn_validate(ctypes.byref(vb.make_cfg(ok, readout_mode=vb.READOUT_FUSED))) == 0
    assert lib.vdn_validate(ctypes.byref(vb.make_cfg(ok, readout_mode=vb.READOUT_FUSED,
                                                      anchor_query_mode=vb.ANCHOR_GLOBAL))) == 0
    assert lib.vdn_validate(ctypes.byref(vb.make_cfg(ok, readout_mode=2))) == 1
    unsupported = [
        vb.make_cfg(vb.Shape(1, 15, 256, 2, 64, 64, 1), readout_mode=vb.READOUT_FUSED),
        vb.make_cfg(vb.Shape(1, 15, 256, 2, 128, 64, 1, fp32=True), readout_mode=vb.READOUT_FUSED),
        vb.make_cfg(ok, readout_mode=vb.READOUT_FUSED, softmax_precision=vb.PREC_FP8),
        vb.make_cfg(ok, readout_mode=vb.READOUT_FUSED, debug_flags=vb.OUT_LINEAR_RAW),
    ]
    split = vb.make_cfg(ok, readout_mode=vb.READOUT_FUSED)
    split.output_mode = vb.OUTPUT_SPLIT
    unsupported.append(split)
    for cfg in unsupported:
        assert lib.vdn_validate(ctypes.byref(cfg)) == 2
    # the injected wait of the fused readout's scan count is a known debug flag
    assert lib.vdn_validate(ctypes.byref(vb.make_cfg(ok, readout_mode=vb.READOUT_FUSED,
                                                      debug_flags=vb.INJECT_TIMEOUT_SCAN))) == 0
    assert lib.vdn_validate(ctypes.byref(vb.make_cfg(ok, debug_flags=256))) == 1
    # the fused step itself checks the requirements whatever the mode says
    cfg = vb.make_cfg(vb.Shape(1, 15, 256, 2, 64, 64, 1))
    assert lib.vdn_sparse_softmax_merge(*([None] * 8), ctypes.byref(cfg), None) == 2


def test_workspace_bytes():
    for w in WORKLOADS:
        n = vb.workspace_bytes(vb.Shape(w.B, w.F, w.P, w.H, w.d, w.T, w.C, w.dtype == "fp32"))
        o_s = w.B * w.N * w.H * max(64, w.d) * 2
        assert n > o_s
        assert n % 1024 == 0
    assert vb.library().vdn_workspace_bytes(ctypes.byref(vb.make_cfg(shape(F=16, C=5)))) == 0


def test_call_errors_before_any_launch():
    """Bad workspace / pointers are reported without touching the GPU."""
    lib = vb.library()
    s = shape()
    cfg = vb.make_cfg(s)  # no workspace
    p = 1 << 20  # aligned fake device addresses; never dereferenced on these paths
    args = [p, p, p, p, p, p, p, p]
    assert lib.vdn_hybrid_attn_fwd(*args, ctypes.byref(cfg), None) == 4
    cfg.workspace = p
    cfg.workspace_bytes = 16
    assert lib.vdn_hybrid_attn_fwd(*args, ctypes.byref(cfg), None) == 4
    cfg.workspace_bytes = vb.workspace_bytes(s)
    cfg.workspace = p + 128  # workspace must be 256-byte aligned
    assert lib.vdn_hybrid_attn_fwd(*args, ctypes.byref(cfg), None) == 3
    cfg.workspace = p
    bad = list(args)
    bad[1] = p + 8  # k misaligned
    assert lib.vdn_hybrid_attn_fwd(*bad, ctypes.byref(cfg), None) == 3
    bad = list(args)
    bad[0] = None  # q missing
    assert lib.vdn_hybrid_attn_fwd(*bad, ctypes.byref(cfg), None) == 1
    bad = list(args)
    bad[3] = None  # text_k missing while T > 0
    assert lib.vdn_hybrid_attn_fwd(*bad, ctypes.byref(cfg), None) == 1
    cfg.debug_flags = vb.EXPORT_STATES  # export requested without buffers
    assert lib.vdn_hybrid_attn_fwd(*args, ctypes.byref(cfg), None) == 1
    assert lib.vdn_state_scan(ctypes.byref(cfg), None) == 1
    cfg.debug_flags = 0
    assert lib.vdn_export_states(ctypes.byref(cfg), None, p, None) == 1  # no buffer
    assert lib.vdn_export_states(ctypes.byref(cfg), p + 4, p, None) == 3  # misaligned
    assert lib.vdn_export_states(ctypes.byref(vb.make_cfg(s)), p, p, None) == 4  # no workspace
    assert lib.vdn_plan_membership(ctypes.byref(cfg), None) == 1
    cfg.output_mode = vb.OUTPUT_SPLIT  # SPLIT without its second output buffer
    assert lib.vdn_hybrid_attn_fwd(*args, ctypes.byref(cfg), None) == 1
    assert lib.vdn_readout_merge(p, p, p, p, ctypes.byref(cfg), None) == 1
    assert lib.vdn_hybrid_attn_fwd_static(*args, ctypes.byref(cfg), None) == 1
    cfg.out_linear = p + 4
    assert lib.vdn_hybrid_attn_fwd(*args, ctypes.byref(cfg), None) == 3


def test_static_call_checks_every_pointer_before_any_cuda_call():
    """vdn_hybrid_attn_fwd_static clears its status slot on the stream before
    the regular path runs, so every pointer rule must be checked first.  On a
    host without a GPU any CUDA call fails (VDN_ERR_CUDA): an alignment or
    argument status therefore shows that the check came before it."""
    lib = vb.library()
    s = shape()
    p = 1 << 20
    args = [p] * 8
    cfg = vb.make_cfg(s)
    cfg.status_word = p + 2  # not 4-byte aligned
    assert lib.vdn_hybrid_attn_fwd_static(*args, ctypes.byref(cfg), None) == 3
    cfg = vb.make_cfg(s)
    cfg.rms_weight = p + 8  # not 16-byte aligned
    assert lib.vdn_hybrid_attn_fwd_static(*args, ctypes.byref(cfg), None) == 3
    cfg = vb.make_cfg(s)
    bad = list(args)
    bad[6] = p + 4  # gate_l misaligned
    assert lib.vdn_hybrid_attn_fwd_static(*bad, ctypes.byref(cfg), None) == 3
    if not torch.cuda.is_available():  # well-formed call: it reaches the CUDA runtime, which has no device here
        assert lib.vdn_hybrid_attn_fwd_static(*args, ctypes.byref(vb.make_cfg(s)), None) == 5


def test_host_call_errors_before_any_copy():
    """vdn_hybrid_attn_fwd_host: argument and staging checks come first."""
    lib = vb.library()
    s = shape()
    cfg = vb.make_cfg(s)
    n = lib.vdn_host_staging_bytes(ctypes.byref(cfg))
    e = 2  # bf16
    vid, txt = s.B * s.N * s.H * s.d * e, s.B * s.T * s.H * s.d * e
    assert n >= 6 * vid + 2 * txt
    split = vb.make_cfg(s)
    split.output_mode = vb.OUTPUT_SPLIT
    assert lib.vdn_host_staging_bytes(ctypes.byref(split)) >= n + vid
    assert lib.vdn_host_staging_bytes(ctypes.byref(vb.make_cfg(shape(F=16, C=5)))) == 0
    p = 1 << 20
    args = [p] * 8
    cfg.workspace, cfg.workspace_bytes = p, vb.workspace_bytes(s)
    assert lib.vdn_hybrid_attn_fwd_host(*args, None, n, ctypes.byref(cfg), None) == 4      # no staging
    assert lib.vdn_hybrid_attn_fwd_host(*args, p, n - 1, ctypes.byref(cfg), None) == 4     # too small
    assert lib.vdn_hybrid_attn_fwd_host(*args, p + 16, n, ctypes.byref(cfg), None) == 3    # misaligned
    bad = list(args)
    bad[0] = None
    assert lib.vdn_hybrid_attn_fwd_host(*bad, p, n, ctypes.byref(cfg), None) == 1
    cfg.output_mode = vb.OUTPUT_SPLIT  # no host out_linear
    assert lib.vdn_hybrid_attn_fwd_host(*args, p, n, ctypes.byref(cfg), None) == 1
    cfg.output_mode = 0
    cfg.workspace = None
    assert lib.vdn_hybrid_attn_fwd_host(*args, p, n, ctypes.byref(cfg), None) == 4


EDGE = [(1, 1), (2, 1), (2, 2), (3, 1), (3, 3), (4, 2), (5, 1), (6, 3), (15, 1), (15, 5), (45, 5), (60, 5),
        (60, 1), (10, 10), (96, 1)]


@pytest.mark.parametrize("F,C", EDGE + [(w.F, w.C) for w in WORKLOADS])
def test_host_membership_matches_oracle(F, C):
    np.testing.assert_array_equal(vb.plan_membership(F, C), O.membership_table(F, C))
    np.testing.assert_array_equal(vb.plan_membership(F, C, vb.ANCHOR_GLOBAL), O.membership_table(F, C, "global"))


def test_timeout_record_reader_matches_the_kernels_layout():
    """binding.timeout_record reads the words the kernels write (the kRec*
    indices of csrc/sm100.cuh, at byte 64 of the workspace as api.cu places
    them), and clear_timeout_record zeroes them."""
    import torch
    csrc = os.path.join(ROOT, "video_diffusion_hybrid_sparse_b200", "csrc")
    idx = {m.group(1): int(m.group(2))
           for m in re.finditer(r"\bkRec(\w+) = (\d+)", open(os.path.join(csrc, "sm100.cuh")).read())}
    assert re.search(r"ws\(cfg, g\.off_status\) \+ 64\)", open(os.path.join(csrc, "api.cu")).read())
    assert idx["Words"] * 4 <= 256 - 64  # inside the 256-byte status slot
    ws = torch.zeros(256, dtype=torch.uint8)
    words = ws[64:128].view(torch.int32)
    ns = 3 * 2**32 + 123456789
    vals = {"Timeouts": 2, "Kernel": 4, "Block": 77, "Warp": 1, "BarOff": 92, "Parity": 1, "Sm": 140}
    for k, v in vals.items():
        words[idx[k]] = v
    words[idx["Ns"]] = ns & 0xFFFFFFFF if ns & 0x80000000 == 0 else (ns & 0xFFFFFFFF) - 2**32
    words[idx["Ns"] + 1] = ns >> 32
    rec = vb.timeout_record(ws)
    assert rec == {"timeouts": 2, "kernel": 4, "block": 77, "warp": 1, "bar_off": 92, "parity": 1, "ns": ns,
                   "sm": 140}
    vb.clear_timeout_record(ws)
    assert int(ws[64:128].sum()) == 0 and vb.timeout_record(ws)["timeouts"] == 0
