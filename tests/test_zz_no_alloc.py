"""The entry point for callers that cannot allocate device memory.

vdn_hybrid_attn_fwd_static serves code that runs inside another runtime's
plugin interface (tensors handed over, no allocator) or in latency-critical
loops where cudaMalloc is not acceptable: it takes no workspace and uses a
32 MiB static device array inside the library instead.  These checks call it
through the C ABI and compare it with the regular entry point (same
tolerance as the other parity tests), over consecutive calls on different
shapes, so stale contents of the shared array would show; and they check
that a problem too large for the array is refused before any work is queued.

This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from video_diffusion_hybrid_sparse_b200 import binding as vb
from video_diffusion_hybrid_sparse_b200.workloads import BY_NAME, make_inputs

pytestmark = pytest.mark.gpu

TOL_ABS, TOL_REL = 2e-2, 1e-2


def _static_call(dev, w, out):
    lib = vb.library()
    s = vb.shape_of(dev["q"], dev["text_k"], w.F, w.C)
    cfg = vb.make_cfg(s)  # no workspace: the static array is used
    code = lib.vdn_hybrid_attn_fwd_static(dev["q"].data_ptr(), dev["k"].data_ptr(), dev["v"].data_ptr(),
                                          dev["text_k"].data_ptr(), dev["text_v"].data_ptr(),
                                          dev["gate_s"].data_ptr(), dev["gate_l"].data_ptr(), out.data_ptr(),
                                          ctypes.byref(cfg), torch.cuda.current_stream().cuda_stream)
    return code


def _close(got, ref):
    got = got.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    assert np.all(np.isfinite(got))
    assert np.abs(got - ref).max() <= TOL_ABS
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= TOL_REL


def test_static_scratch_matches_regular_entry_point():
    assert vb.library().vdn_static_scratch_bytes() == 32 << 20
    seq = ["small_bf16", "tiny_fp32", "small_bf16"]  # consecutive calls, different shapes
    cache = {}
    for name in seq:
        w = BY_NAME[name]
        if name not in cache:
            dev = {k: t.cuda() for k, t in make_inputs(w).items()}
            ref = vb.hybrid_attn_fwd(dev["q"], dev["k"], dev["v"], dev["text_k"], dev["text_v"], dev["gate_s"],
                                     dev["gate_l"], frames=w.F, chunk_frames=w.C)
            cache[name] = (dev, ref)
        dev, ref = cache[name]
        out = torch.full_like(dev["q"], float("nan"))
        assert _static_call(dev, w, out) == 0
        torch.cuda.synchronize()
        _close(out, ref)


def test_static_scratch_refuses_too_large_problem():
    w = BY_NAME["768p_h4_bf16"]  # needs about 77 MiB of scratch
    small = BY_NAME["small_bf16"]
    dev = {k: t.cuda() for k, t in make_inputs(small).items()}
    lib = vb.library()
    cfg = vb.make_cfg(vb.Shape(w.B, w.F, w.P, w.H, w.d, w.T, w.C))
    assert vb.workspace_bytes(vb.Shape(w.B, w.F, w.P, w.H, w.d, w.T, w.C)) > (32 << 20)
    p = dev["q"].data_ptr()
    code = lib.vdn_hybrid_attn_fwd_static(p, p, p, p, p, p, p, p, ctypes.byref(cfg),
                                          torch.cuda.current_stream().cuda_stream)
    assert code == 4  # workspace too small, nothing queued
