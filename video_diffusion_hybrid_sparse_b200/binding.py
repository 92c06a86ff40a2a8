"""ctypes binding of libvdnattn (argument marshalling only).

Every step of the hybrid attention runs in the library's CUDA kernels; this
module only turns torch tensors into pointers, fills the ``vdn_cfg`` struct,
passes the current CUDA stream and maps status codes to exceptions.  It
raises if the library has not been built: there is no other path.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvdnattn.so")
_lib = None

VDN_BF16, VDN_FP32 = 0, 1
OUT_SOFTMAX_ONLY, OUT_LINEAR_ONLY, OUT_LINEAR_RAW, EXPORT_STATES, INJECT_TIMEOUT = 1, 2, 4, 8, 16
STALL_READOUT_MMA, POISON_WS, INJECT_TIMEOUT_SCAN = 32, 64, 128
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "pointer not aligned",
          4: "workspace missing or too small", 5: "CUDA error", 6: "device wait timed out"}

EXPORTED = ["vdn_version", "vdn_status_string", "vdn_validate", "vdn_workspace_bytes", "vdn_plan_membership",
            "vdn_membership_device", "vdn_hybrid_attn_fwd", "vdn_stage_inputs", "vdn_state_build",
            "vdn_state_scan", "vdn_sparse_softmax", "vdn_softmax_and_scan", "vdn_readout_merge",
            "vdn_sparse_softmax_merge",
            "vdn_hybrid_attn_fwd_static",
            "vdn_static_scratch_bytes", "vdn_host_staging_bytes", "vdn_hybrid_attn_fwd_host", "vdn_export_states"]


class VdnError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, 'unknown')} (status {code})")
        self.code = code


class VdnCfg(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("frames", ctypes.c_int32), ("tokens_per_frame", ctypes.c_int32),
        ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("text_tokens", ctypes.c_int32),
        ("chunk_frames", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float), ("rms_eps", ctypes.c_float),
        ("rms_weight", ctypes.c_void_p),
        ("debug_flags", ctypes.c_int32), ("anchor_query_mode", ctypes.c_int32),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("status_word", ctypes.c_void_p),
        ("export_fwd", ctypes.c_void_p), ("export_bwd", ctypes.c_void_p),
        ("output_mode", ctypes.c_int32), ("softmax_precision", ctypes.c_int32),
        ("out_linear", ctypes.c_void_p), ("readout_mode", ctypes.c_int32),
    ]


def library() -> ctypes.CDLL:
    """Load libvdnattn.so from the package directory (raises if not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m video_diffusion_hybrid_sparse_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        C = ctypes.POINTER(VdnCfg)
        lib.vdn_version.restype = ctypes.c_int32
        lib.vdn_status_string.restype = ctypes.c_char_p
        lib.vdn_status_string.argtypes = [ctypes.c_int]
        lib.vdn_validate.argtypes = [C]
        lib.vdn_workspace_bytes.restype = ctypes.c_size_t
        lib.vdn_workspace_bytes.argtypes = [C]
        lib.vdn_plan_membership.argtypes = [C, P]
        lib.vdn_membership_device.argtypes = [C, P, P]
        lib.vdn_hybrid_attn_fwd.argtypes = [P, P, P, P, P, P, P, P, C, P]
        lib.vdn_stage_inputs.argtypes = [P, P, P, P, P, C, P]
        lib.vdn_state_build.argtypes = [P, P, P, P, C, P]
        lib.vdn_state_scan.argtypes = [C, P]
        lib.vdn_export_states.argtypes = [C, P, P, P]
        lib.vdn_sparse_softmax.argtypes = [P, P, P, P, P, C, P]
        lib.vdn_softmax_and_scan.argtypes = [P, P, P, P, P, P, C, P]
        lib.vdn_readout_merge.argtypes = [P, P, P, P, C, P]
        lib.vdn_sparse_softmax_merge.argtypes = [P, P, P, P, P, P, P, P, C, P]
        lib.vdn_hybrid_attn_fwd_static.argtypes = [P, P, P, P, P, P, P, P, C, P]
        lib.vdn_static_scratch_bytes.restype = ctypes.c_size_t
        lib.vdn_host_staging_bytes.restype = ctypes.c_size_t
        lib.vdn_host_staging_bytes.argtypes = [C]
        lib.vdn_hybrid_attn_fwd_host.argtypes = [P, P, P, P, P, P, P, P, P, ctypes.c_size_t, C, P]
        for name in EXPORTED:
            if name not in ("vdn_version", "vdn_status_string", "vdn_workspace_bytes", "vdn_static_scratch_bytes",
                            "vdn_host_staging_bytes"):
                getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


@dataclass
class Shape:
    """Sizes of one call: batch, latent frames, tokens per frame, heads,
    head_dim, text tokens, frames per chunk."""
    B: int
    F: int
    P: int
    H: int
    d: int
    T: int
    C: int
    fp32: bool = False

    @property
    def N(self) -> int:
        return self.F * self.P


ANCHOR_LOCAL, ANCHOR_GLOBAL = 0, 1
OUTPUT_MERGED, OUTPUT_SPLIT = 0, 1
PREC_BF16, PREC_FP8 = 0, 1
READOUT_SEPARATE, READOUT_FUSED = 0, 1


def make_cfg(s: Shape, *, softmax_scale: float = 0.0, rms_eps: float = -1.0, rms_weight=None,
             debug_flags: int = 0, workspace=None, status=None, export=None,
             anchor_query_mode: int = ANCHOR_LOCAL, out_linear=None, softmax_precision: int = PREC_BF16,
             readout_mode: int = READOUT_SEPARATE) -> VdnCfg:
    cfg = VdnCfg()
    cfg.batch, cfg.frames, cfg.tokens_per_frame = s.B, s.F, s.P
    cfg.heads, cfg.head_dim, cfg.text_tokens, cfg.chunk_frames = s.H, s.d, s.T, s.C
    cfg.dtype = VDN_FP32 if s.fp32 else VDN_BF16
    cfg.softmax_scale = softmax_scale
    cfg.rms_eps = rms_eps
    cfg.rms_weight = _ptr(rms_weight)
    cfg.debug_flags = debug_flags
    cfg.anchor_query_mode = anchor_query_mode
    cfg.output_mode = OUTPUT_SPLIT if out_linear is not None else OUTPUT_MERGED
    cfg.softmax_precision = softmax_precision
    cfg.out_linear = _ptr(out_linear)
    cfg.readout_mode = readout_mode
    if workspace is not None:
        cfg.workspace = workspace.data_ptr()
        cfg.workspace_bytes = workspace.numel() * workspace.element_size()
    cfg.status_word = _ptr(status)
    if export is not None:
        cfg.export_fwd = export[0].data_ptr()
        cfg.export_bwd = export[1].data_ptr()
    return cfg


def _ptr(t):
    return None if t is None else t.data_ptr()


def _check(code: int, where: str):
    if code != 0:
        raise VdnError(code, where)


def _stream(stream=None) -> int:
    return (stream if stream is not None else torch.cuda.current_stream()).cuda_stream


def shape_of(q: torch.Tensor, text_k: torch.Tensor, frames: int, chunk_frames: int) -> Shape:
    B, N, H, d = q.shape
    if N % frames:
        raise ValueError("video tokens must be frames * tokens_per_frame")
    return Shape(B, frames, N // frames, H, d, text_k.shape[1], chunk_frames, q.dtype == torch.float32)


def workspace_bytes(s: Shape, softmax_precision: int = PREC_BF16) -> int:
    cfg = make_cfg(s, softmax_precision=softmax_precision)
    n = library().vdn_workspace_bytes(ctypes.byref(cfg))
    if n == 0:
        _check(library().vdn_validate(ctypes.byref(cfg)), "vdn_workspace_bytes")
    return n


_WS: dict = {}


def new_workspace(s: Shape, device, softmax_precision: int = PREC_BF16) -> torch.Tensor:
    """A fresh device workspace for shape s (one per call in flight)."""
    return torch.empty(workspace_bytes(s, softmax_precision), dtype=torch.uint8, device=torch.device(device))


def workspace_for(s: Shape, device, softmax_precision: int = PREC_BF16) -> torch.Tensor:
    """A cached device workspace large enough for shape s."""
    n = workspace_bytes(s, softmax_precision)
    dev = torch.device(device)
    key = (dev.index if dev.index is not None else torch.cuda.current_device())
    buf = _WS.get(key)
    if buf is None or buf.numel() < n:
        buf = torch.empty(n, dtype=torch.uint8, device=dev)
        _WS[key] = buf
    return buf


def hybrid_attn_fwd(q, k, v, text_k, text_v, gate_s, gate_l, *, frames: int, chunk_frames: int, out=None,
                    softmax_scale: float = 0.0, rms_eps: float = -1.0, rms_weight=None, debug_flags: int = 0,
                    workspace=None, status=None, export=None, stream=None,
                    anchor_query_mode: int = ANCHOR_LOCAL, out_linear=None,
                    softmax_precision: int = PREC_BF16, readout_mode: int = READOUT_SEPARATE) -> torch.Tensor:
    """The whole hybrid attention call on the current CUDA stream.

    q, k, v, gate_s, gate_l: [B, F*P, H, d]; text_k, text_v: [B, T, H, d];
    all contiguous CUDA tensors of one dtype (bf16 or fp32).  With
    ``out_linear`` (a tensor like q) the SPLIT output is written: ``out``
    gets sigmoid(gate_s) * o_s and ``out_linear`` sigmoid(gate_l) * r.
    ``readout_mode=READOUT_FUSED`` runs the readout and merge in the softmax
    kernel's epilogue (bf16, head_dim 128, merged output)."""
    s = shape_of(q, text_k, frames, chunk_frames)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = workspace_for(s, q.device, softmax_precision)
    cfg = make_cfg(s, softmax_scale=softmax_scale, rms_eps=rms_eps, rms_weight=rms_weight,
                   debug_flags=debug_flags, workspace=workspace, status=status, export=export,
                   anchor_query_mode=anchor_query_mode, out_linear=out_linear,
                   softmax_precision=softmax_precision, readout_mode=readout_mode)
    code = library().vdn_hybrid_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(text_k), _ptr(text_v),
                                         gate_s.data_ptr(), gate_l.data_ptr(), out.data_ptr(),
                                         ctypes.byref(cfg), _stream(stream))
    _check(code, "vdn_hybrid_attn_fwd")
    return out


def export_states(s: Shape, workspace: torch.Tensor, fwd: torch.Tensor, bwd: torch.Tensor, *, stream=None,
                  softmax_precision: int = PREC_BF16) -> None:
    """S_F / z_F and S_B / z_B ([B, F/C, H, d+1, d] fp32 each) recomputed from
    the state partials that the last call on `workspace` left there."""
    cfg = make_cfg(s, workspace=workspace, softmax_precision=softmax_precision)
    _check(library().vdn_export_states(ctypes.byref(cfg), fwd.data_ptr(), bwd.data_ptr(), _stream(stream)),
           "vdn_export_states")


_STAGING: dict = {}


_REC_FIELDS = ("timeouts", "kernel", "block", "warp", "bar_off", "parity")
# kernel ids in the record: 1 state build, 3 softmax (bf16), 31 softmax (fp8),
# 4 readout + merge (TMA-fed), 41 readout + merge (general)


def timeout_record(workspace: torch.Tensor) -> dict:
    """The kernels' timeout record: 16 int32 words at byte 64 of the
    workspace, describing the first bounded wait that ran out since the record
    was cleared (kernel id, block, warp, barrier as its byte distance to the
    CTA's abort flag, phase parity, global nanoseconds waited, SM)."""
    w = workspace[64:128].view(torch.int32).cpu().tolist()
    rec = dict(zip(_REC_FIELDS, w[:6]))
    rec["ns"] = (w[6] & 0xFFFFFFFF) | (w[7] << 32)
    rec["sm"] = w[8]
    return rec


def clear_timeout_record(workspace: torch.Tensor) -> None:
    workspace[64:128].zero_()


def staging_bytes(s: Shape, split: bool = False) -> int:
    """Bytes of the device staging buffer :func:`hybrid_attn_fwd_host` needs."""
    cfg = make_cfg(s)
    if split:
        cfg.output_mode = OUTPUT_SPLIT
    n = library().vdn_host_staging_bytes(ctypes.byref(cfg))
    if n == 0:
        _check(library().vdn_validate(ctypes.byref(cfg)), "vdn_host_staging_bytes")
    return n


def new_staging(s: Shape, device, split: bool = False) -> torch.Tensor:
    """A fresh device staging buffer (one per host call in flight)."""
    return torch.empty(staging_bytes(s, split), dtype=torch.uint8, device=torch.device(device))


def staging_for(s: Shape, device, split: bool = False) -> torch.Tensor:
    """A cached device staging buffer for :func:`hybrid_attn_fwd_host`."""
    n = staging_bytes(s, split)
    dev = torch.device(device)
    key = (dev.index if dev.index is not None else torch.cuda.current_device())
    buf = _STAGING.get(key)
    if buf is None or buf.numel() < n:
        buf = torch.empty(n, dtype=torch.uint8, device=dev)
        _STAGING[key] = buf
    return buf


def hybrid_attn_fwd_host(q, k, v, text_k, text_v, gate_s, gate_l, *, frames: int, chunk_frames: int, out=None,
                         softmax_scale: float = 0.0, rms_eps: float = -1.0, rms_weight=None, workspace=None,
                         staging=None, stream=None, anchor_query_mode: int = ANCHOR_LOCAL,
                         out_linear=None, device="cuda", softmax_precision: int = PREC_BF16,
                         readout_mode: int = READOUT_SEPARATE) -> torch.Tensor:
    """The whole call on HOST tensors (contiguous CPU tensors, ideally pinned),
    copies overlapped with the kernels inside the library.  Returns the host
    ``out``; synchronise ``stream`` (default: the current stream of
    ``device``) before reading it."""
    s = shape_of(q, text_k, frames, chunk_frames)
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=q.is_pinned())
    if workspace is None:
        workspace = workspace_for(s, device, softmax_precision)
    if staging is None:
        staging = staging_for(s, device, out_linear is not None)
    cfg = make_cfg(s, softmax_scale=softmax_scale, rms_eps=rms_eps, rms_weight=rms_weight, workspace=workspace,
                   anchor_query_mode=anchor_query_mode, out_linear=out_linear, softmax_precision=softmax_precision,
                   readout_mode=readout_mode)
    code = library().vdn_hybrid_attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(text_k), _ptr(text_v),
                                              gate_s.data_ptr(), gate_l.data_ptr(), out.data_ptr(),
                                              staging.data_ptr(), staging.numel(), ctypes.byref(cfg),
                                              _stream(stream))
    _check(code, "vdn_hybrid_attn_fwd_host")
    return out


class Steps:
    """The separately scheduled steps of one call (same arguments as
    :func:`hybrid_attn_fwd`), for per-kernel timing and stream overlap."""

    def __init__(self, q, k, v, text_k, text_v, gate_s, gate_l, out, *, frames, chunk_frames, workspace=None,
                 debug_flags=0, rms_weight=None, export=None, status=None, anchor_query_mode=ANCHOR_LOCAL,
                 out_linear=None, softmax_precision=PREC_BF16, readout_mode=READOUT_SEPARATE):
        self.t = (q, k, v, text_k, text_v, gate_s, gate_l, out)
        self.s = shape_of(q, text_k, frames, chunk_frames)
        self.ws = workspace if workspace is not None else workspace_for(self.s, q.device, softmax_precision)
        self.cfg = make_cfg(self.s, workspace=self.ws, debug_flags=debug_flags, rms_weight=rms_weight,
                            export=export, status=status, anchor_query_mode=anchor_query_mode,
                            out_linear=out_linear, softmax_precision=softmax_precision,
                            readout_mode=readout_mode)
        self.lib = library()

    def stage(self, stream=None):
        q, k, v, tk, tv = self.t[:5]
        _check(self.lib.vdn_stage_inputs(q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(tk), _ptr(tv),
                                         ctypes.byref(self.cfg), _stream(stream)), "vdn_stage_inputs")

    def state_build(self, stream=None):
        _, k, v, tk, tv = self.t[:5]
        _check(self.lib.vdn_state_build(k.data_ptr(), v.data_ptr(), _ptr(tk), _ptr(tv), ctypes.byref(self.cfg),
                                        _stream(stream)), "vdn_state_build")

    def state_scan(self, stream=None):
        _check(self.lib.vdn_state_scan(ctypes.byref(self.cfg), _stream(stream)), "vdn_state_scan")

    def sparse_softmax(self, stream=None):
        q, k, v, tk, tv = self.t[:5]
        _check(self.lib.vdn_sparse_softmax(q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(tk), _ptr(tv),
                                           ctypes.byref(self.cfg), _stream(stream)), "vdn_sparse_softmax")

    def softmax_and_scan(self, stream=None, gate=True):
        """The softmax branch and the scan; with ``gate`` the kernel also
        applies the softmax branch's gate (as the whole call does)."""
        q, k, v, tk, tv, gs = self.t[:6]
        _check(self.lib.vdn_softmax_and_scan(q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(tk), _ptr(tv),
                                             gs.data_ptr() if gate else None, ctypes.byref(self.cfg),
                                             _stream(stream)),
               "vdn_softmax_and_scan")

    def readout_merge(self, stream=None):
        q, gs, gl, out = self.t[0], self.t[5], self.t[6], self.t[7]
        _check(self.lib.vdn_readout_merge(q.data_ptr(), gs.data_ptr(), gl.data_ptr(), out.data_ptr(),
                                          ctypes.byref(self.cfg), _stream(stream)), "vdn_readout_merge")

    def softmax_merge(self, stream=None):
        """The softmax branch with the scan inside and the readout and merge
        in its epilogue (after state_build)."""
        q, k, v, tk, tv, gs, gl, out = self.t
        _check(self.lib.vdn_sparse_softmax_merge(q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(tk), _ptr(tv),
                                                 gs.data_ptr(), gl.data_ptr(), out.data_ptr(),
                                                 ctypes.byref(self.cfg), _stream(stream)),
               "vdn_sparse_softmax_merge")

    def all_fused(self, stream=None):
        """The sequence of a call with the fused readout."""
        self.state_build(stream)
        self.softmax_merge(stream)

    def all(self, stream=None):
        """The whole call's sequence (the scan inside the softmax kernel)."""
        self.stage(stream)
        self.state_build(stream)
        self.softmax_and_scan(stream)
        self.readout_merge(stream)

    def all_separate(self, stream=None):
        """The same result with the scan as a kernel of its own."""
        self.stage(stream)
        self.state_build(stream)
        self.state_scan(stream)
        self.sparse_softmax(stream)
        self.readout_merge(stream)


def plan_membership(F: int, C: int, anchor_query_mode: int = ANCHOR_LOCAL) -> np.ndarray:
    """Host membership table from the library (1 softmax, 2 forward, 3 backward)."""
    s = Shape(1, F, 1, 1, 64, 0, C)
    table = np.zeros((F, F), dtype=np.uint8)
    cfg = make_cfg(s, anchor_query_mode=anchor_query_mode)
    _check(library().vdn_plan_membership(ctypes.byref(cfg), table.ctypes.data), "vdn_plan_membership")
    return table


def membership_device(F: int, C: int, P: int = 1, T: int = 0, device="cuda",
                      anchor_query_mode: int = ANCHOR_LOCAL) -> np.ndarray:
    """The membership table as the kernels' index logic produces it on the GPU."""
    s = Shape(1, F, P, 1, 64, T, C)
    table = torch.zeros((F, F), dtype=torch.uint8, device=device)
    cfg = make_cfg(s, anchor_query_mode=anchor_query_mode)
    _check(library().vdn_membership_device(ctypes.byref(cfg), table.data_ptr(), _stream()),
           "vdn_membership_device")
    torch.cuda.synchronize()
    return table.cpu().numpy()


def validate(s: Shape, **kw) -> int:
    """Status code of the host-side argument check (no CUDA call)."""
    return library().vdn_validate(ctypes.byref(make_cfg(s, **kw)))
