"""Workload shapes and seeded synthetic inputs.

This module holds no arithmetic of the method: it only describes problem sizes
and draws random tensors.  It is the one module that both the CUDA path's
tests/benchmark and the CPU oracle's tests read their inputs from.

The shapes stand in for the VDN-H3 article's measured workload (a 768p,
~14.4 s video; section 性能实测表现): the page gives no latent shape, so a
15 x (48 x 84) latent (the frame-7 example implies 15 latent frames) and a
60-frame long variant are used, plus three smaller cases.

Draw recipe: ``torch.Generator('cpu').manual_seed(seed)`` with
``seed = 20261202 + index``; tensors drawn in the order q, k, v, text_k,
text_v, gate_s, gate_l as float32 N(0, 1), then shaped per ``dist``:
``"normal"`` keeps them, ``"half"`` multiplies q/k/v/text by 0.5, ``"rms"``
divides every (token, head) vector of q/k/v/text by its root-mean-square over
head_dim (the per-head QK-norm scale common in video DiTs).  Gates are always
N(0, 1).  Finally every tensor is cast to the workload dtype.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch

SEED_BASE = 20261202


@dataclass(frozen=True)
class Workload:
    name: str
    B: int  # batch
    F: int  # latent frames
    P: int  # tokens per frame
    H: int  # heads
    d: int  # head_dim
    T: int  # text tokens
    C: int  # frames per chunk
    dtype: str  # "fp32" or "bf16"
    dist: str  # "normal", "half" or "rms"
    index: int = 0

    @property
    def N(self) -> int:
        return self.F * self.P

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = [
    Workload("tiny_fp32", 1, 15, 16, 2, 32, 8, 1, "fp32", "normal", 0),
    Workload("small_bf16", 1, 15, 256, 8, 64, 64, 1, "bf16", "half", 1),
    Workload("chunk5_bf16", 1, 45, 1024, 16, 128, 256, 5, "bf16", "normal", 2),
    Workload("768p_bf16", 1, 15, 4032, 24, 128, 512, 1, "bf16", "rms", 3),
    Workload("768p_long_bf16", 1, 60, 4032, 24, 128, 512, 5, "bf16", "rms", 4),
    # profiling shape: the 768p latent with 4 of its 24 heads (inputs still larger than L2)
    Workload("768p_h4_bf16", 1, 15, 4032, 4, 128, 512, 1, "bf16", "rms", 5),
    # profiling shape: half the heads (every SM gets half the steady-state work of the full launch)
    Workload("768p_h12_bf16", 1, 15, 4032, 12, 128, 512, 1, "bf16", "rms", 6),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def _shape(x: torch.Tensor, dist: str) -> torch.Tensor:
    if dist == "half":
        return x * 0.5
    if dist == "rms":
        return x / x.pow(2).mean(dim=-1, keepdim=True).sqrt()
    return x


def make_inputs(w: Workload, seed: int | None = None) -> dict[str, torch.Tensor]:
    """Host tensors q, k, v [B,N,H,d], text_k, text_v [B,T,H,d], gate_s,
    gate_l [B,N,H,d] in the workload dtype, drawn as described above."""
    g = torch.Generator("cpu").manual_seed(w.seed if seed is None else seed)
    vid = (w.B, w.N, w.H, w.d)
    txt = (w.B, w.T, w.H, w.d)
    out = {}
    for name, shp, shaped in (("q", vid, True), ("k", vid, True), ("v", vid, True),
                              ("text_k", txt, True), ("text_v", txt, True),
                              ("gate_s", vid, False), ("gate_l", vid, False)):
        x = torch.randn(shp, generator=g, dtype=torch.float32)
        if shaped:
            x = _shape(x, w.dist)
        out[name] = x.to(w.torch_dtype).contiguous()
    return out


def as_float64_numpy(inputs: dict[str, torch.Tensor]) -> dict:
    """The exact stored values of each input, widened to float64 numpy."""
    return {k: t.to(torch.float64).numpy() for k, t in inputs.items()}
