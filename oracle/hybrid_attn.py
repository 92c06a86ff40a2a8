"""Plain fp64 CPU oracle for the VDN-H3 dual-branch hybrid attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
executes this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it.  It shares no code, constant or helper
with the CUDA library.

Source of every step: the VDN-H3 article "VDN-Minimax-H3 ... 11.23 秒生成
14.4 秒 768p 视频" (tahou.com, article 216474224916730885), section
"技术核心设计 / 双分支混合注意力机制" (dual-branch hybrid attention) and section
"自适应门控融合双分支输出" (adaptive gated fusion).  What those sections fix:

* video-token attention is split into an exact local softmax branch and a
  bidirectional linear-attention branch for far context;
* the local branch works on chunks of consecutive latent frames; a chunk
  attends to itself and its two neighbouring chunks; the first and last frames
  are global anchors that every frame reads;
* the linear branch keeps a forward state that sums the context before the
  local window and a backward state that sums the context after it; both leave
  out the window frames and the anchor frames.  Worked example on the page:
  for latent frame 7 the softmax branch keeps frames 6, 7, 8 and anchors 0 and
  14, the forward state covers frames 1-5 and the backward state frames 9-13;
* text tokens are read by every frame in the softmax branch; in the linear
  branch the text is written at half weight into each of the two states, so
  that it counts once when the two sides are read together;
* each branch gets its own input-dependent sigmoid gate; the linear output is
  RMS-normalised before its element-wise gate; the two are summed.

Readings of points the page leaves open:
chunk size C is a parameter (5 in the chunking sentence, 1 in the frame-7
example); the window is clipped at the sequence ends; anchor frames as queries
follow the same rule as every other frame (LOCAL, the default) -- the other
reading of "the first and last frames also interact with the other frames",
GLOBAL, where an anchor query attends through the softmax branch to every
frame and reads nothing through the states, is available as
``anchor_query_mode="global"``; the feature map is
phi(x) = elu(x) + 1; the softmax scale is 1/sqrt(d); the two directional
states are summed before one normalised read (numerator phi(q)^T (S_F + S_B),
denominator phi(q) . (z_F + z_B)), which is the reading under which a half
write into each side counts the text once; an empty state (no text and no
frames) reads as zero; RMSNorm is over head_dim per (token, head) with
eps = 1e-6 and an optional per-head weight gamma; gates are element-wise
logits supplied as inputs; text tokens are keys/values only.  The two gated
branch terms sigmoid(g_s) * o_s and sigmoid(g_l) * r are also returned
separately (the SPLIT output, for callers that apply a projection per branch
before summing, as the fusion section's per-branch outputs suggest).

Layout: video tensors are [B, N, H, d] with N = F*P frame-major tokens (token n
lies in frame n // P); text tensors are [B, T, H, d]; gates [B, N, H, d].
All arithmetic is numpy float64.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

# --------------------------------------------------------------------------
# Problem description
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class Problem:
    """Sizes of one hybrid-attention call (names follow the page's setting:
    latent frames, tokens per frame, heads, head_dim, text tokens, chunk)."""

    B: int  # batch
    F: int  # latent frames
    P: int  # tokens per latent frame
    H: int  # heads
    d: int  # head_dim
    T: int  # text tokens
    C: int  # frames per chunk
    scale: float | None = None  # softmax scale; None -> 1/sqrt(d)
    eps: float = 1e-6  # RMSNorm epsilon
    anchor_query_mode: str = "local"  # "local" or "global" (see module docstring)

    @property
    def N(self) -> int:
        return self.F * self.P

    @property
    def n_chunks(self) -> int:
        return self.F // self.C

    @property
    def softmax_scale(self) -> float:
        return (1.0 / np.sqrt(self.d)) if self.scale is None else float(self.scale)

    def check(self) -> None:
        if min(self.B, self.F, self.P, self.H, self.d, self.C) < 1 or self.T < 0:
            raise ValueError("sizes must be positive (T >= 0)")
        if self.F % self.C:
            raise ValueError("frames must be a whole number of chunks")
        if self.anchor_query_mode not in ("local", "global"):
            raise ValueError("anchor_query_mode is 'local' or 'global'")


# --------------------------------------------------------------------------
# Membership: which frame each query frame reads through which branch
# ("双分支混合注意力机制": chunked window, boundary anchors, linear memory)
# --------------------------------------------------------------------------


def anchor_frames(F: int) -> list[int]:
    """First and last latent frame are the boundary anchors (one frame if F == 1)."""
    return sorted({0, F - 1})


def chunk_of(f: int, C: int) -> int:
    return f // C


def window_frames(f: int, F: int, C: int) -> list[int]:
    """Frames of the query's chunk and of its two neighbouring chunks, clipped
    at the ends of the sequence (the window is not shifted at the edges)."""
    n_chunks = F // C
    c = chunk_of(f, C)
    lo = max(0, c - 1)
    hi = min(n_chunks - 1, c + 1)
    return list(range(lo * C, (hi + 1) * C))


def global_anchor_query(f: int, F: int, mode: str) -> bool:
    """True when query frame f is an anchor that, under the GLOBAL reading,
    attends to every frame through the softmax branch."""
    return mode == "global" and f in anchor_frames(F)


def softmax_frames(f: int, F: int, C: int, mode: str = "local") -> list[int]:
    """Frames read exactly by the softmax branch: the window plus the anchors,
    each frame once (every frame for a GLOBAL anchor query)."""
    if global_anchor_query(f, F, mode):
        return list(range(F))
    return sorted(set(window_frames(f, F, C)) | set(anchor_frames(F)))


def forward_frames(f: int, F: int, C: int, mode: str = "local") -> list[int]:
    """Frames summed by the forward state: every chunk before the window,
    anchors excluded (none for a GLOBAL anchor query)."""
    if global_anchor_query(f, F, mode):
        return []
    c = chunk_of(f, C)
    anchors = set(anchor_frames(F))
    return [g for g in range(F) if chunk_of(g, C) <= c - 2 and g not in anchors]


def backward_frames(f: int, F: int, C: int, mode: str = "local") -> list[int]:
    """Frames summed by the backward state: every chunk after the window,
    anchors excluded (none for a GLOBAL anchor query)."""
    if global_anchor_query(f, F, mode):
        return []
    c = chunk_of(f, C)
    anchors = set(anchor_frames(F))
    return [g for g in range(F) if chunk_of(g, C) >= c + 2 and g not in anchors]


SOFTMAX, FORWARD, BACKWARD = 1, 2, 3


def membership_table(F: int, C: int, mode: str = "local") -> np.ndarray:
    """uint8 [F, F]: entry (f, g) says how query frame f reads key frame g:
    1 = softmax branch, 2 = forward state, 3 = backward state.  Every key frame
    is read through exactly one branch ("其余帧则进入线性记忆模块")."""
    if F % C:
        raise ValueError("frames must be a whole number of chunks")
    table = np.zeros((F, F), dtype=np.uint8)
    for f in range(F):
        for g in softmax_frames(f, F, C, mode):
            table[f, g] = SOFTMAX
        for g in forward_frames(f, F, C, mode):
            table[f, g] = FORWARD
        for g in backward_frames(f, F, C, mode):
            table[f, g] = BACKWARD
    return table


# --------------------------------------------------------------------------
# Softmax branch: exact attention over window + anchors + text
# --------------------------------------------------------------------------


def _frame_rows(frames: list[int], P: int) -> np.ndarray:
    if not frames:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(g * P, (g + 1) * P) for g in frames])


def softmax_branch_rows(q, k, v, tk, tv, prob: Problem, b: int, h: int, rows) -> np.ndarray:
    """o_s for the query tokens ``rows`` (indices into N) of batch b, head h.

    o_s[i] = sum_j softmax_j(scale * q_i . k_j) v_j over the keys of the
    softmax frames of i's frame plus all T text tokens; exact two-pass softmax
    (max subtraction, then normalisation) in float64."""
    rows = np.asarray(rows, dtype=np.int64)
    out = np.zeros((rows.size, prob.d), dtype=np.float64)
    frames_of_rows = rows // prob.P
    for f in np.unique(frames_of_rows):
        sel = np.nonzero(frames_of_rows == f)[0]
        key_rows = _frame_rows(softmax_frames(int(f), prob.F, prob.C, prob.anchor_query_mode), prob.P)
        keys = np.concatenate([k[b, key_rows, h, :], tk[b, :, h, :]], axis=0).astype(np.float64)
        vals = np.concatenate([v[b, key_rows, h, :], tv[b, :, h, :]], axis=0).astype(np.float64)
        qf = q[b, rows[sel], h, :].astype(np.float64)
        scores = prob.softmax_scale * (qf @ keys.T)
        scores -= scores.max(axis=1, keepdims=True)
        w = np.exp(scores)
        w /= w.sum(axis=1, keepdims=True)
        out[sel] = w @ vals
    return out


def softmax_branch(q, k, v, tk, tv, prob: Problem) -> np.ndarray:
    """o_s for every video query: [B, N, H, d] float64."""
    o = np.zeros((prob.B, prob.N, prob.H, prob.d), dtype=np.float64)
    all_rows = np.arange(prob.N)
    for b in range(prob.B):
        for h in range(prob.H):
            o[b, :, h, :] = softmax_branch_rows(q, k, v, tk, tv, prob, b, h, all_rows)
    return o


# --------------------------------------------------------------------------
# Linear branch: per-frame states, forward/backward states, readout
# --------------------------------------------------------------------------


def phi(x):
    """Feature map phi(x) = elu(x) + 1: x + 1 for x > 0, exp(x) otherwise."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def frame_states(k, v, prob: Problem, b: int, h: int):
    """Per latent frame f: S_f = sum_{n in f} phi(k_n) v_n^T  [F, d, d] and
    z_f = sum_{n in f} phi(k_n)  [F, d]."""
    S = np.zeros((prob.F, prob.d, prob.d))
    z = np.zeros((prob.F, prob.d))
    for f in range(prob.F):
        fk = phi(k[b, f * prob.P:(f + 1) * prob.P, h, :])
        fv = v[b, f * prob.P:(f + 1) * prob.P, h, :].astype(np.float64)
        S[f] = fk.T @ fv
        z[f] = fk.sum(axis=0)
    return S, z


def text_state(tk, tv, b: int, h: int, d: int):
    """S_t = sum_t phi(tk_t) tv_t^T, z_t = sum_t phi(tk_t)."""
    if tk.shape[1] == 0:
        return np.zeros((d, d)), np.zeros(d)
    fk = phi(tk[b, :, h, :])
    return fk.T @ tv[b, :, h, :].astype(np.float64), fk.sum(axis=0)


def directional_states(S, z, S_t, z_t, prob: Problem, text_weights=(0.5, 0.5)):
    """Forward and backward states of every chunk, summed directly over the
    membership sets (no scan):

        S_F(c) = w_F * S_t + sum_{g in forward_frames}  S_g
        S_B(c) = w_B * S_t + sum_{g in backward_frames} S_g

    and the same for z.  ``text_weights`` = (w_F, w_B) is (1/2, 1/2) on the
    page ("文本会先按一半比例分别写入正向和反向记忆状态"); other values exist
    only so that tests can show the count-once property."""
    n_chunks = prob.n_chunks
    wF, wB = text_weights
    SF = np.zeros((n_chunks, prob.d, prob.d))
    SB = np.zeros_like(SF)
    zF = np.zeros((n_chunks, prob.d))
    zB = np.zeros_like(zF)
    for c in range(n_chunks):
        f = c * prob.C  # any frame of the chunk: membership is per chunk
        SF[c] = wF * S_t + sum((S[g] for g in forward_frames(f, prob.F, prob.C)), np.zeros((prob.d, prob.d)))
        zF[c] = wF * z_t + sum((z[g] for g in forward_frames(f, prob.F, prob.C)), np.zeros(prob.d))
        SB[c] = wB * S_t + sum((S[g] for g in backward_frames(f, prob.F, prob.C)), np.zeros((prob.d, prob.d)))
        zB[c] = wB * z_t + sum((z[g] for g in backward_frames(f, prob.F, prob.C)), np.zeros(prob.d))
    return SF, zF, SB, zB


def state_token_count(c: int, prob: Problem) -> int:
    """Number of key tokens held by the two states of chunk c (text counted once)."""
    f = c * prob.C
    n_frames = len(forward_frames(f, prob.F, prob.C)) + len(backward_frames(f, prob.F, prob.C))
    return prob.T + prob.P * n_frames


def linear_readout_rows(q, SF, zF, SB, zB, prob: Problem, b: int, h: int, rows) -> np.ndarray:
    """o_l for query tokens ``rows``: one normalised read of the summed
    states, phi(q)^T (S_F + S_B) / (phi(q) . (z_F + z_B)); zero when the
    states hold no token, and zero for GLOBAL anchor queries (they read
    nothing through the states)."""
    rows = np.asarray(rows, dtype=np.int64)
    out = np.zeros((rows.size, prob.d))
    frames = rows // prob.P
    chunks = frames // prob.C
    reads = np.array([not global_anchor_query(int(f), prob.F, prob.anchor_query_mode) for f in frames], dtype=bool)
    for c in np.unique(chunks):
        sel = np.nonzero((chunks == c) & reads)[0]
        if sel.size == 0 or state_token_count(int(c), prob) == 0:
            continue
        fq = phi(q[b, rows[sel], h, :])
        num = fq @ (SF[c] + SB[c])
        den = fq @ (zF[c] + zB[c])
        out[sel] = num / den[:, None]
    return out


def linear_branch(q, k, v, tk, tv, prob: Problem, text_weights=(0.5, 0.5)):
    """o_l for every video query [B, N, H, d], plus the per-(b, h) states."""
    o = np.zeros((prob.B, prob.N, prob.H, prob.d))
    states = {}
    rows = np.arange(prob.N)
    for b in range(prob.B):
        for h in range(prob.H):
            S, z = frame_states(k, v, prob, b, h)
            S_t, z_t = text_state(tk, tv, b, h, prob.d)
            SF, zF, SB, zB = directional_states(S, z, S_t, z_t, prob, text_weights)
            o[b, :, h, :] = linear_readout_rows(q, SF, zF, SB, zB, prob, b, h, rows)
            states[(b, h)] = dict(S=S, z=z, S_t=S_t, z_t=z_t, SF=SF, zF=zF, SB=SB, zB=zB)
    return o, states


# --------------------------------------------------------------------------
# Gated fusion ("自适应门控融合双分支输出")
# --------------------------------------------------------------------------


def rms_norm(x, eps: float, gamma=None):
    """RMSNorm over the last axis (head_dim): x / sqrt(mean(x^2) + eps) * gamma."""
    x = np.asarray(x, dtype=np.float64)
    r = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    if gamma is not None:
        r = r * gamma
    return r


def sigmoid(x):
    """Logistic sigmoid 1 / (1 + exp(-x))."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def gated_terms(o_s, r, g_s, g_l):
    """The two gated branch terms (sigmoid(g_s) * o_s, sigmoid(g_l) * r): the
    SPLIT output."""
    return sigmoid(g_s) * o_s, sigmoid(g_l) * r


def merge(o_s, r, g_s, g_l):
    """out = sigmoid(g_s) * o_s + sigmoid(g_l) * r, element-wise."""
    return sigmoid(g_s) * o_s + sigmoid(g_l) * r


def hybrid_attn(q, k, v, tk, tv, g_s, g_l, prob: Problem, gamma=None, text_weights=(0.5, 0.5)):
    """Whole call.  Returns a dict with out, o_s, o_l, r, and the SPLIT
    terms out_s = sigmoid(g_s) * o_s, out_l = sigmoid(g_l) * r (all
    [B, N, H, d] float64), the per-(b, h) states and the membership table.

    ``gamma`` is None (ones) or [H, d]."""
    prob.check()
    o_s = softmax_branch(q, k, v, tk, tv, prob)
    o_l, states = linear_branch(q, k, v, tk, tv, prob, text_weights)
    g = None if gamma is None else np.asarray(gamma, dtype=np.float64)[None, None, :, :]
    r = rms_norm(o_l, prob.eps, g)
    out = merge(o_s, r, g_s.astype(np.float64), g_l.astype(np.float64))
    out_s, out_l = gated_terms(o_s, r, g_s.astype(np.float64), g_l.astype(np.float64))
    return dict(out=out, o_s=o_s, o_l=o_l, r=r, out_s=out_s, out_l=out_l, states=states,
                membership=membership_table(prob.F, prob.C, prob.anchor_query_mode))


def hybrid_attn_rows(q, k, v, tk, tv, g_s, g_l, prob: Problem, b: int, h: int, rows,
                     gamma=None, frame_state_cache=None):
    """``out`` for a subset of query rows of one (batch, head), for checks at
    sizes where the whole call is too slow on the host.  Same steps as
    :func:`hybrid_attn`."""
    rows = np.asarray(rows, dtype=np.int64)
    o_s = softmax_branch_rows(q, k, v, tk, tv, prob, b, h, rows)
    if frame_state_cache is not None and (b, h) in frame_state_cache:
        S, z = frame_state_cache[(b, h)]
    else:
        S, z = frame_states(k, v, prob, b, h)
        if frame_state_cache is not None:
            frame_state_cache[(b, h)] = (S, z)
    S_t, z_t = text_state(tk, tv, b, h, prob.d)
    SF, zF, SB, zB = directional_states(S, z, S_t, z_t, prob)
    o_l = linear_readout_rows(q, SF, zF, SB, zB, prob, b, h, rows)
    g = None if gamma is None else np.asarray(gamma, dtype=np.float64)[h]
    r = rms_norm(o_l, prob.eps, g)
    gs, gl = g_s[b, rows, h, :].astype(np.float64), g_l[b, rows, h, :].astype(np.float64)
    out = merge(o_s, r, gs, gl)
    out_s, out_l = gated_terms(o_s, r, gs, gl)
    return dict(out=out, o_s=o_s, o_l=o_l, r=r, out_s=out_s, out_l=out_l)


# --------------------------------------------------------------------------
# Algorithmic work (used by the benchmark's roofline arithmetic)
# --------------------------------------------------------------------------


def softmax_pairs(prob: Problem) -> int:
    """Number of (query, key) pairs the softmax branch must score, per (b, h)."""
    total = 0
    for f in range(prob.F):
        total += prob.P * (prob.P * len(softmax_frames(f, prob.F, prob.C, prob.anchor_query_mode)) + prob.T)
    return total
