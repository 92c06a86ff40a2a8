"""Independent formulations used only to pin the oracle (TEST INFRASTRUCTURE).

Nothing here is used by the product path.  Each function computes a piece of
the hybrid attention a second way, from a token-level predicate rather than
from the oracle's frame lists, so that a slip in one of them (a wrong window
edge, an anchor counted twice, a text term dropped or doubled, a transposed
operand) makes the two disagree:

* :func:`dense_masked_softmax` - the softmax branch as ordinary dense
  attention over all N + T keys with a boolean mask, evaluated by the library
  routine ``torch.nn.functional.scaled_dot_product_attention`` in float64.
  Mask predicate (VDN-H3 article, section 双分支混合注意力机制): query token i
  may read key token j when their chunks differ by at most one, or when j lies
  in the first or last latent frame; every text key is readable.  Under the
  GLOBAL anchor reading a query in the first or last frame reads every key.
* :func:`pairwise_linear` - the linear branch without any state: for each
  query, a weighted mean over every key outside the window and outside the
  anchors plus every text key taken once, with weights phi(q_i) . phi(k_j)
  (nothing for a GLOBAL anchor query).
"""
from __future__ import annotations

import numpy as np
import torch


def _token_frame_chunk(prob):
    n = np.arange(prob.N)
    frame = n // prob.P
    return frame, frame // prob.C


def _global_anchor_query(prob, frame) -> np.ndarray:
    mode = getattr(prob, "anchor_query_mode", "local")
    return ((frame == 0) | (frame == prob.F - 1)) & (mode == "global")


def softmax_mask(prob) -> np.ndarray:
    """bool [N, N + T]: True where query i reads key j in the softmax branch."""
    frame, chunk = _token_frame_chunk(prob)
    near = np.abs(chunk[:, None] - chunk[None, :]) <= 1
    anchor_key = (frame == 0) | (frame == prob.F - 1)
    video = near | anchor_key[None, :] | _global_anchor_query(prob, frame)[:, None]
    text = np.ones((prob.N, prob.T), dtype=bool)
    return np.concatenate([video, text], axis=1)


def linear_mask(prob) -> np.ndarray:
    """bool [N, N]: True where video key j is read by query i through a state."""
    frame, chunk = _token_frame_chunk(prob)
    far = np.abs(chunk[:, None] - chunk[None, :]) >= 2
    anchor_key = (frame == 0) | (frame == prob.F - 1)
    return far & ~anchor_key[None, :] & ~_global_anchor_query(prob, frame)[:, None]


def dense_masked_softmax(q, k, v, tk, tv, prob) -> np.ndarray:
    """o_s [B, N, H, d] via masked dense SDPA (float64, CPU)."""
    mask = torch.from_numpy(softmax_mask(prob))
    out = np.zeros((prob.B, prob.N, prob.H, prob.d))
    for b in range(prob.B):
        keys = np.concatenate([k[b], tk[b]], axis=0)  # [N+T, H, d]
        vals = np.concatenate([v[b], tv[b]], axis=0)
        qt = torch.from_numpy(np.ascontiguousarray(np.asarray(q[b], np.float64).transpose(1, 0, 2)))
        kt = torch.from_numpy(np.ascontiguousarray(np.asarray(keys, np.float64).transpose(1, 0, 2)))
        vt = torch.from_numpy(np.ascontiguousarray(np.asarray(vals, np.float64).transpose(1, 0, 2)))
        o = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, attn_mask=mask, scale=prob.softmax_scale)
        out[b] = o.numpy().transpose(1, 0, 2)
    return out


def _elu_plus_one(x) -> np.ndarray:
    return torch.nn.functional.elu(torch.from_numpy(np.asarray(x, np.float64))).numpy() + 1.0


def pairwise_linear(q, k, v, tk, tv, prob) -> np.ndarray:
    """o_l [B, N, H, d] with no states: per query i,

        o_l[i] = (sum_j w_ij v_j + sum_t w_it tv_t) / (sum_j w_ij + sum_t w_it)

    over video keys j of :func:`linear_mask` and every text token t once,
    w = phi(q) . phi(k); zero when there is no such key."""
    lm = linear_mask(prob).astype(np.float64)
    out = np.zeros((prob.B, prob.N, prob.H, prob.d))
    for b in range(prob.B):
        for h in range(prob.H):
            fq = _elu_plus_one(q[b, :, h, :])
            fk = _elu_plus_one(k[b, :, h, :])
            w = (fq @ fk.T) * lm  # [N, N]
            num = w @ np.asarray(v[b, :, h, :], np.float64)
            den = w.sum(axis=1)
            if prob.T:
                ftk = _elu_plus_one(tk[b, :, h, :])
                wt = (fq @ ftk.T) * (~_global_anchor_query(prob, np.arange(prob.N) // prob.P))[:, None]
                num = num + wt @ np.asarray(tv[b, :, h, :], np.float64)
                den = den + wt.sum(axis=1)
            frame = np.arange(prob.N) // prob.P
            has = ((lm.sum(axis=1) > 0) | (prob.T > 0)) & ~_global_anchor_query(prob, frame)
            o = np.zeros_like(num)
            o[has] = num[has] / den[has, None]
            out[b, :, h, :] = o
    return out
