"""Head-parallel hybrid attention across ranks (one process per GPU).

The heads of the hybrid attention are independent: every head has its own
softmax branch, its own forward/backward states and its own RMSNorm (over
head_dim, per (token, head)), so a rank that holds all tokens of a subset of
the heads computes those heads completely, with no communication.  Callers
that shard the sequence instead (each rank holding a contiguous block of the
frame-major tokens of every head, as in sequence-parallel video denoisers)
re-shard with one all-to-all before the call and one after it (the
Ulysses scheme the VDN-H3 article's multi-GPU launch script names):

    sequence-sharded [B, N/R, H, d]  --all-to-all-->  head-sharded [B, N, H/R, d]
    hybrid attention on H/R heads (the C-ABI call, this GPU only)
    head-sharded [B, N, H/R, d]      --all-to-all-->  sequence-sharded [B, N/R, H, d]

The all-to-alls are ``torch.distributed.all_to_all_single`` (NCCL between
GPUs, gloo on the host); the packing around them is a copy into the layout
the exchange needs.  Text tokens are keys and values only: every rank holds
all of them and takes its heads' slice.  The attention itself is whatever
``attn_fn`` computes on the head-sharded tensors; by default the library's
``hybrid_attn_fwd``.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def head_block(H: int, world: int, rank: int) -> tuple[int, int]:
    """The heads [h0, h1) that rank `rank` of `world` computes (H % world == 0)."""
    if H % world:
        raise ValueError(f"{H} heads do not split evenly over {world} ranks")
    n = H // world
    return rank * n, (rank + 1) * n


def seq_to_heads(x: torch.Tensor, group=None) -> torch.Tensor:
    """[B, N/R, H, d] (this rank's tokens, all heads) -> [B, N, H/R, d] (all
    tokens, this rank's heads), ranks' token blocks in rank order."""
    R = dist.get_world_size(group)
    B, n, H, d = x.shape
    if H % R:
        raise ValueError(f"{H} heads do not split evenly over {R} ranks")
    hr = H // R
    send = x.reshape(B, n, R, hr, d).permute(2, 0, 1, 3, 4).contiguous()  # [R dest, B, n, hr, d]
    recv = torch.empty_like(send)  # [R source, B, n, hr, d]
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 0, 2, 3, 4).reshape(B, R * n, hr, d)


def heads_to_seq(y: torch.Tensor, group=None) -> torch.Tensor:
    """Inverse of :func:`seq_to_heads`: [B, N, H/R, d] -> [B, N/R, H, d]."""
    R = dist.get_world_size(group)
    B, N, hr, d = y.shape
    if N % R:
        raise ValueError(f"{N} tokens do not split evenly over {R} ranks")
    n = N // R
    send = y.reshape(B, R, n, hr, d).permute(1, 0, 2, 3, 4).contiguous()  # [R dest (token block), B, n, hr, d]
    recv = torch.empty_like(send)  # [R source (head block), B, n, hr, d]
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 2, 0, 3, 4).reshape(B, n, R * hr, d)


def _default_attn(q, k, v, text_k, text_v, gate_s, gate_l, *, frames, chunk_frames, **kw):
    from . import binding

    return binding.hybrid_attn_fwd(q, k, v, text_k, text_v, gate_s, gate_l, frames=frames,
                                   chunk_frames=chunk_frames, **kw)


def hybrid_attn_fwd_seq_sharded(q, k, v, text_k, text_v, gate_s, gate_l, *, frames: int, chunk_frames: int,
                                group=None, attn_fn=None, rms_weight=None, **kw) -> torch.Tensor:
    """The whole hybrid attention for sequence-sharded inputs.

    q, k, v, gate_s, gate_l: [B, N/R, H, d], this rank's block of the
    frame-major tokens (rank r holds tokens r*N/R .. (r+1)*N/R - 1); text_k,
    text_v: [B, T, H, d], the same on every rank; rms_weight: [H, d] or None.
    Returns this rank's block of the output, [B, N/R, H, d].  Every rank
    calls it with the same shapes (collective)."""
    R = dist.get_world_size(group)
    rank = dist.get_rank(group)
    H = q.shape[2]
    h0, h1 = head_block(H, R, rank)
    attn = attn_fn or _default_attn
    qh, kh, vh, gsh, glh = (seq_to_heads(t, group) for t in (q, k, v, gate_s, gate_l))
    tk, tv = (t[:, :, h0:h1].contiguous() for t in (text_k, text_v))
    gamma = None if rms_weight is None else rms_weight[h0:h1].contiguous()
    out_h = attn(qh, kh, vh, tk, tv, gsh, glh, frames=frames, chunk_frames=chunk_frames, rms_weight=gamma, **kw)
    return heads_to_seq(out_h, group)
