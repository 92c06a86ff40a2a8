"""Head-parallel call for sequence-sharded inputs (ulysses.py), on the host:
world size 2 over gloo.  The attention on each rank's heads is the fp64
oracle (injected as attn_fn; the library call needs a GPU), so the check is of
the partition and the two all-to-all re-shards: every rank's output block must
equal the oracle on the whole, unsharded problem."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import hybrid_attn as O
from video_diffusion_hybrid_sparse_b200 import ulysses

B, F, P, H, D, T, C = 1, 6, 8, 4, 32, 5, 1


def _inputs():
    g = torch.Generator("cpu").manual_seed(20261203)
    N = F * P
    x = {k: torch.randn((B, N, H, D), generator=g, dtype=torch.float64) for k in ("q", "k", "v", "gate_s", "gate_l")}
    x.update({k: torch.randn((B, T, H, D), generator=g, dtype=torch.float64) for k in ("text_k", "text_v")})
    gamma = torch.rand((H, D), generator=g, dtype=torch.float64) + 0.5
    return x, gamma


def _oracle_attn(q, k, v, text_k, text_v, gate_s, gate_l, *, frames, chunk_frames, rms_weight=None):
    n = q.shape[1]
    prob = O.Problem(B=q.shape[0], F=frames, P=n // frames, H=q.shape[2], d=q.shape[3], T=text_k.shape[1],
                     C=chunk_frames)
    a = [t.numpy() for t in (q, k, v, text_k, text_v, gate_s, gate_l)]
    out = O.hybrid_attn(*a, prob, gamma=None if rms_weight is None else rms_weight.numpy())["out"]
    return torch.from_numpy(out)


def _worker(rank, world, port, result):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, gamma = _inputs()
        n = F * P // world
        loc = {k: (t[:, rank * n:(rank + 1) * n].contiguous() if k not in ("text_k", "text_v") else t)
               for k, t in x.items()}
        # the re-shard alone is a permutation: there and back is the identity
        back = ulysses.heads_to_seq(ulysses.seq_to_heads(loc["q"]))
        assert torch.equal(back, loc["q"])
        h0, h1 = ulysses.head_block(H, world, rank)
        assert torch.equal(ulysses.seq_to_heads(loc["k"]), x["k"][:, :, h0:h1])
        out = ulysses.hybrid_attn_fwd_seq_sharded(loc["q"], loc["k"], loc["v"], loc["text_k"], loc["text_v"],
                                                  loc["gate_s"], loc["gate_l"], frames=F, chunk_frames=C,
                                                  attn_fn=_oracle_attn, rms_weight=gamma)
        full = _oracle_attn(*(x[k] for k in ("q", "k", "v", "text_k", "text_v", "gate_s", "gate_l")), frames=F,
                            chunk_frames=C, rms_weight=gamma)
        result[rank] = float((out - full[:, rank * n:(rank + 1) * n]).abs().max())
    finally:
        dist.destroy_process_group()


def test_sequence_sharded_call_equals_unsharded_oracle_gloo_world2():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    result = mgr.dict()
    port = 29700 + os.getpid() % 200
    procs = [ctx.Process(target=_worker, args=(r, 2, port, result)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    assert result[0] <= 1e-12 and result[1] <= 1e-12, dict(result)


def test_head_block_partition():
    assert [ulysses.head_block(24, 8, r) for r in range(8)] == [(3 * r, 3 * r + 3) for r in range(8)]
    with pytest.raises(ValueError):
        ulysses.head_block(24, 5, 0)
    # the blocks cover every head once
    cover = np.zeros(24, int)
    for r in range(4):
        h0, h1 = ulysses.head_block(24, 4, r)
        cover[h0:h1] += 1
    assert (cover == 1).all()
