"""The head-parallel wrapper on the GPU: one NCCL rank (world size 1, the
only size a one-GPU machine can run), the real C-ABI call underneath.  With one
rank the two all-to-alls are permutations onto itself, so the result must
equal the direct call bit for bit; the multi-rank partition is covered on the
host (test_ulysses_host.py)."""
import os

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_sequence_sharded_wrapper_equals_direct_call_nccl_world1():
    import torch.distributed as dist

    from video_diffusion_hybrid_sparse_b200 import binding as vb
    from video_diffusion_hybrid_sparse_b200 import ulysses
    from video_diffusion_hybrid_sparse_b200.workloads import BY_NAME, make_inputs

    w = BY_NAME["small_bf16"]
    x = {k: t.cuda() for k, t in make_inputs(w).items()}
    torch.cuda.set_device(0)
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", str(29900 + os.getpid() % 90))
    own = not dist.is_initialized()
    if own:
        dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        args = [x[k] for k in ("q", "k", "v", "text_k", "text_v", "gate_s", "gate_l")]
        direct = vb.hybrid_attn_fwd(*args, frames=w.F, chunk_frames=w.C)
        split = ulysses.hybrid_attn_fwd_seq_sharded(*args, frames=w.F, chunk_frames=w.C)
        torch.cuda.synchronize()
        assert torch.equal(direct, split)
    finally:
        if own:
            dist.destroy_process_group()
