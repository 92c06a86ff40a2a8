"""Accuracy of the CUDA path against the fp64 oracle on the five configurations
(run on a GPU machine: ``python tests/accuracy_report.py``).  Prints one line per
configuration: max-abs and relative-L2 error of ``out``, the largest |out| and
the location of the largest error.  Small shapes are compared on the whole
output; the large ones on sampled rows (chunk edges, ragged tile tails,
random rows) of sampled heads, the same rows the GPU parity tests use."""
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from oracle import hybrid_attn as O  # noqa: E402
from test_parity_gpu import sample_rows  # noqa: E402
from video_diffusion_hybrid_sparse_b200 import binding as vb  # noqa: E402
from video_diffusion_hybrid_sparse_b200.workloads import BY_NAME, make_inputs  # noqa: E402


def stats(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    i = np.unravel_index(np.argmax(err), err.shape)
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    return float(err[i]), rel, float(np.abs(got).max()), tuple(int(x) for x in i)


def main():
    for name, heads in [("tiny_fp32", None), ("small_bf16", None), ("chunk5_bf16", [0, 15]),
                        ("768p_bf16", [0, 23]), ("768p_long_bf16", [7])]:
        w = BY_NAME[name]
        inputs = make_inputs(w)
        dev = {k: t.cuda() for k, t in inputs.items()}
        out = vb.hybrid_attn_fwd(dev["q"], dev["k"], dev["v"], dev["text_k"], dev["text_v"], dev["gate_s"],
                                 dev["gate_l"], frames=w.F, chunk_frames=w.C)
        torch.cuda.synchronize()
        del dev
        if heads is None:
            x = {k: t.to(torch.float64).numpy() for k, t in inputs.items()}
            prob = O.Problem(B=w.B, F=w.F, P=w.P, H=w.H, d=w.d, T=w.T, C=w.C)
            ref = O.hybrid_attn(x["q"], x["k"], x["v"], x["text_k"], x["text_v"], x["gate_s"], x["gate_l"],
                                prob)["out"]
            got = out.float().cpu().numpy()
            where = "whole output"
        else:
            rows = sample_rows(w, np.random.default_rng(7))
            prob = O.Problem(B=1, F=w.F, P=w.P, H=1, d=w.d, T=w.T, C=w.C)
            refs, gots = [], []
            for h in heads:
                x = {k: t[:, :, h:h + 1, :].to(torch.float64).numpy() for k, t in inputs.items()}
                refs.append(O.hybrid_attn_rows(x["q"], x["k"], x["v"], x["text_k"], x["text_v"], x["gate_s"],
                                               x["gate_l"], prob, 0, 0, rows)["out"])
                gots.append(out[0, torch.from_numpy(rows).cuda(), h, :].float().cpu().numpy())
            ref, got = np.stack(refs), np.stack(gots)
            where = f"{len(rows)} sampled rows x heads {heads}"
        mx, rel, amax, at = stats(got, ref)
        print(f"{name}: max-abs {mx:.3e}  rel-L2 {rel:.3e}  max|out| {amax:.3f}  worst at {at}  ({where})", flush=True)


if __name__ == "__main__":
    main()
