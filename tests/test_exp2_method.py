"""The FMA-pipe exponential of the softmax kernel, checked as a method.

The kernel evaluates part of its 2^x with Cody-Waite style range reduction
(x = n + f, n = round(x) by the 1.5 * 2^23 magic-number addition), a degree-3
polynomial for 2^f on [-1/2, 1/2] (coefficients fitted by
csrc/exp2_poly.py) and an exponent-field add for 2^n.  This replays those
float32 steps in numpy and bounds the relative error against the exact 2^x
(float64), and checks that the kernel source carries the fitted coefficients.
"""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "video_diffusion_hybrid_sparse_b200", "csrc")


def load_fit():
    spec = importlib.util.spec_from_file_location("exp2_poly", os.path.join(CSRC, "exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def exp2_steps(x, c):
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.full_like(f, np.float32(c[3]))
    for k in (2, 1, 0):
        p = (p * f + np.float32(c[k])).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.astype(np.int32).view(np.float32)


def test_polynomial_relative_error_bound():
    m = load_fit()
    c = m.fit().astype(np.float32)
    x = np.linspace(-120.0, 8.0, 400001, dtype=np.float32)
    got = exp2_steps(x, c).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4  # far below bf16's 2^-9, the precision P is stored in


def test_clamped_tail_is_tiny_and_finite():
    c = load_fit().fit().astype(np.float32)
    y = exp2_steps(np.array([-np.inf, -1e30, -200.0, -126.0], np.float32), c)
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 2e-38)


def test_kernel_source_uses_fitted_coefficients():
    c = load_fit().fit().astype(np.float32)
    src = open(os.path.join(CSRC, "sm100.cuh")).read()
    body = src[src.index("float exp2_fma"):]
    body = body[:body.index("}")]
    nums = [np.float32(float(v)) for v in re.findall(r"(\d\.\d+)f", body)]
    for k in range(4):
        assert any(v == c[k] for v in nums), f"coefficient c{k} differs from the fit"
