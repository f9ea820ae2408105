"""The polynomial the fused kernel uses for part of its exponentials: its
coefficients are re-derived here (Remez fit of 2^f on [-1/2, 1/2], minimax
relative error) and its error bound checked against the exact 2^x in float64,
with the kernel's float32 arithmetic replayed step by step in numpy."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_attention_124_b200", "csrc")


def _kernel_coeffs():
    text = open(os.path.join(CSRC, "fused_fwd.cuh")).read()
    return [np.float32(float(re.search(rf"EXP2_C{i} = ([0-9.eE+-]+)f;", text).group(1)))
            for i in range(4)]


def _fitter():
    spec = importlib.util.spec_from_file_location("gen", os.path.join(CSRC, "gen_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_coefficients_are_the_fitted_ones():
    coeffs, err = _fitter().remez()
    assert err < 1e-4
    for a, b in zip(_kernel_coeffs(), coeffs):
        assert a == np.float32(b)


def _kernel_exp2(x):
    """The kernel's steps in float32: clamp, round via 1.5*2^23, Horner, exponent add."""
    c0, c1, c2, c3 = _kernel_coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    M = np.float32(12582912.0)
    t = (x + M).astype(np.float32)
    n = (t - M).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = np.float32(c3) * f + c2          # the kernel's FMAs round once; float32 products
    q = (q.astype(np.float32) * f + c1).astype(np.float32)  # of numpy round twice, so the
    q = (q * f + c0).astype(np.float32)  # bound below leaves room for that
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_error_bound_over_the_range_the_kernel_feeds_it():
    x = np.concatenate([np.linspace(-124.9, 8.0, 2_000_001, dtype=np.float64),
                        np.arange(-124, 9, dtype=np.float64)])
    got = _kernel_exp2(x.astype(np.float32)).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1.5e-4, rel.max()


def test_clamp_keeps_results_normal_and_tiny():
    x = np.array([-1e30, -200.0, -126.0, -125.0], dtype=np.float32)
    y = _kernel_exp2(x)
    assert np.all(y > 0) and np.all(y <= np.float32(2.0 ** -124))
    assert np.all(np.isfinite(y))
