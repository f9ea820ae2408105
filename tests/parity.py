"""Element-by-element comparison of the CUDA path with the float64 oracle.

Tolerances (the stated parity bar for this path): O as bf16 upcast to f64
against the oracle's O: max-abs <= 2e-2 and mean-abs <= 2e-3; lse: the relative
bound 1e-3 read as |delta| <= 1e-3 * max(1, |lse_ref|), because a causal row 0
can have lse = scale * q0.k0 close to zero, where a purely relative bound is
ill-posed.  "Exact" means the same operation, not bit-identical execution
("FlashAttention -- avoid writing the giant intermediate", "Exact attention
has limits").
"""
from __future__ import annotations

import numpy as np

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_TOL = 1e-3


def compare(o_dev, lse_dev, o_ref, lse_ref):
    """o_dev/lse_dev: float64 numpy arrays shaped like o_ref/lse_ref."""
    o_dev = np.asarray(o_dev, dtype=np.float64)
    lse_dev = np.asarray(lse_dev, dtype=np.float64)
    err = np.abs(o_dev - o_ref)
    lerr = np.abs(lse_dev - lse_ref)
    return {
        "o_max_abs": float(np.max(err)) if err.size else 0.0,
        "o_mean_abs": float(np.mean(err)) if err.size else 0.0,
        "lse_max_scaled": float(np.max(lerr / np.maximum(1.0, np.abs(lse_ref)))) if lerr.size else 0.0,
        "lse_max_rel": float(np.max(lerr / np.maximum(1e-30, np.abs(lse_ref)))) if lerr.size else 0.0,
        "finite": bool(np.all(np.isfinite(o_dev)) and np.all(np.isfinite(lse_dev))),
    }


def ok(stats) -> bool:
    return (stats["finite"] and stats["o_max_abs"] <= O_MAX_ABS
            and stats["o_mean_abs"] <= O_MEAN_ABS and stats["lse_max_scaled"] <= LSE_TOL)


def assert_parity(stats, label=""):
    assert ok(stats), f"parity failed {label}: {stats}"
