"""Float64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and it
never calls the CUDA library; the two share only the seeded inputs from
``attn_inputs``.

The arithmetic lives in ``attn_oracle.c`` (plain C, float64, built with gcc
without fast-math or FMA contraction).  This module builds it on demand and
marshals numpy arrays.

Every function is pinned by ``tests/test_oracle_*.py`` against what the pages
fix (the two-score example, the Figure 4 rows, probabilities summing to one,
masked entries exactly zero, causal row 0), closed forms and a 50-digit brute
force on tiny inputs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into liboracle.so next to it (gcc, -O2, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
               "-shared", "-pthread", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        lib.oracle_softmax_row.restype = ctypes.c_double
        lib.oracle_softmax_row.argtypes = [P, P, ctypes.c_int, P]
        lib.oracle_head_scores_probs.restype = None
        lib.oracle_head_scores_probs.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                 ctypes.c_double, P, ctypes.c_int64, P, P, P]
        lib.oracle_attn_fwd_gqa.restype = ctypes.c_int
        lib.oracle_attn_fwd_gqa.argtypes = [P, P, P, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_double, P, ctypes.c_int64, P,
                                            ctypes.c_int64, P, P, ctypes.c_int]
        lib.oracle_head_fwd_f64.restype = None
        lib.oracle_head_fwd_f64.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_double, P, P]
        lib.oracle_head_bwd_f64.restype = None
        lib.oracle_head_bwd_f64.argtypes = [P, P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_double, P, P, P]
        lib.oracle_attn_bwd.restype = ctypes.c_int
        lib.oracle_attn_bwd.argtypes = [P, P, P, P, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_double, P, P, P, ctypes.c_int]
        lib.oracle_attn_decode.restype = ctypes.c_int
        lib.oracle_attn_decode.argtypes = [P, P, P, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_double, P, P]
        lib.oracle_attn_fwd.restype = ctypes.c_int
        lib.oracle_attn_fwd.argtypes = [P, P, P, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_double, P, ctypes.c_int64, P,
                                        ctypes.c_int64, P, P, ctypes.c_int]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def softmax_row(scores, masked=None):
    """Row softmax of ``scores`` (float64).  ``masked`` marks excluded entries.
    Returns (p, lse)."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    n = s.shape[0]
    m = None if masked is None else np.ascontiguousarray(masked, dtype=np.uint8)
    p = np.empty(n, dtype=np.float64)
    lse = _load().oracle_softmax_row(_ptr(s), _ptr(m), n, _ptr(p))
    return p, lse


def head_scores_probs(q_bits, k_bits, causal: bool, scale: float, rows=None):
    """S (scaled, unmasked), P and lse of one head.  q_bits/k_bits: uint16
    [T, D] bf16 patterns.  Returns (S, P, lse) for ``rows`` (default all)."""
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k = np.ascontiguousarray(k_bits, dtype=np.uint16)
    T, D = q.shape
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nr = T if r is None else r.shape[0]
    S = np.empty((nr, T), dtype=np.float64)
    P = np.empty((nr, T), dtype=np.float64)
    L = np.empty(nr, dtype=np.float64)
    _load().oracle_head_scores_probs(_ptr(q), _ptr(k), T, D, int(bool(causal)), float(scale),
                                     _ptr(r), nr, _ptr(S), _ptr(P), _ptr(L))
    return S, P, L


def attn_fwd(q_bits, k_bits, v_bits, causal: bool, scale: float, heads=None, rows=None,
             nthreads: int | None = None):
    """Attention forward in float64.

    q_bits/k_bits/v_bits: uint16 bf16 patterns shaped [..., T, D] (leading dims
    flattened to heads).  Returns (o, lse) with o [nheads, nrows, D] and
    lse [nheads, nrows] (natural log)."""
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v = np.ascontiguousarray(v_bits, dtype=np.uint16)
    T, D = q.shape[-2], q.shape[-1]
    BH = int(np.prod(q.shape[:-2])) if q.ndim > 2 else 1
    h = None if heads is None else np.ascontiguousarray(heads, dtype=np.int64)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nh = BH if h is None else h.shape[0]
    nr = T if r is None else r.shape[0]
    o = np.empty((nh, nr, D), dtype=np.float64)
    lse = np.empty((nh, nr), dtype=np.float64)
    rc = _load().oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), BH, T, D, int(bool(causal)),
                                 float(scale), _ptr(h), nh, _ptr(r), nr, _ptr(o), _ptr(lse),
                                 int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_attn_fwd: bad argument")
    return o, lse


def attn_fwd_gqa(q_bits, k_bits, v_bits, causal: bool, scale: float, heads=None, rows=None,
                 nthreads: int | None = None):
    """Grouped-query attention forward in float64.

    q_bits: uint16 [B, H, T, D]; k_bits/v_bits: uint16 [B, H_kv, T, D] with
    H % H_kv == 0; query head h reads K/V head h // (H // H_kv).  Returns
    (o, lse) with o [nheads, nrows, D] and lse [nheads, nrows] over flat query
    heads b*H + h."""
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v = np.ascontiguousarray(v_bits, dtype=np.uint16)
    B, H, T, D = q.shape
    H_kv = k.shape[1]
    h = None if heads is None else np.ascontiguousarray(heads, dtype=np.int64)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nh = B * H if h is None else h.shape[0]
    nr = T if r is None else r.shape[0]
    o = np.empty((nh, nr, D), dtype=np.float64)
    lse = np.empty((nh, nr), dtype=np.float64)
    rc = _load().oracle_attn_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), B, H, H_kv, T, D,
                                     int(bool(causal)), float(scale), _ptr(h), nh, _ptr(r), nr,
                                     _ptr(o), _ptr(lse), int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_attn_fwd_gqa: bad argument")
    return o, lse


def head_fwd_f64(q, k, v, causal: bool, scale: float):
    """Forward of one head on float64 inputs [T, D]; returns (o, lse)."""
    q, k, v = (np.ascontiguousarray(a, dtype=np.float64) for a in (q, k, v))
    T, D = q.shape
    o = np.empty((T, D))
    lse = np.empty(T)
    _load().oracle_head_fwd_f64(_ptr(q), _ptr(k), _ptr(v), T, D, int(bool(causal)),
                                float(scale), _ptr(o), _ptr(lse))
    return o, lse


def head_bwd_f64(q, k, v, dout, causal: bool, scale: float):
    """Gradients (dq, dk, dv) of one head on float64 inputs [T, D]."""
    q, k, v, g = (np.ascontiguousarray(a, dtype=np.float64) for a in (q, k, v, dout))
    T, D = q.shape
    dq, dk, dv = (np.empty((T, D)) for _ in range(3))
    _load().oracle_head_bwd_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(g), T, D, int(bool(causal)),
                                float(scale), _ptr(dq), _ptr(dk), _ptr(dv))
    return dq, dk, dv


def attn_bwd(q_bits, k_bits, v_bits, dout_bits, causal: bool, scale: float,
             nthreads: int | None = None):
    """Gradients in float64 from bf16 inputs.  q/dout [B, H, T, D], k/v
    [B, H_kv, T, D].  Returns dq [B, H, T, D] and dk, dv [B, H_kv, T, D]
    (summed over the query heads of each group)."""
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v = np.ascontiguousarray(v_bits, dtype=np.uint16)
    g = np.ascontiguousarray(dout_bits, dtype=np.uint16)
    B, H, T, D = q.shape
    H_kv = k.shape[1]
    dq = np.empty((B, H, T, D))
    dkh = np.empty((B, H, T, D))
    dvh = np.empty((B, H, T, D))
    rc = _load().oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), B, H, H_kv, T, D,
                                 int(bool(causal)), float(scale), _ptr(dq), _ptr(dkh), _ptr(dvh),
                                 int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_attn_bwd: bad argument")
    grp = H // H_kv
    dk = dkh.reshape(B, H_kv, grp, T, D).sum(axis=2)
    dv = dvh.reshape(B, H_kv, grp, T, D).sum(axis=2)
    return dq, dk, dv


def attn_decode(q_bits, k_bits, v_bits, causal: bool, scale: float):
    """Decode attention in float64: q [B, H, Tq, D] against a cache k/v
    [B, H_kv, Tk, D]; query i sits at position Tk - Tq + i.  Returns
    (o [B, H, Tq, D], lse [B, H, Tq])."""
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v = np.ascontiguousarray(v_bits, dtype=np.uint16)
    B, H, Tq, D = q.shape
    H_kv, Tk = k.shape[1], k.shape[2]
    o = np.empty((B, H, Tq, D))
    lse = np.empty((B, H, Tq))
    rc = _load().oracle_attn_decode(_ptr(q), _ptr(k), _ptr(v), B, H, H_kv, Tq, Tk, D,
                                    int(bool(causal)), float(scale), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attn_decode: bad argument")
    return o, lse
