"""Helpers shared by the GPU tests: run the CUDA path, run the oracle on the
same seeded inputs, compare."""
from __future__ import annotations

import numpy as np
import torch

import exact_attention_124_b200 as attn
import oracle
from attn_inputs import bf16_bits, make_qkv, sample_rows
from tests.parity import compare


def require_gpu():
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"
    attn.load_library()


def to_dev(*ts):
    return [t.cuda() for t in ts]


def run_fused(q, k, v, causal, scale):
    qd, kd, vd = to_dev(q, k, v)
    o, lse = attn.fwd(qd, kd, vd, causal, scale)
    rc = attn.last_error()
    assert rc == 0, f"device status {rc}"
    return o, lse


def oracle_ref(q, k, v, causal, scale, heads=None, rows=None):
    return oracle.attn_fwd(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, scale,
                           heads=heads, rows=rows)


def gather(o, lse, heads, rows):
    """Device outputs for (heads, rows) as float64 numpy, oracle layout."""
    B, H, T, D = o.shape
    of = o.reshape(B * H, T, D)
    lf = lse.reshape(B * H, T)
    h = torch.as_tensor(heads if heads is not None else list(range(B * H)), device=o.device)
    r = torch.as_tensor(rows if rows is not None else list(range(T)), device=o.device)
    oo = of.index_select(0, h).index_select(1, r).double().cpu().numpy()
    ll = lf.index_select(0, h).index_select(1, r).double().cpu().numpy()
    return oo, ll


def check_full(q, k, v, causal, scale):
    o, lse = run_fused(q, k, v, causal, scale)
    ro, rl = oracle_ref(q, k, v, causal, scale)
    oo, ll = gather(o, lse, None, None)
    return compare(oo, ll, ro, rl), (o, lse)
