"""Parity of the sm_100a backward pass (attn_bwd) with the float64 oracle's
gradients, on the same bf16 inputs.  The GPU backward takes the GPU forward's
O and lse (as a training step would); the oracle recomputes everything in
float64.

Bounds: the kernels round P and dS to bf16 for the tensor cores (unit
roundoff 2^-8), use the bf16-rounded forward output O in D = rowsum(dO o O),
and round the gradients to bf16; errors are measured relative to the size of
each gradient: max |d - ref| <= 2^-6 max |ref| and mean |d - ref| <=
2^-7 mean |ref| (per tensor); measured: about 0.5 % and 0.25 %."""
import math

import numpy as np
import pytest
import torch

import exact_attention_124_b200 as attn
import oracle
from attn_inputs import bf16_bits, make_qkv
from tests.gpu_util import require_gpu, to_dev

pytestmark = pytest.mark.gpu

MAX_REL = 2.0 ** -6
MEAN_REL = 2.0 ** -7


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _rel(got, ref):
    d = np.abs(got - ref)
    return float(d.max() / np.abs(ref).max()), float(d.mean() / np.abs(ref).mean())


def _run(B, H, H_kv, T, D, causal, seed, mult=1.0):
    q, _, _ = make_qkv(B, H, T, D, seed, mult)
    _, k, v = make_qkv(B, H_kv, T, D, seed + 1, mult)
    g, _, _ = make_qkv(B, H, T, D, seed + 2)
    qd, kd, vd, gd = to_dev(q, k, v, g)
    o, lse = attn.fwd_gqa(qd, kd, vd, causal)
    dq, dk, dv = attn.bwd(qd, kd, vd, o, lse, gd, causal)
    assert attn.last_error() == 0
    rq, rk, rv = oracle.attn_bwd(bf16_bits(q), bf16_bits(k), bf16_bits(v), bf16_bits(g), causal,
                                 1 / math.sqrt(D))
    out = {}
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        out[name] = _rel(got.double().cpu().numpy(), ref)
    return out


CASES = [(1, 2, 2, 128, 64, True), (1, 2, 2, 256, 128, True), (2, 2, 2, 384, 64, False),
         (1, 4, 2, 512, 128, True), (1, 2, 1, 256, 128, False), (1, 3, 3, 640, 128, True),
         # T not a multiple of 128: the last key/query block is padded inside attn_bwd
         (1, 2, 2, 200, 64, True), (1, 2, 1, 333, 128, False),
         (2, 2, 2, 1000, 128, True), (1, 3, 3, 129, 64, False), (1, 4, 2, 700, 64, True)]


@pytest.mark.parametrize("B,H,H_kv,T,D,causal", CASES)
def test_backward_every_element(B, H, H_kv, T, D, causal):
    errs = _run(B, H, H_kv, T, D, causal, 6000 + T + D + H)
    print(f"bwd B={B} H={H} H_kv={H_kv} T={T} D={D} causal={causal}: {errs}")
    for name, (mx, mean) in errs.items():
        assert mx <= MAX_REL and mean <= MEAN_REL, (name, mx, mean)


def test_backward_bench_size_whole_head():
    """One whole head at the size the backward is benchmarked on (T = 8192,
    d_h = 128, causal): every element of dQ, dK and dV."""
    errs = _run(1, 1, 1, 8192, 128, True, 6200)
    print("bwd T=8192 d_h=128 causal, one head:", errs)
    for name, (mx, mean) in errs.items():
        assert mx <= MAX_REL and mean <= MEAN_REL, (name, mx, mean)


def test_backward_logit_stress():
    errs = _run(1, 2, 2, 512, 128, False, 6100, mult=2.0)
    print("bwd x2 logits:", errs)
    for name, (mx, mean) in errs.items():
        assert mx <= MAX_REL and mean <= MEAN_REL, (name, mx, mean)


def test_backward_deterministic():
    q, k, v = to_dev(*make_qkv(1, 4, 512, 128, 71))
    g = to_dev(*make_qkv(1, 4, 512, 128, 72))[0]
    o, lse = attn.fwd(q, k, v, True)
    a = attn.bwd(q, k, v, o, lse, g, True)
    b = attn.bwd(q, k, v, o, lse, g, True)
    assert attn.last_error() == 0
    assert all(torch.equal(x, y) for x, y in zip(a, b))
