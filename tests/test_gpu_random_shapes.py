"""Seeded random shapes through every GPU entry point, each checked against
the float64 oracle with the bar of its own parity tests: grouped-query
forward (any T, both d_h, causal or not), backward (long enough for the K/V
rings to wrap several times, T a multiple of 128 or not) and decode (fixed,
balanced and automatic partitions, 1, 2 or 4 row copies)."""
import math
import random

import numpy as np
import pytest
import torch

import exact_attention_124_b200 as attn
import oracle
from attn_inputs import bf16_bits, make_qkv
from tests.gpu_util import require_gpu, to_dev
from tests.parity import assert_parity, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _fwd_cases(n=16, seed=424242):
    rng = random.Random(seed)
    out = []
    for i in range(n):
        H_kv = rng.randint(1, 3)
        out.append((rng.randint(1, 2), H_kv * rng.randint(1, 3), H_kv, rng.randint(1, 700),
                    rng.choice([64, 128]), rng.random() < 0.6, 31000 + i))
    return out


@pytest.mark.parametrize("B,H,H_kv,T,D,causal,seed", _fwd_cases())
def test_random_forward(B, H, H_kv, T, D, causal, seed):
    q, _, _ = make_qkv(B, H, T, D, seed)
    _, k, v = make_qkv(B, H_kv, T, D, seed + 500)
    o, lse = attn.fwd_gqa(*to_dev(q, k, v), causal)
    assert attn.last_error() == 0
    ro, rl = oracle.attn_fwd_gqa(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, 1 / math.sqrt(D))
    st = compare(o.double().cpu().numpy().reshape(ro.shape),
                 lse.double().cpu().numpy().reshape(rl.shape), ro, rl)
    assert_parity(st, f"fwd B={B} H={H} H_kv={H_kv} T={T} D={D} causal={causal}")


BWD_CASES = [(1, 2, 1, 2048, 128, True, 32001), (1, 2, 2, 1536, 64, False, 32002),
             (2, 4, 2, 1024, 128, True, 32003), (1, 3, 1, 1280, 64, True, 32004),
             # ragged T: the last 128-row block of queries and keys is padded
             (1, 2, 1, 1999, 128, True, 32005), (2, 2, 2, 777, 64, False, 32006),
             (1, 4, 2, 1153, 128, False, 32007), (1, 2, 2, 321, 64, True, 32008)]


@pytest.mark.parametrize("B,H,H_kv,T,D,causal,seed", BWD_CASES)
def test_random_backward(B, H, H_kv, T, D, causal, seed):
    q, _, _ = make_qkv(B, H, T, D, seed)
    _, k, v = make_qkv(B, H_kv, T, D, seed + 1)
    g, _, _ = make_qkv(B, H, T, D, seed + 2)
    qd, kd, vd, gd = to_dev(q, k, v, g)
    o, lse = attn.fwd_gqa(qd, kd, vd, causal)
    grads = attn.bwd(qd, kd, vd, o, lse, gd, causal)
    assert attn.last_error() == 0
    refs = oracle.attn_bwd(bf16_bits(q), bf16_bits(k), bf16_bits(v), bf16_bits(g), causal,
                           1 / math.sqrt(D))
    for name, got, ref in zip(("dq", "dk", "dv"), grads, refs):
        d = np.abs(got.double().cpu().numpy() - ref)
        mx, mean = float(d.max() / np.abs(ref).max()), float(d.mean() / np.abs(ref).mean())
        assert mx <= 2.0 ** -6 and mean <= 2.0 ** -7, (name, mx, mean)


def _dec_cases(n=12, seed=777001):
    rng = random.Random(seed)
    out = []
    for i in range(n):
        H_kv = rng.choice([1, 2, 4])
        Tq = rng.choice([1, 1, 2, 5, 16, 40])
        out.append((rng.randint(1, 6), H_kv * rng.choice([1, 2, 4, 8]), H_kv, Tq,
                    rng.randint(Tq, 5000), rng.choice([64, 128]), rng.random() < 0.7,
                    rng.choice([-1, 0, 0, 1, 3, 5]), 33000 + i))
    return out


@pytest.mark.parametrize("B,H,H_kv,Tq,Tk,D,causal,splits,seed", _dec_cases())
def test_random_decode(B, H, H_kv, Tq, Tk, D, causal, splits, seed):
    q, _, _ = make_qkv(B, H, Tq, D, seed)
    _, k, v = make_qkv(B, H_kv, Tk, D, seed + 1)
    o, lse = attn.fwd_decode(*to_dev(q, k, v), causal, splits=splits)
    assert attn.last_error() == 0
    ro, rl = oracle.attn_decode(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, 1 / math.sqrt(D))
    st = compare(o.double().cpu().numpy(), lse.double().cpu().numpy(), ro, rl)
    assert_parity(st, f"decode B={B} H={H} H_kv={H_kv} Tq={Tq} Tk={Tk} D={D} splits={splits}")
