"""Pins of the oracle's gradients (the backward pass that recomputes S and P,
"Attention Mechanism: Computation & Memory Patterns", section 4): central
finite differences of the forward definition, and invariants that hold for
any inputs."""
import math

import numpy as np
import pytest

import oracle
from attn_inputs import bf16_bits, make_qkv


def _rand(T, D, seed):
    r = np.random.default_rng(seed)
    return [r.normal(size=(T, D)) for _ in range(4)]


def _loss(q, k, v, dout, causal, scale):
    o, _ = oracle.head_fwd_f64(q, k, v, causal, scale)
    return float(np.sum(o * dout))


@pytest.mark.parametrize("causal", [True, False])
def test_gradients_match_central_differences(causal):
    T, D, scale = 7, 3, 0.6
    q, k, v, g = _rand(T, D, 3 + causal)
    dq, dk, dv = oracle.head_bwd_f64(q, k, v, g, causal, scale)
    eps = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in [(0, 0), (2, 1), (T - 1, 2), (3, 0)]:
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            num = (_loss(args_p["q"], args_p["k"], args_p["v"], g, causal, scale) -
                   _loss(args_m["q"], args_m["k"], args_m["v"], g, causal, scale)) / (2 * eps)
            assert abs(num - grad[idx]) < 1e-7 * max(1.0, abs(num)), (name, idx, num, grad[idx])


def test_invariants():
    T, D, scale = 12, 5, 0.4
    q, k, v, g = _rand(T, D, 9)
    for causal in (True, False):
        dq, dk, dv = oracle.head_bwd_f64(q, k, v, g, causal, scale)
        # shifting every key by the same vector changes no probability
        assert np.max(np.abs(dk.sum(axis=0))) < 1e-12
        # each row of P sums to one, so the values' gradients sum to dO's
        assert np.max(np.abs(dv.sum(axis=0) - g.sum(axis=0))) < 1e-12
    dq, dk, dv = oracle.head_bwd_f64(q, k, v, g, True, scale)
    # causal row 0 sees one key with probability 1: no gradient reaches q_0
    assert np.max(np.abs(dq[0])) < 1e-15
    # the last key is seen only by the last query: its dv is that row's p * dO
    o, lse = oracle.head_fwd_f64(q, k, v, True, scale)
    p_last = math.exp(scale * float(q[T - 1] @ k[T - 1]) - lse[T - 1])
    assert np.max(np.abs(dv[T - 1] - p_last * g[T - 1])) < 1e-12


def test_bf16_entry_sums_group_contributions():
    B, H, H_kv, T, D = 1, 4, 2, 10, 4
    q, _, _ = make_qkv(B, H, T, D, 61)
    _, k, v = make_qkv(B, H_kv, T, D, 62)
    g, _, _ = make_qkv(B, H, T, D, 63)
    dq, dk, dv = oracle.attn_bwd(bf16_bits(q), bf16_bits(k), bf16_bits(v), bf16_bits(g), True, 0.5)
    f = lambda t: t.double().numpy()
    for h in range(H):
        dq1, dk1, dv1 = oracle.head_bwd_f64(f(q[0, h]), f(k[0, h // 2]), f(v[0, h // 2]),
                                            f(g[0, h]), True, 0.5)
        assert np.allclose(dq[0, h], dq1, rtol=0, atol=1e-14)
    dk_sum = sum(oracle.head_bwd_f64(f(q[0, h]), f(k[0, 0]), f(v[0, 0]), f(g[0, h]), True, 0.5)[1]
                 for h in (0, 1))
    assert np.allclose(dk[0, 0], dk_sum, rtol=0, atol=1e-13)
