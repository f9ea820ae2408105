"""Pins of the oracle's attention forward: invariants the pages fix, closed
forms, and a 50-digit brute force on tiny inputs.

Pages: "Why Attention Is Difficult to Optimize" ("The Attention Computation
Flow": scaling, causal mask "itself and earlier tokens", rows of P summing to
1); "Attention Mechanism: Computation & Memory Patterns" (section 1: S = QK^T,
P = softmax(S / sqrt(d_k)), O = PV).
"""
import math

import mpmath
import numpy as np
import pytest
import torch

import oracle
from attn_inputs import bf16_bits, make_qkv


def _f64(bits):
    return bits.astype(np.uint32).__lshift__(16).view(np.float32).astype(np.float64)


def _bits(x: torch.Tensor):
    return bf16_bits(x.to(torch.bfloat16))


def _rand_head(T, D, seed, mult=1.0):
    q, k, v = make_qkv(1, 1, T, D, seed, mult)
    return bf16_bits(q[0, 0]), bf16_bits(k[0, 0]), bf16_bits(v[0, 0])


@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one_and_future_is_zero(causal):
    T, D = 37, 16
    q, k, _ = _rand_head(T, D, 5)
    S, P, _ = oracle.head_scores_probs(q, k, causal, 1 / math.sqrt(D))
    assert np.all(np.abs(P.sum(axis=1) - 1.0) < 1e-12)
    if causal:
        iu = np.triu_indices(T, 1)
        assert np.all(P[iu] == 0.0)  # exactly zero, not merely small
        assert np.all(P[np.tril_indices(T)] > 0.0)
    else:
        assert np.all(P > 0.0)


def test_scores_are_scaled_q_dot_k_not_transposed():
    T, D = 6, 4
    q, k, _ = _rand_head(T, D, 11)
    scale = 0.37
    S, _, _ = oracle.head_scores_probs(q, k, False, scale)
    qf, kf = _f64(q), _f64(k)
    mpmath.mp.dps = 50
    for i in range(T):
        for j in range(T):
            ref = mpmath.mpf(scale) * mpmath.fsum(mpmath.mpf(qf[i, c]) * mpmath.mpf(kf[j, c])
                                                  for c in range(D))
            assert abs(S[i, j] - float(ref)) < 1e-14 * max(1.0, abs(float(ref)))
    # Q and K are not symmetric, so a transposed product would differ
    assert not np.allclose(S, S.T)


@pytest.mark.parametrize("T", [1, 2, 5, 64, 65, 130])
def test_causal_row0_is_v0(T):
    D = 8
    q, k, v = _rand_head(T, D, 100 + T)
    o, lse = oracle.attn_fwd(q, k, v, True, 1 / math.sqrt(D))
    assert np.array_equal(o[0, 0], _f64(v)[0])  # exactly: P_00 = 1
    qk = float(np.dot(_f64(q)[0], _f64(k)[0]))
    assert abs(lse[0, 0] - qk / math.sqrt(D)) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_zero_keys_give_prefix_means(causal):
    T, D = 77, 8
    q, _, v = _rand_head(T, D, 7)
    k = np.zeros_like(q)
    o, lse = oracle.attn_fwd(q, k, v, causal, 0.125)
    vf = _f64(v)
    if causal:
        ref = np.cumsum(vf, axis=0) / np.arange(1, T + 1)[:, None]
        ref_lse = np.log(np.arange(1, T + 1))
    else:
        ref = np.broadcast_to(vf.mean(axis=0), (T, D))
        ref_lse = np.full(T, math.log(T))
    assert np.max(np.abs(o[0] - ref)) < 1e-12
    assert np.max(np.abs(lse[0] - ref_lse)) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_constant_values_pass_through(causal):
    T, D = 50, 16
    q, k, _ = _rand_head(T, D, 8, 4.0)
    v = _bits(torch.full((T, D), -1.75))
    o, _ = oracle.attn_fwd(q, k, v, causal, 1 / 4)
    assert np.max(np.abs(o + 1.75)) < 1e-12


def test_single_token_output_is_v():
    q, k, v = _rand_head(1, 64, 9)
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, causal, 0.125)
        assert np.array_equal(o[0, 0], _f64(v)[0])


def test_noncausal_permutation_invariance():
    T, D = 40, 8
    q, k, v = _rand_head(T, D, 10)
    perm = np.random.default_rng(0).permutation(T)
    o1, l1 = oracle.attn_fwd(q, k, v, False, 0.3)
    o2, l2 = oracle.attn_fwd(q, k[perm], v[perm], False, 0.3)
    assert np.max(np.abs(o1 - o2)) < 1e-12 and np.max(np.abs(l1 - l2)) < 1e-12


def _brute(qf, kf, vf, causal, scale):
    """Naive formula at 50 digits, no max subtraction: o_i = sum_j e^{s_ij} v_j / sum_j e^{s_ij}."""
    mpmath.mp.dps = 50
    T, D = qf.shape
    o = np.zeros((T, D))
    lse = np.zeros(T)
    for i in range(T):
        js = [j for j in range(T) if not (causal and j > i)]
        e = {}
        for j in js:
            s = mpmath.mpf(scale) * mpmath.fsum(mpmath.mpf(qf[i, c]) * mpmath.mpf(kf[j, c])
                                                for c in range(D))
            e[j] = mpmath.exp(s)
        den = mpmath.fsum(e.values())
        for c in range(D):
            o[i, c] = float(mpmath.fsum(e[j] * mpmath.mpf(vf[j, c]) for j in js) / den)
        lse[i] = float(mpmath.log(den))
    return o, lse


@pytest.mark.parametrize("T,D,causal,mult", [(1, 1, True, 1.0), (3, 2, True, 1.0),
                                             (7, 4, False, 1.0), (16, 8, True, 1.0),
                                             (16, 8, False, 4.0), (11, 5, True, 4.0)])
def test_brute_force_tiny(T, D, causal, mult):
    q, k, v = _rand_head(T, D, 1000 + 31 * T + D, mult)
    scale = 1 / math.sqrt(D)
    o, lse = oracle.attn_fwd(q, k, v, causal, scale)
    bo, bl = _brute(_f64(q), _f64(k), _f64(v), causal, scale)
    assert np.max(np.abs(o[0] - bo)) < 1e-13
    assert np.max(np.abs(lse[0] - bl)) < 1e-13 * max(1.0, float(np.max(np.abs(bl))))


def test_subsets_match_full():
    B, H, T, D = 2, 2, 150, 16
    q, k, v = make_qkv(B, H, T, D, 3)
    qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    o, l = oracle.attn_fwd(qb, kb, vb, True, 0.25)
    heads = [3, 0]
    rows = [149, 0, 63, 64, 65, 127, 128]
    os_, ls = oracle.attn_fwd(qb, kb, vb, True, 0.25, heads=heads, rows=rows, nthreads=3)
    for a, h in enumerate(heads):
        assert np.array_equal(os_[a], o[h][rows])
        assert np.array_equal(ls[a], l[h][rows])


def test_bad_arguments_raise():
    q, k, v = _rand_head(8, 4, 1)
    with pytest.raises(ValueError):
        oracle.attn_fwd(q, k, v, True, 1.0, rows=[8])
    with pytest.raises(ValueError):
        oracle.attn_fwd(q, k, v, True, 1.0, heads=[1])


def _brute_gqa(qf, kf, vf, causal, scale, group):
    """Definition of grouped-query attention at 50 digits: query head h uses
    K/V head h // group."""
    H = qf.shape[0]
    outs, lses = [], []
    for h in range(H):
        o, l = _brute(qf[h], kf[h // group], vf[h // group], causal, scale)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


@pytest.mark.parametrize("H,H_kv,causal", [(4, 2, True), (6, 1, False), (4, 4, True)])
def test_gqa_brute_force_tiny(H, H_kv, causal):
    T, D = 9, 4
    q, _, _ = make_qkv(1, H, T, D, 300 + H)
    _, k, v = make_qkv(1, H_kv, T, D, 400 + H_kv)
    scale = 0.5
    o, lse = oracle.attn_fwd_gqa(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, scale)
    bo, bl = _brute_gqa(_f64(bf16_bits(q[0])), _f64(bf16_bits(k[0])), _f64(bf16_bits(v[0])),
                        causal, scale, H // H_kv)
    assert np.max(np.abs(o - bo)) < 1e-13 and np.max(np.abs(lse - bl)) < 1e-12


def test_gqa_batch_entries_use_their_own_kv_heads():
    # B = 2: batch entry 1's query heads must read batch entry 1's K/V heads
    B, H, H_kv, T, D = 2, 4, 2, 33, 8
    q, _, _ = make_qkv(B, H, T, D, 51)
    _, k, v = make_qkv(B, H_kv, T, D, 52)
    o, lse = oracle.attn_fwd_gqa(bf16_bits(q), bf16_bits(k), bf16_bits(v), True, 0.3)
    for b in range(B):
        for h in range(H):
            ob, lb = oracle.attn_fwd(bf16_bits(q[b, h]), bf16_bits(k[b, h // 2]),
                                     bf16_bits(v[b, h // 2]), True, 0.3)
            assert np.array_equal(o[b * H + h], ob[0]) and np.array_equal(lse[b * H + h], lb[0])


def test_decode_with_tq_equal_tk_is_the_forward():
    B, H, H_kv, T, D = 1, 4, 2, 40, 8
    q, _, _ = make_qkv(B, H, T, D, 81)
    _, k, v = make_qkv(B, H_kv, T, D, 82)
    for causal in (True, False):
        o, l = oracle.attn_decode(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, 0.4)
        of, lf = oracle.attn_fwd_gqa(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, 0.4)
        assert np.array_equal(o.reshape(of.shape), of) and np.array_equal(l.reshape(lf.shape), lf)


def test_decode_last_rows_of_causal_forward():
    # Tq new tokens at the end of a Tk-token sequence: the same rows as the
    # last Tq rows of the causal forward over all Tk tokens
    B, H, Tk, Tq, D = 1, 2, 37, 5, 8
    q, k, v = make_qkv(B, H, Tk, D, 83)
    o, l = oracle.attn_decode(bf16_bits(q[:, :, Tk - Tq:]), bf16_bits(k), bf16_bits(v), True, 0.3)
    of, lf = oracle.attn_fwd(bf16_bits(q), bf16_bits(k), bf16_bits(v), True, 0.3)
    assert np.array_equal(o.reshape(B * H, Tq, D), of[:, Tk - Tq:])
    assert np.array_equal(l.reshape(B * H, Tq), lf[:, Tk - Tq:])


def test_decode_brute_force_tiny():
    B, H, H_kv, Tq, Tk, D = 1, 2, 1, 3, 11, 4
    q, _, _ = make_qkv(B, H, Tq, D, 84)
    _, k, v = make_qkv(B, H_kv, Tk, D, 85)
    o, l = oracle.attn_decode(bf16_bits(q), bf16_bits(k), bf16_bits(v), True, 0.5)
    mpmath.mp.dps = 50
    qf, kf, vf = _f64(bf16_bits(q[0])), _f64(bf16_bits(k[0, 0])), _f64(bf16_bits(v[0, 0]))
    for h in range(H):
        for i in range(Tq):
            js = range(Tk - Tq + i + 1)
            e = [mpmath.exp(mpmath.mpf(0.5) * mpmath.fsum(mpmath.mpf(qf[h, i, c]) * mpmath.mpf(kf[j, c])
                                                          for c in range(D))) for j in js]
            den = mpmath.fsum(e)
            for c in range(D):
                ref = float(mpmath.fsum(e[n] * mpmath.mpf(vf[j, c]) for n, j in enumerate(js)) / den)
                assert abs(o[0, h, i, c] - ref) < 1e-13
            assert abs(l[0, h, i] - float(mpmath.log(den))) < 1e-13
