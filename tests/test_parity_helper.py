"""The comparator used by the GPU parity tests flags a planted mistake.
The mistake is planted in the oracle's output, on the CPU."""
import math

import numpy as np

import oracle
from attn_inputs import bf16_bits, make_qkv
from tests.parity import compare, ok


def _ref():
    q, k, v = make_qkv(1, 2, 150, 64, 42)
    return oracle.attn_fwd(bf16_bits(q), bf16_bits(k), bf16_bits(v), True, 0.125)


def test_identical_passes():
    o, l = _ref()
    assert ok(compare(o, l, o, l))


def test_bf16_rounding_of_output_passes():
    o, l = _ref()
    import torch
    ob = torch.from_numpy(o).to(torch.bfloat16).to(torch.float64).numpy()
    assert ok(compare(ob, l, o, l))


def test_single_wrong_element_fails():
    o, l = _ref()
    bad = o.copy()
    bad[1, 77, 5] += 0.05
    assert not ok(compare(bad, l, o, l))


def test_dropped_diagonal_fails():
    # a mask that hides the diagonal (j < i instead of j <= i) is a plausible bug
    q, k, v = make_qkv(1, 1, 64, 64, 43)
    qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    o, l = oracle.attn_fwd(qb, kb, vb, True, 0.125)
    # emulate: row i sees keys < i; row 0 then sees nothing -> use rows >= 1
    S, _, _ = oracle.head_scores_probs(qb[0, 0], kb[0, 0], False, 0.125)
    vf = v[0, 0].double().numpy()
    wrong = np.zeros_like(o[0])
    for i in range(1, 64):
        p, _ = oracle.softmax_row(S[i, :i])
        wrong[i] = p @ vf[:i]
    wrong[0] = o[0, 0]
    assert not ok(compare(wrong[None], l, o, l))


def test_lse_offset_fails():
    o, l = _ref()
    assert not ok(compare(o, l + 2e-3 * np.maximum(1, np.abs(l)), o, l))
    assert ok(compare(o, l + 5e-4, o, l))
