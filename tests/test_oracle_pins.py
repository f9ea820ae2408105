"""Pins of the oracle's softmax core to the numbers the pages print.

Fixtures: tests/golden/two_score.json ("FlashAttention -- avoid writing the
giant intermediate", small normalization exercise) and tests/golden/fig4.json
("Why Attention Is Difficult to Optimize", Figure 4).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_two_score_example():
    g = _load("two_score.json")
    p, lse = oracle.softmax_row([0.0, math.log(3.0)])
    assert np.allclose(p, g["weights"], rtol=0, atol=1e-15)
    # the denominator is 1 + 3 = 4
    assert abs(lse - math.log(4.0)) < 1e-15


def test_two_score_independent_normalisation_is_what_the_page_calls_wrong():
    g = _load("two_score.json")
    # each score alone, as a one-element softmax, gives weight 1: the page's wrong answer
    alone = [oracle.softmax_row([s])[0][0] for s in (0.0, math.log(3.0))]
    assert alone == g["independent_one_element_weights"]
    full, _ = oracle.softmax_row([0.0, math.log(3.0)])
    assert not np.allclose(full, alone)


def test_two_score_shifted_far_out():
    # adding a constant to every score leaves softmax unchanged; with scores
    # near 1000 a missing max subtraction would overflow exp()
    p, lse = oracle.softmax_row([1000.0, 1000.0 + math.log(3.0)])
    assert np.allclose(p, [0.25, 0.75], rtol=0, atol=1e-13)
    assert abs(lse - (1000.0 + math.log(4.0))) < 1e-12


def test_figure4_rows():
    g = _load("fig4.json")
    left, right = g["rows"]
    p, lse = oracle.softmax_row(left["scores"])
    assert p[0] == left["p0"] and np.all(p == 0.25)
    assert abs(math.exp(lse) - left["exp_sum"]) < 1e-12
    p, lse = oracle.softmax_row(right["scores"])
    assert abs(p[0] - right["p0"]) <= right["p0_tol"]
    assert abs(p[0] - 1.0 / (2.0 + 2.0 * math.exp(2.0))) < 1e-15
    assert abs(math.exp(lse) - right["exp_sum"]) <= right["exp_sum_tol"]
    # the exponential of the later score: p2/p0 = e^2
    assert abs(p[2] / p[0] - right["exp_2"]) <= right["exp_2_tol"]


def test_figure4_first_two_alone_differs():
    g = _load("fig4.json")
    part = g["first_two_alone"]
    p2, _ = oracle.softmax_row(part["scores"])
    assert np.all(p2 == part["p"])
    p4, _ = oracle.softmax_row([0, 0, 0, 0])
    assert p4[0] != p2[0]  # 25% across the full row, not 50%


def test_masked_entries_are_exactly_zero_and_rest_renormalised():
    s = [0.3, -1.0, 2.5, 0.0, 7.0]
    masked = [0, 0, 0, 1, 1]
    p, lse = oracle.softmax_row(s, masked)
    assert p[3] == 0.0 and p[4] == 0.0
    q, lse3 = oracle.softmax_row(s[:3])
    assert np.allclose(p[:3], q, rtol=0, atol=1e-16)
    assert lse == lse3


def test_fully_masked_row():
    p, lse = oracle.softmax_row([1.0, 2.0], [1, 1])
    assert np.all(p == 0.0) and lse == -math.inf


@pytest.mark.parametrize("n", [1, 2, 7, 128, 1000])
def test_row_sums_to_one(n):
    rng = np.random.default_rng(n)
    p, _ = oracle.softmax_row(rng.normal(0, 5, n))
    assert abs(p.sum() - 1.0) < 1e-12
