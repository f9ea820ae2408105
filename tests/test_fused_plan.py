"""The fused forward's work units (attn_selftest_fused_plan: the kernel's own
unit function run on the CPU): every (query head, block of 256 query rows) is
computed exactly once, by one CTA, with the right K/V head (grouped-query
attention) and the right number of 128-key tiles per 128-row query tile
(causal: up to the diagonal; tiles past T: none); causal blocks are dealt in
pairs (q, nqb - 1 - q) so every pair costs the same."""
import pytest

import exact_attention_124_b200 as attn

SHAPES = [(1, 1, 1, 1, True), (1, 1, 1, 128, True), (1, 2, 2, 300, True), (1, 2, 1, 768, True),
          (2, 6, 3, 1000, True), (2, 6, 3, 1000, False), (4, 32, 8, 8192, True),
          (16, 16, 16, 2048, False), (1, 8, 8, 65536, True), (3, 5, 1, 257, False)]


@pytest.mark.parametrize("B,H,H_kv,T,causal", SHAPES)
@pytest.mark.parametrize("sms", [148, 7, 1])
def test_fused_plan_covers_every_block_once(B, H, H_kv, T, causal, sms):
    units, ctas = attn.fused_plan(B, H, H_kv, T, causal, sms)
    nqb = (T + 255) // 256
    nkv = (T + 127) // 128
    work = B * H * ((nqb + 1) // 2 if causal else nqb)
    assert ctas == min(sms, work)
    seen = {}
    per_cta = {}
    group = H // H_kv
    for c, k, bh, kvh, i0, n0, n1 in units:
        assert 0 <= c < ctas and (bh, i0) not in seen
        seen[(bh, i0)] = c
        per_cta.setdefault(c, []).append((k, bh, i0, n0, n1))
        assert kvh == (bh // H) * H_kv + (bh % H) // group
        l0 = i0 // 128 + 1
        if causal:
            assert n0 == min(nkv, l0)
            assert n1 == (0 if i0 + 128 >= T else min(nkv, l0 + 1))
        else:
            assert n0 == nkv and n1 == (0 if i0 + 128 >= T else nkv)
    assert set(seen) == {(bh, 256 * q) for bh in range(B * H) for q in range(nqb)}
    for c, lst in per_cta.items():
        ks = [x[0] for x in lst]
        assert ks == sorted(ks) and len(set(ks)) == len(ks)
        if causal:  # unit 2m is block nqb-1-p of a head, unit 2m+1 block p of the same head
            by_k = {x[0]: x for x in lst}
            for kk, (_, bh, i0, _, _) in by_k.items():
                if kk % 2 == 1 and kk - 1 in by_k:
                    _, bh0, i00, _, _ = by_k[kk - 1]
                    assert bh0 == bh and i00 // 256 + i0 // 256 == nqb - 1


def test_fused_plan_causal_pairs_balance_the_ctas():
    units, ctas = attn.fused_plan(4, 32, 8, 8192, True, 148)
    cost = {}
    for c, k, bh, kvh, i0, n0, n1 in units:
        cost[c] = cost.get(c, 0) + n0 + n1
    pair = 2 * ((8192 + 127) // 128) + 2  # n0 + n1 summed over a pair (q, nqb-1-q)
    assert max(cost.values()) - min(cost.values()) <= pair


def test_fused_plan_rejects_bad_sizes():
    with pytest.raises(ValueError):
        attn.fused_plan(1, 6, 4, 128, True, 148)
    with pytest.raises(ValueError):
        attn.fused_plan(1, 4, 4, 0, True, 148)
