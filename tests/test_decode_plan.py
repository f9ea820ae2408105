"""The decode work plan (attn_selftest_decode_plan: the library's own host and
kernel partition code run on the CPU) covers every (head, key tile) exactly
once, gives every head's partial slots 0 .. nseg-1 exactly once (the slots the
merge kernel reads; a segment fills one slot per copy of the packed rows),
stays inside the workspace's slot count, and in balanced mode deals the same
number of tiles (within one) to every CTA."""
import itertools
import random
from collections import Counter, defaultdict

import pytest

import exact_attention_124_b200 as attn


def _check(B, H, H_kv, Tq, Tk, splits, sms):
    segs, nseg, slots, copies = attn.decode_plan(B, H, H_kv, Tq, Tk, splits, sms)
    nkt = (Tk + 127) // 128
    rows = (H // H_kv) * Tq
    nrb = (rows + 127) // 128
    assert copies == (4 if rows <= 32 else 2 if rows <= 64 else 1)
    heads = B * H_kv * nrb
    assert len(nseg) == heads
    covered = Counter()
    head_slots = defaultdict(list)
    per_cta = Counter()
    ctas = set()
    for bx, by, bz, kvbh, qt, t0, n, slot in segs:
        assert 0 <= kvbh < B * H_kv and 0 <= qt < nrb
        assert n >= 1 and 0 <= t0 and t0 + n <= nkt
        w = kvbh * nrb + qt
        for t in range(t0, t0 + n):
            covered[(w, t)] += 1
        head_slots[w].extend(range(slot, slot + copies))
        per_cta[(bx, by, bz)] += n
        ctas.add((bx, by, bz))
        assert 0 <= slot and slot + copies <= slots
    assert len(covered) == heads * nkt and set(covered.values()) == {1}
    for w in range(heads):
        assert sorted(head_slots[w]) == list(range(nseg[w])), (w, head_slots[w], nseg[w])
    if splits < 0:
        assert len(ctas) == min(sms, heads * nkt)
        assert max(per_cta.values()) - min(per_cta.values()) <= 1
    if splits > 0:
        s = min(splits, nkt)
        chunk = -(-nkt // s)
        assert len(ctas) == heads * (-(-nkt // chunk))
    return segs, nseg, slots, len(ctas), copies


SHAPES = [(2, 8, 2, 1, 4096), (1, 4, 4, 16, 1000), (1, 32, 8, 64, 2048), (3, 6, 3, 5, 333),
          (1, 2, 1, 1, 1), (1, 2, 1, 1, 16384), (64, 8, 8, 1, 512), (2, 32, 4, 40, 700),
          (3, 12, 4, 7, 5000), (4, 32, 8, 1, 8192), (8, 32, 8, 1, 32768)]


@pytest.mark.parametrize("B,H,H_kv,Tq,Tk", SHAPES)
@pytest.mark.parametrize("splits", [-1, 0, 1, 3, 7])
@pytest.mark.parametrize("sms", [148, 7, 1])
def test_decode_plan_covers_everything_once(B, H, H_kv, Tq, Tk, splits, sms):
    _check(B, H, H_kv, Tq, Tk, splits, sms)


def test_decode_plan_random_shapes():
    rng = random.Random(5)
    for _ in range(150):
        H_kv = rng.choice([1, 2, 4, 8])
        H = H_kv * rng.randint(1, 8)
        Tk = rng.randint(1, 20000)
        Tq = rng.randint(1, min(Tk, 300))
        _check(rng.randint(1, 40), H, H_kv, Tq, Tk, rng.choice([-1, 0, 2]), rng.choice([148, 132, 3]))


def test_decode_plan_automatic_choice():
    # 32 heads of 64 tiles: 4 splits fill 128 of 148 SMs (86 %) in one wave
    segs, _, _, ctas, copies = _check(4, 32, 8, 1, 8192, 0, 148)
    assert ctas == 128 and all(n == 16 for *_, n, _s in segs)
    assert copies == 4  # group 4 x Tq 1 = 4 rows: four copies, 32 keys of every tile each
    # 100 heads: one wave of fixed splits would leave a third of the SMs idle -> balanced
    segs, _, _, ctas, _ = _check(100, 8, 8, 1, 8192, 0, 148)
    assert ctas == 148 and all(c[1:3] == (0, 0) for c in segs)


def test_decode_plan_balanced_spans_heads_and_ctas():
    # one head over 128 CTAs of one tile each, and 512 short heads over 148 CTAs
    segs, nseg, _, _, copies = _check(1, 2, 1, 1, 16384, -1, 148)
    assert nseg == [128 * copies]
    segs, nseg, _, _, _ = _check(64, 8, 8, 1, 512, -1, 148)
    per_cta = Counter(s[0] for s in segs)
    assert max(per_cta.values()) >= 4  # several heads (segments) in one CTA


def test_decode_plan_rejects_bad_sizes():
    with pytest.raises(ValueError):
        attn.decode_plan(1, 6, 4, 1, 128, 0, 148)
    with pytest.raises(ValueError):
        attn.decode_plan(1, 4, 4, 8, 4, 0, 148)
