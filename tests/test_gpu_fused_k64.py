"""Parity of the fused forward's 64-key-tile schedule (two score buffers per
query tile, the next score MMA overlapping the softmax; selected with
attn.set_key_tile(64)) with the float64 oracle -- the same bar and cases as
the 128-key-tile kernel: ragged tiny sizes, the x4 logit stress (frequent
rescales), grouped-query heads, sampled rows of the full-size workloads,
causal row 0, determinism."""
import math

import pytest
import torch

import exact_attention_124_b200 as attn
import oracle
from attn_inputs import WORKLOADS, bf16_bits, make_qkv, make_workload, sample_rows
from tests.gpu_util import check_full, gather, oracle_ref, require_gpu, run_fused, to_dev
from tests.parity import assert_parity, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _k64():
    require_gpu()
    prev = attn.set_key_tile(64)
    yield
    attn.set_key_tile(prev)


SWEEP_T = [1, 2, 17, 63, 64, 65, 127, 128, 129, 191, 255, 256, 257, 300, 513]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("T", SWEEP_T)
def test_k64_tiny_sweep_every_element(T, D, causal):
    q, k, v = make_qkv(1, 2, T, D, 17000 + T + D + int(causal))
    st, _ = check_full(q, k, v, causal, 1 / math.sqrt(D))
    assert_parity(st, f"k64 T={T} D={D} causal={causal}")


@pytest.mark.parametrize("D", [64, 128])
def test_k64_logit_stress_every_element(D):
    # the inputs of the 128-key kernel's stress test: at x4 logits the max-abs
    # error of either kernel is set by bf16 rounding of O near |O| = 4 and
    # sits close to the bar on some seeds (both kernels alike)
    q, k, v = make_qkv(2, 3, 640, D, 8100 + D, qk_mult=4.0)
    for causal in (False, True):
        st, _ = check_full(q, k, v, causal, 1 / math.sqrt(D))
        assert_parity(st, f"k64 x4 D={D} causal={causal}")


@pytest.mark.parametrize("D", [64, 128])
def test_k64_agrees_with_k128(D):
    """Both key tiles compute the same exact attention; they differ only in
    where the online softmax rescales, i.e. by rounding."""
    q, k, v = to_dev(*make_qkv(2, 4, 1536 + 32, D, 18300 + D, qk_mult=4.0))
    for causal in (True, False):
        o64, l64 = attn.fwd(q, k, v, causal)
        attn.set_key_tile(128)
        try:
            o128, l128 = attn.fwd(q, k, v, causal)
        finally:
            attn.set_key_tile(64)
        assert attn.last_error() == 0
        # P is rounded to bf16 after subtracting a running maximum that moves
        # at different keys in the two schedules, so the rounded P differ; O
        # stays within two bf16 units in the last place of the larger value
        # (2^-6 relative, 2^-6 absolute below 1), and on average far closer
        d = (o64.float() - o128.float()).abs()
        ulp = torch.clamp(torch.maximum(o64.float().abs(), o128.float().abs()), min=1.0) * 2.0 ** -6
        assert (d <= ulp).all(), (d.max().item(), (d / ulp).max().item())
        assert d.mean().item() <= 1e-4, d.mean().item()
        assert (l64 - l128).abs().max().item() <= 1e-4


@pytest.mark.parametrize("name", ["causal_T4096_d64", "causal_T8192_d128", "full_T2048_d128_qk4"])
def test_k64_full_size_sampled_rows(name):
    w = WORKLOADS[name]
    q, k, v = make_workload(w)
    o, lse = run_fused(q, k, v, w.causal, w.scale)
    heads = sorted({0, 1, w.heads // 2, w.heads - 1})
    rows = sample_rows(w.T, w.seed, n_random=256 if w.T >= 8192 else 512)
    ro, rl = oracle_ref(q, k, v, w.causal, w.scale, heads=heads, rows=rows)
    oo, ll = gather(o, lse, heads, rows)
    st = compare(oo, ll, ro, rl)
    print(name, st)
    assert_parity(st, f"k64 {name}")
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_k64_gqa_every_element():
    B, H, H_kv, T, D = 2, 6, 2, 700, 128
    q, _, _ = make_qkv(B, H, T, D, 18500)
    _, k, v = make_qkv(B, H_kv, T, D, 18501)
    for causal in (True, False):
        o, lse = attn.fwd_gqa(*to_dev(q, k, v), causal)
        assert attn.last_error() == 0
        ro, rl = oracle.attn_fwd_gqa(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, 1 / math.sqrt(D))
        st = compare(o.double().cpu().numpy().reshape(ro.shape),
                     lse.double().cpu().numpy().reshape(rl.shape), ro, rl)
        assert_parity(st, f"k64 gqa causal={causal}")


def test_k64_causal_row0_and_determinism():
    q, k, v = make_qkv(2, 4, 1000, 128, 19)
    o, lse = run_fused(q, k, v, True, 1 / math.sqrt(128))
    assert torch.equal(o[:, :, 0, :].cpu(), v[:, :, 0, :])
    qd, kd, vd = to_dev(*make_qkv(2, 8, 2048, 128, 20))
    o1, l1 = attn.fwd(qd, kd, vd, True)
    o2, l2 = attn.fwd(qd, kd, vd, True)
    assert attn.last_error() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
