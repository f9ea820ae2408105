"""Parity of the split-KV decode path (attn_fwd_decode) with the float64
oracle: Tq new queries against a Tk-token K/V cache, query i at position
Tk - Tq + i ("FlashAttention -- avoid writing the giant intermediate": the
persistent K/V state of cached decoding).  Same bounds as the prefill path.
The cases cover fixed, balanced and automatic partitions and 1, 2 and 4
copies of the packed query rows (more than 64, 33-64 and at most 32 rows),
including row counts that are not a multiple of the splits."""
import math

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


def _case(B, H, H_kv, Tq, Tk, D, causal, splits, seed):
    q, _, _ = make_qkv(B, H, Tq, D, seed)
    _, k, v = make_qkv(B, H_kv, Tk, D, seed + 1)
    o, lse = attn.fwd_decode(*to_dev(q, k, v), causal, splits=splits)
    assert attn.last_error() == 0
    ro, rl = oracle.attn_decode(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, 1 / math.sqrt(D))
    return compare(o.double().cpu().numpy(), lse.double().cpu().numpy(), ro, rl)


@pytest.mark.parametrize("B,H,H_kv,Tq,Tk,D,causal,splits", [
    (2, 8, 2, 1, 4096, 128, True, 0),
    (2, 8, 2, 1, 4096, 128, True, 1),
    (2, 8, 2, 1, 4096, 128, True, 7),
    (1, 4, 4, 16, 1000, 64, True, 3),
    (1, 4, 4, 16, 1000, 64, False, 0),
    (1, 32, 8, 64, 2048, 128, True, 4),
    (3, 6, 3, 5, 333, 128, True, 2),
    (1, 2, 1, 1, 1, 64, True, 0),
    # balanced partition (splits < 0): one head over 128 CTAs of one tile each
    (1, 2, 1, 1, 16384, 128, True, -1),
    # 512 heads of 4 tiles over the SMs: several heads (segments) per CTA
    (64, 8, 8, 1, 512, 64, True, -1),
    (64, 8, 8, 1, 512, 64, True, 0),
    # three blocks of packed rows per K/V head (8 x 40 = 320 rows), 6 tiles each
    (2, 32, 4, 40, 700, 128, True, -1),
    (2, 32, 4, 40, 700, 128, True, 0),
    (3, 12, 4, 7, 5000, 128, False, -1),
    (3, 12, 4, 7, 5000, 128, False, 0),
    # 33-64 packed rows: two copies of the rows, 64 keys of every tile each
    (2, 8, 2, 12, 3000, 128, True, 0),
    (1, 16, 2, 5, 900, 64, False, -1),
    (1, 16, 2, 8, 260, 64, True, 3),
    # 5 rows over 3 splits, 16 rows over 8, 1 row over 8
    (1, 5, 1, 1, 3000, 128, True, 3),
    (2, 16, 1, 1, 2000, 64, True, 8),
    (1, 8, 8, 1, 1024, 128, False, 8),
    # 24 rows (four copies): fixed splits and balanced
    (2, 8, 2, 6, 1500, 128, True, 4),
    (2, 8, 2, 6, 1500, 64, True, -1),
    # 4 rows over 16 splits
    (2, 8, 2, 1, 4096, 128, True, 16),
])
def test_decode_every_element(B, H, H_kv, Tq, Tk, D, causal, splits):
    st = _case(B, H, H_kv, Tq, Tk, D, causal, splits, 7700 + Tq + Tk + D + splits)
    assert_parity(st, f"decode B={B} H={H} H_kv={H_kv} Tq={Tq} Tk={Tk} D={D} splits={splits}")


def _rising_cache(B, H, H_kv, Tq, Tk, D, seed, slope=0.06):
    """Queries share one direction u and cache key j is slope * j * u plus unit
    noise: every row's running maximum jumps by far more than the lazy
    rescale threshold (32 in log2 units) from one key tile to the next, in
    every copy of the packed rows."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    u = torch.randn(D, generator=g)
    q = (u + 0.1 * torch.randn(B, H, Tq, D, generator=g)).to(torch.bfloat16)
    j = torch.arange(Tk, dtype=torch.float32).view(1, 1, Tk, 1)
    k = (slope * j * u + torch.randn(B, H_kv, Tk, D, generator=g)).to(torch.bfloat16)
    v = torch.randn(B, H_kv, Tk, D, generator=g).to(torch.bfloat16)
    return q.contiguous(), k.contiguous(), v.contiguous()


@pytest.mark.parametrize("B,H,H_kv,Tq,Tk,D,splits", [
    (1, 4, 1, 1, 1000, 128, 0),     # 4 packed rows: four copies of 32 keys per tile
    (1, 4, 1, 1, 1000, 128, 2),     # the same over 2 fixed splits
    (1, 8, 2, 6, 1100, 64, 3),      # 24 rows: four copies, 3 fixed splits
    (1, 4, 4, 40, 700, 64, -1),     # 40 rows: two copies of 64 keys, balanced partition
    (1, 2, 1, 80, 900, 128, 2),     # 160 rows: two row blocks, one copy, fixed splits
])
def test_decode_rescale_path_every_element(B, H, H_kv, Tq, Tk, D, splits):
    """The O rescale (which waits for the previous P.V) runs on nearly every tile."""
    q, k, v = _rising_cache(B, H, H_kv, Tq, Tk, D, 7900 + Tq + D)
    o, lse = attn.fwd_decode(*to_dev(q, k, v), True, splits=splits)
    assert attn.last_error() == 0
    ro, rl = oracle.attn_decode(bf16_bits(q), bf16_bits(k), bf16_bits(v), True, 1 / math.sqrt(D))
    st = compare(o.double().cpu().numpy(), lse.double().cpu().numpy(), ro, rl)
    print(f"decode rising Tq={Tq} D={D} splits={splits}", st)
    assert_parity(st, f"decode rising Tq={Tq} D={D} splits={splits}")


def test_decode_with_tq_equal_tk_matches_prefill():
    q, k, v = to_dev(*make_qkv(1, 4, 512, 128, 91))
    o1, l1 = attn.fwd(q, k, v, True)
    o2, l2 = attn.fwd_decode(q, k, v, True, splits=2)
    assert attn.last_error() == 0
    assert (o1.double() - o2.double()).abs().max().item() < 2e-2
    assert (l1 - l2).abs().max().item() < 1e-3


def test_decode_rejects_cache_shorter_than_queries():
    q = torch.zeros((1, 1, 8, 64), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 1, 4, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(attn.AttnError):
        attn.fwd_decode(q, k, k, True, ws=torch.empty(64, dtype=torch.uint8, device="cuda"))
