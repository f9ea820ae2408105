"""One-tile checks of the tcgen05 building blocks, then the bounded-wait
failure path.  Reference products are float64 matmuls on the host; the
tensor cores accumulate in fp32, so agreement is to fp32 rounding."""
import pytest
import torch

import exact_attention_124_b200 as attn
from tests.gpu_util import require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


@pytest.mark.parametrize("D", [64, 128])
def test_score_tile(D):
    g = torch.Generator().manual_seed(D)
    q = torch.randn(128, D, generator=g).to(torch.bfloat16)
    k = torch.randn(128, D, generator=g).to(torch.bfloat16)
    s = attn.selftest_qk_tile(q.cuda(), k.cuda())
    assert attn.last_error() == 0
    ref = q.double() @ k.double().T
    err = (s.double().cpu() - ref).abs().max().item()
    assert err < 1e-3 * max(1.0, ref.abs().max().item()), err


@pytest.mark.parametrize("D", [64, 128])
def test_pv_tile_from_tensor_memory(D):
    g = torch.Generator().manual_seed(100 + D)
    p = torch.rand(128, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(128, D, generator=g).to(torch.bfloat16)
    o = attn.selftest_pv_tile(p.cuda(), v.cuda())
    assert attn.last_error() == 0
    ref = p.double() @ v.double()
    err = (o.double().cpu() - ref).abs().max().item()
    assert err < 1e-3 * max(1.0, ref.abs().max().item()), err


def test_bounded_wait_reports_timeout_and_context_survives():
    attn.selftest_timeout(2000)
    assert attn.last_error() == 7  # ATTN_ERR_TIMEOUT
    assert attn.last_error() == 0  # cleared
    q = torch.randn(1, 1, 128, 64).to(torch.bfloat16).cuda()
    o, lse = attn.fwd(q, q, q, True)
    assert attn.last_error() == 0
    assert torch.isfinite(o.float()).all()
