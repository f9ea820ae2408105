"""The torch.autograd wrapper (exact_attention_124_b200.attention) runs the
library's own forward and backward: its output and its gradients equal, bit
for bit, those of attn_fwd / attn_fwd_gqa and attn_bwd called directly with
the same upstream gradient (whose parity with the oracle the forward and
backward tests establish)."""
import pytest
import torch

import exact_attention_124_b200 as attn
from attn_inputs import make_qkv
from tests.gpu_util import require_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


@pytest.mark.parametrize("B,H,H_kv,T,D,causal", [
    (1, 4, 4, 256, 128, True),
    (2, 2, 2, 200, 64, False),
    (1, 8, 2, 384, 128, True),   # grouped-query
])
def test_autograd_matches_direct_calls(B, H, H_kv, T, D, causal):
    q, _, _ = make_qkv(B, H, T, D, 3100 + T)
    _, k, v = make_qkv(B, H_kv, T, D, 3200 + T)
    q, k, v = to_dev(q, k, v)
    g = torch.Generator(device="cpu")
    g.manual_seed(3300 + T)
    w = torch.randn(B, H, T, D, generator=g).to(torch.bfloat16).cuda()
    ql, kl, vl = (t.clone().requires_grad_(True) for t in (q, k, v))
    o = attn.attention(ql, kl, vl, causal)
    (o.float() * w.float()).sum().backward()
    assert attn.last_error() == 0
    o2, lse2 = (attn.fwd_gqa if H_kv != H else attn.fwd)(q, k, v, causal)
    dq2, dk2, dv2 = attn.bwd(q, k, v, o2, lse2, w, causal)
    assert attn.last_error() == 0
    assert torch.equal(o, o2)
    assert torch.equal(ql.grad, dq2) and torch.equal(kl.grad, dk2) and torch.equal(vl.grad, dv2)
