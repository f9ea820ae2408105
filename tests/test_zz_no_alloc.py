"""The allocation-free unfused forward (attn_fwd_unfused_noalloc).

It serves callers that cannot call cudaMalloc -- a plug-in inside a host
application that owns the device through its own memory pool, or code that
must not risk the synchronisation an allocation can cause -- by keeping S and
P in a static device array inside the library instead of caller workspaces.
These tests call it through the C ABI and check it against the workspace
entry point (attn_fwd_unfused) on two calls in a row, so contents left in the
shared array by the first call cannot leak into the second.  This file is
collected last on purpose.
"""
import ctypes
import math

import pytest
import torch

import exact_attention_124_b200 as attn
from exact_attention_124_b200 import _lib
from attn_inputs import make_qkv
from tests.parity import LSE_TOL, O_MAX_ABS, O_MEAN_ABS

pytestmark = pytest.mark.gpu

ATTN_ERR_WORKSPACE_LIMIT = 10


def _handle():
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"
    attn.load_library()
    lib = ctypes.CDLL(_lib.library_path())
    f = lib.attn_fwd_unfused_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, P, P, I, I, I, I, I, ctypes.c_float, P]
    f.restype = ctypes.c_int
    return f


def _call(f, q, k, v, o, lse, causal):
    B, H, T, D = q.shape
    return f(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, T, D,
             int(causal), 1.0 / math.sqrt(D), torch.cuda.current_stream().cuda_stream)


def test_matches_workspace_entry_point_on_two_calls_in_a_row():
    f = _handle()
    cases = [((1, 4, 1024, 128), True, 4101), ((2, 2, 512, 64), False, 4102)]
    for shape, causal, seed in cases:
        q, k, v = [t.cuda() for t in make_qkv(*shape, seed)]
        o_ref, lse_ref, _, _ = attn.fwd_unfused(q, k, v, causal)
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
        assert _call(f, q, k, v, o, lse, causal) == 0
        assert attn.last_error() == 0
        err = (o.double() - o_ref.double()).abs()
        assert err.max().item() <= O_MAX_ABS and err.mean().item() <= O_MEAN_ABS, shape
        lerr = (lse.double() - lse_ref.double()).abs() / lse_ref.double().abs().clamp(min=1.0)
        assert lerr.max().item() <= LSE_TOL, shape


def test_rejects_problems_beyond_the_static_workspace():
    f = _handle()
    q = torch.zeros((1, 2, 4096, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 2, 4096), dtype=torch.float32, device="cuda")
    # 2 heads x 4096^2 entries exceed the 16,777,216 each of S and P can hold
    assert _call(f, q, q, q, q, lse, True) == ATTN_ERR_WORKSPACE_LIMIT
    assert attn.last_error() == 0
