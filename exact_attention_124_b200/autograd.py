"""A torch.autograd wrapper over the library's forward and backward entry
points: ``attention(q, k, v, causal=True, scale=None)`` returns O and is
differentiable in q, k and v.  The forward runs attn_fwd (attn_fwd_gqa when k
and v carry fewer heads than q) and keeps O and the row log-sum-exp; the
backward runs attn_bwd on them, which recomputes S and P from Q, K and the
log-sum-exp instead of storing them ("Attention Mechanism: Computation &
Memory Patterns", section 4).  Argument marshalling only: every step runs in
the library's kernels."""
import torch

from . import _lib


class _Attention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, scale):
        grouped = int(k.shape[1]) != int(q.shape[1])
        o, lse = (_lib.fwd_gqa if grouped else _lib.fwd)(q, k, v, causal, scale)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.causal = causal
        ctx.scale = scale
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = _lib.bwd(q, k, v, o, lse, do.contiguous(), ctx.causal, ctx.scale)
        return dq, dk, dv, None, None


def attention(q, k, v, causal: bool = True, scale: float | None = None):
    """O = softmax(mask(scale Q K^T)) V for bf16 CUDA tensors q [B, H, T, d_h]
    and k, v [B, H_kv, T, d_h] (H % H_kv == 0), differentiable in q, k and v."""
    return _Attention.apply(q, k, v, bool(causal), scale)
