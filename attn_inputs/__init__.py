"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This module holds workload shapes and random-number recipes only; none of the
attention arithmetic lives here.  Both sides receive the very same bf16 tensors.

Recipe (one head is a T x d_h slab of a [B, H, T, d_h] contiguous tensor, the
shape the pages give for Q, K and V: "Why Attention Is Difficult to Optimize",
section "The Attention Computation Flow"; "Attention Mechanism: Computation &
Memory Patterns", section 1):

* ``torch.Generator('cpu').manual_seed(seed)``;
* Q, then K, then V drawn with ``torch.randn(B, H, T, d_h, dtype=float32)``;
* each rounded to bf16 (round-to-nearest-even, torch's conversion);
* for the "logit stress" workload Q and K are multiplied by 4 after rounding
  (exact: a power of two), so scaled logits have a standard deviation near 16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    """One synthetic attention workload: shapes, mask and seed."""

    name: str
    B: int
    H: int
    T: int
    D: int
    causal: bool
    seed: int
    qk_mult: float = 1.0
    note: str = ""

    @property
    def scale(self) -> float:
        """Score scale passed to the kernels (1/sqrt(d_h), the configs' choice)."""
        return 1.0 / math.sqrt(self.D)

    @property
    def heads(self) -> int:
        return self.B * self.H

    def flops(self) -> float:
        """Counted FLOPs: 4*T^2*d_h per head, halved when causal."""
        f = 4.0 * self.T * self.T * self.D * self.heads
        return f / 2.0 if self.causal else f

    def describe(self) -> str:
        m = "causal" if self.causal else "full"
        x = f", QK x{self.qk_mult:g}" if self.qk_mult != 1.0 else ""
        return f"B={self.B} H={self.H} T={self.T} d_h={self.D} {m}{x}"


# The five workloads: shapes, masks and value distributions as specified for
# this path (T = 4,096 and 8,192 are the sizes of the pages' worked examples,
# 65,536 stands in for their "64k").
WORKLOADS = {
    "tiny_causal_T128_d64": Workload("tiny_causal_T128_d64", 1, 1, 128, 64, True, 1001),
    "causal_T4096_d64": Workload("causal_T4096_d64", 8, 16, 4096, 64, True, 1002),
    "causal_T8192_d128": Workload("causal_T8192_d128", 4, 32, 8192, 128, True, 1003),
    "full_T2048_d128_qk4": Workload("full_T2048_d128_qk4", 16, 16, 2048, 128, False, 1004, 4.0),
    "causal_T65536_d128": Workload("causal_T65536_d128", 1, 8, 65536, 128, True, 1005),
}
ORDER = list(WORKLOADS)  # smallest first; index 2 is the T=8192, d_h=128 headline case


def make_qkv(B: int, H: int, T: int, D: int, seed: int, qk_mult: float = 1.0):
    """Return CPU bf16 tensors (q, k, v), each [B, H, T, D] contiguous."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    out = []
    for _ in range(3):
        x = torch.randn((B, H, T, D), generator=g, dtype=torch.float32)
        out.append(x.to(torch.bfloat16))
    q, k, v = out
    if qk_mult != 1.0:
        q = q * qk_mult
        k = k * qk_mult
    return q.contiguous(), k.contiguous(), v.contiguous()


def make_workload(w: Workload):
    return make_qkv(w.B, w.H, w.T, w.D, w.seed, w.qk_mult)


def sample_rows(T: int, seed: int, n_random: int = 512):
    """Rows checked one by one at full size: the first and last 256, every
    97th, and ``n_random`` seeded random rows (sorted, unique)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + 77)
    rows = set(range(min(T, 256)))
    rows.update(range(max(0, T - 256), T))
    rows.update(range(0, T, 97))
    if n_random:
        rows.update(torch.randint(0, T, (n_random,), generator=g).tolist())
    return sorted(rows)


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 array of its bit patterns (no copy of values)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view("uint16")
