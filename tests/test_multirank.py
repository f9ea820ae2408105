"""The N>1 host path of the benchmark on CPU ranks (gloo, world size 2):
each rank draws its own seeded inputs, no data crosses ranks, and the job's
step time is the maximum over ranks.  Heads are independent ("Attention
Mechanism: Computation & Memory Patterns", section 2 counts memory per head),
so ranks run whole workloads side by side (weak scaling)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from attn_inputs import WORKLOADS, make_qkv


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = WORKLOADS["tiny_causal_T128_d64"]
        seed = bench.rank_seed(w, rank)
        q, _, _ = make_qkv(w.B, w.H, w.T, w.D, seed)
        local_ms = 1.0 + rank  # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, world)
        out[rank] = (seed, float(q.float().sum()), ms,
                     bench.whole_job_tflops(w.flops(), world, ms))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    (s0, x0, ms0, v0), (s1, x1, ms1, v1) = out[0], out[1]
    assert s0 != s1 and x0 != x1          # independent inputs per rank
    assert ms0 == ms1 == 2.0              # both report the slowest rank
    w = WORKLOADS["tiny_causal_T128_d64"]
    assert v0 == v1 == pytest.approx(w.flops() * 2 / 2e-3 / 1e12)


def test_single_rank_is_plain():
    assert bench.max_over_ranks(3.5, 1) == 3.5
