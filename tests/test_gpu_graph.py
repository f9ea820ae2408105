"""The device entry points inside CUDA graphs: each call is captured once
(torch.cuda.graph) and replayed, and every replay must equal the direct call
on the same inputs bit for bit -- also after new values are copied into the
captured input buffers, so the graph really recomputes rather than replaying
stale results.  The library makes no runtime call that stream capture forbids
once its device set-up has run (a first direct call does that)."""
import pytest
import torch

import exact_attention_124_b200 as attn

pytestmark = pytest.mark.gpu


def _randn(shape, seed, mult=1.0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.randn(shape, generator=g) * mult).to(torch.bfloat16).cuda()


def _capture(fn):
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def _replay(g):
    g.replay()
    torch.cuda.synchronize()
    assert attn.last_error() == 0


@pytest.mark.parametrize("D,causal,T", [(64, True, 300), (128, False, 257), (128, True, 1024)])
def test_forward_graph_replay_matches_direct_call(D, causal, T):
    B, H = 2, 3
    q, k, v = (_randn((B, H, T, D), 50 + i) for i in range(3))
    attn.fwd(q, k, v, causal)  # device set-up outside the capture
    o = torch.empty_like(q)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    g = _capture(lambda: attn.fwd(q, k, v, causal, o=o, lse=lse))
    for step in range(2):
        if step:
            q.copy_(_randn((B, H, T, D), 60, 2.0))
            v.copy_(_randn((B, H, T, D), 61))
        _replay(g)
        o_ref, lse_ref = attn.fwd(q, k, v, causal)
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_grouped_query_forward_graph_replay():
    B, H, H_kv, T, D = 1, 8, 2, 384, 128
    q = _randn((B, H, T, D), 70)
    k, v = _randn((B, H_kv, T, D), 71), _randn((B, H_kv, T, D), 72)
    attn.fwd_gqa(q, k, v, True)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    g = _capture(lambda: attn.fwd_gqa(q, k, v, True, o=o, lse=lse))
    k.copy_(_randn((B, H_kv, T, D), 73))
    _replay(g)
    o_ref, lse_ref = attn.fwd_gqa(q, k, v, True)
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


@pytest.mark.parametrize("splits", [0, 3, -1])
def test_decode_graph_replay_matches_direct_call(splits):
    # two launches (partials, then the merge as a programmatic dependent)
    B, H, H_kv, Tq, Tk, D = 2, 8, 2, 1, 1000, 128
    q = _randn((B, H, Tq, D), 80)
    k, v = _randn((B, H_kv, Tk, D), 81), _randn((B, H_kv, Tk, D), 82)
    attn.fwd_decode(q, k, v, True, splits=splits)
    lib = attn.load_library()
    ws = torch.empty(max(16, int(lib.attn_decode_workspace_bytes(B, H, H_kv, Tq, Tk, D, splits))),
                     dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Tq), dtype=torch.float32, device=q.device)
    g = _capture(lambda: attn.fwd_decode(q, k, v, True, splits=splits, o=o, lse=lse, ws=ws))
    for step in range(2):
        if step:
            q.copy_(_randn((B, H, Tq, D), 83, 3.0))
        _replay(g)
        o_ref, lse_ref = attn.fwd_decode(q, k, v, True, splits=splits)
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_backward_graph_replay_matches_direct_call():
    B, H, T, D = 1, 4, 384, 64
    q, k, v = (_randn((B, H, T, D), 90 + i) for i in range(3))
    do = _randn((B, H, T, D), 93)
    o, lse = attn.fwd(q, k, v, True)
    attn.bwd(q, k, v, o, lse, do, True)
    lib = attn.load_library()
    ws = torch.empty(int(lib.attn_bwd_workspace_bytes(B, H, T)), dtype=torch.uint8, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    g = _capture(lambda: attn.bwd(q, k, v, o, lse, do, True, dq=dq, dk=dk, dv=dv, ws=ws))
    for step in range(2):
        if step:
            do.copy_(_randn((B, H, T, D), 94))
        _replay(g)
        ref = attn.bwd(q, k, v, o, lse, do, True)
        assert all(torch.equal(a, b) for a, b in zip((dq, dk, dv), ref))


def test_unfused_graph_replay_matches_direct_call():
    # three kernels (S to memory, softmax, P.V) in one graph
    B, H, T, D = 1, 2, 256, 64
    q, k, v = (_randn((B, H, T, D), 100 + i) for i in range(3))
    o_ref, lse_ref, _, _ = attn.fwd_unfused(q, k, v, True)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    s_ws = torch.empty((B, H, T, T), dtype=torch.bfloat16, device=q.device)
    p_ws = torch.empty_like(s_ws)
    g = _capture(lambda: attn.fwd_unfused(q, k, v, True, o=o, lse=lse, s_ws=s_ws, p_ws=p_ws))
    for step in range(2):
        if step:
            k.copy_(_randn((B, H, T, D), 103, 2.0))
            o_ref, lse_ref, _, _ = attn.fwd_unfused(q, k, v, True)
        _replay(g)
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_host_buffer_forward_graph_replay():
    # the copies run on the library's own two streams, forked from and joined
    # back to the capturing stream through events, so the graph holds them too
    B, H, T, D = 1, 3, 200, 128
    q, k, v = (_randn((B, H, T, D), 110 + i) for i in range(3))
    qh, kh, vh = [t.cpu().pin_memory() for t in (q, k, v)]
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((B, H, T), dtype=torch.float32).pin_memory()
    dq, dk, dv, do_ = (torch.empty_like(q) for _ in range(4))
    dl = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    attn.fwd_host(qh, kh, vh, oh, lh, dq, dk, dv, do_, dl, True)  # set-up: streams, events
    torch.cuda.synchronize()
    g = _capture(lambda: attn.fwd_host(qh, kh, vh, oh, lh, dq, dk, dv, do_, dl, True))
    for step in range(2):
        if step:
            qh.copy_(_randn((B, H, T, D), 113, 2.0).cpu())
        oh.zero_()
        lh.zero_()
        _replay(g)
        o_ref, lse_ref = attn.fwd(qh.cuda(), kh.cuda(), vh.cuda(), True)
        assert torch.equal(oh, o_ref.cpu()) and torch.equal(lh, lse_ref.cpu())
