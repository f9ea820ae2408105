"""ctypes binding of ``libattn_b200.so`` -- argument marshalling only.

Names follow the C ABI (include/attn.h, include/attn_selftest.h).  Tensors
must already live on the current CUDA device; their ``data_ptr()`` and the
current torch stream are handed to the library, which does all the work.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libattn_b200.so")
_lib = None

ATTN_OK = 0


class AttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_str(code) if _lib else code} (status {code})")


def library_path() -> str:
    return _SO


def load_library():
    """Load the in-tree CUDA library; raise if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_SO):
        raise ImportError(f"{_SO} is missing: build it with `python -m exact_attention_124_b200.build`"
                          " (the attention path has no fallback)")
    lib = ctypes.CDLL(_SO)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, F, P]
    lib.attn_fwd_gqa.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.attn_fwd_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, F, I, P]
    lib.attn_decode_workspace_bytes.argtypes = [I, I, I, I, I, I, I]
    lib.attn_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_bwd_workspace_bytes.argtypes = [I, I, I]
    lib.attn_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_fwd_unfused.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, F, P]
    lib.attn_fwd_host.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, F, P]
    lib.attn_unfused_workspace_bytes.argtypes = [I, I, I]
    lib.attn_unfused_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_last_error.argtypes = []
    lib.attn_status_str.argtypes = [I]
    lib.attn_status_str.restype = ctypes.c_char_p
    lib.attn_fused_grid_ctas.argtypes = [I, I, I, I, I]
    lib.attn_version.restype = ctypes.c_char_p
    lib.attn_selftest_qk_tile.argtypes = [P, P, P, I, P]
    lib.attn_selftest_pv_tile.argtypes = [P, P, P, I, P]
    lib.attn_selftest_timeout.argtypes = [I, P]
    lib.attn_selftest_set_mma_order.argtypes = [I]
    lib.attn_selftest_last_wait_site.argtypes = []
    lib.attn_selftest_set_exp_split.argtypes = [I]
    lib.attn_selftest_decode_plan.argtypes = [I, I, I, I, I, I, I, P, I, P, I, P, P]
    lib.attn_selftest_fused_plan.argtypes = [I, I, I, I, I, I, P, I, P]
    for name in ("attn_fwd", "attn_fwd_gqa", "attn_bwd", "attn_fwd_decode", "attn_fwd_unfused", "attn_fwd_host", "attn_last_error",
                 "attn_fused_grid_ctas", "attn_selftest_qk_tile", "attn_selftest_pv_tile",
                 "attn_selftest_timeout", "attn_selftest_set_mma_order",
                 "attn_selftest_last_wait_site", "attn_selftest_set_exp_split",
                 "attn_selftest_decode_plan",
                 "attn_selftest_fused_plan"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def status_str(code: int) -> str:
    return load_library().attn_status_str(int(code)).decode()


def version() -> str:
    return load_library().attn_version().decode()


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(rc: int, what: str):
    if rc != ATTN_OK:
        raise AttnError(rc, what)


def _shape(q: torch.Tensor):
    if q.dim() != 4:
        raise ValueError("expected [B, H, T, d_h] tensors")
    return tuple(int(x) for x in q.shape)


def _want(t: torch.Tensor, name: str):
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")


def fwd(q, k, v, causal: bool, scale: float | None = None, o=None, lse=None, stream=None):
    """Fused forward.  Returns (o bf16 [B,H,T,d_h], lse fp32 [B,H,T])."""
    lib = load_library()
    B, H, T, D = _shape(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _want(t, n)
        if tuple(t.shape) != (B, H, T, D):
            raise ValueError("q, k, v shapes differ")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    rc = lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                      B, H, T, D, int(bool(causal)), float(scale), _stream(stream))
    _check(rc, "attn_fwd")
    return o, lse


def fwd_gqa(q, k, v, causal: bool, scale: float | None = None, o=None, lse=None, stream=None):
    """Fused forward with grouped-query attention: q [B, H, T, d_h], k and v
    [B, H_kv, T, d_h] with H % H_kv == 0.  Returns (o, lse)."""
    lib = load_library()
    B, H, T, D = _shape(q)
    Bk, H_kv, Tk, Dk = _shape(k)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _want(t, n)
    if (Bk, Tk, Dk) != (B, T, D) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k/v must be [B, H_kv, T, d_h] matching q")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    rc = lib.attn_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                          B, H, H_kv, T, D, int(bool(causal)), float(scale), _stream(stream))
    _check(rc, "attn_fwd_gqa")
    return o, lse


def bwd(q, k, v, o, lse, dout, causal: bool, scale: float | None = None, dq=None, dk=None,
        dv=None, ws=None, stream=None):
    """Backward pass: gradients (dq, dk, dv) from the forward's o and lse and
    the output gradient dout.  q/o/dout [B, H, T, d_h], k/v [B, H_kv, T, d_h],
    any T."""
    lib = load_library()
    B, H, T, D = _shape(q)
    H_kv = int(k.shape[1])
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _want(t, n)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if ws is None:
        ws = torch.empty(int(lib.attn_bwd_workspace_bytes(B, H, T)), dtype=torch.uint8,
                         device=q.device)
    rc = lib.attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                      dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(),
                      B, H, H_kv, T, D, int(bool(causal)), float(scale), _stream(stream))
    _check(rc, "attn_bwd")
    return dq, dk, dv


def fwd_decode(q, k, v, causal: bool, scale: float | None = None, splits: int = 0, o=None,
               lse=None, ws=None, stream=None):
    """Decode forward: q [B, H, Tq, d_h] against a cache k/v [B, H_kv, Tk, d_h]
    (query i at position Tk - Tq + i), split-KV over ``splits`` key ranges per head
    (< 0: balanced ranges of all heads' tiles over the SMs)
    (0: automatic).  Returns (o, lse)."""
    lib = load_library()
    B, H, Tq, D = _shape(q)
    _, H_kv, Tk, _ = _shape(k)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _want(t, n)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Tq), dtype=torch.float32, device=q.device)
    if ws is None:
        nbytes = int(lib.attn_decode_workspace_bytes(B, H, H_kv, Tq, Tk, D, int(splits)))
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    rc = lib.attn_fwd_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             lse.data_ptr(), ws.data_ptr(), B, H, H_kv, Tq, Tk, D,
                             int(bool(causal)), float(scale), int(splits), _stream(stream))
    _check(rc, "attn_fwd_decode")
    return o, lse


def unfused_workspace_bytes(B: int, H: int, T: int) -> int:
    return int(load_library().attn_unfused_workspace_bytes(B, H, T))


def fwd_unfused(q, k, v, causal: bool, scale: float | None = None, o=None, lse=None,
                s_ws=None, p_ws=None, stream=None):
    """Three-kernel forward with S and P in device memory.
    Returns (o, lse, s_ws, p_ws); the workspaces hold S and P ([B,H,T,T] bf16)."""
    lib = load_library()
    B, H, T, D = _shape(q)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    if s_ws is None:
        s_ws = torch.empty((B, H, T, T), dtype=torch.bfloat16, device=q.device)
    if p_ws is None:
        p_ws = torch.empty((B, H, T, T), dtype=torch.bfloat16, device=q.device)
    rc = lib.attn_fwd_unfused(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              lse.data_ptr(), s_ws.data_ptr(), p_ws.data_ptr(), B, H, T, D,
                              int(bool(causal)), float(scale), _stream(stream))
    _check(rc, "attn_fwd_unfused")
    return o, lse, s_ws, p_ws


def fwd_host(q_host, k_host, v_host, o_host, lse_host, dq, dk, dv, do_, dlse, causal: bool,
             scale: float | None = None, stream=None):
    """Host-buffer forward: H2D copies, the fused kernel and D2H copies, all
    enqueued on ``stream`` by the library.  Host tensors should be pinned."""
    lib = load_library()
    B, H, T, D = _shape(q_host)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    rc = lib.attn_fwd_host(q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(),
                           o_host.data_ptr(), lse_host.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                           dv.data_ptr(), do_.data_ptr(), dlse.data_ptr(), B, H, T, D,
                           int(bool(causal)), float(scale), _stream(stream))
    _check(rc, "attn_fwd_host")


def last_error() -> int:
    """Synchronise the device and return (and clear) the device status word."""
    return int(load_library().attn_last_error())


def last_wait_site() -> int:
    return int(load_library().attn_selftest_last_wait_site())


def set_mma_order(mode: int) -> int:
    prev = load_library().attn_selftest_set_mma_order(int(mode))
    if prev < 0:
        raise ValueError("mode must be 0 or 1")
    return prev


def set_exp_split(pairs_of_8: int) -> int:
    """Column pairs out of every 8 whose exponentials run on the FMA pipe
    (0, 2, 3, 4; -1 = default).  Returns the previous setting."""
    prev = load_library().attn_selftest_set_exp_split(int(pairs_of_8))
    if prev == -2:
        raise ValueError("exp split must be -1, 0, 2, 3 or 4")
    return prev


def fused_plan(B: int, H: int, H_kv: int, T: int, causal: bool, sms: int):
    """Host-side work units of the fused forward on a device with ``sms`` SMs
    (no device needed): (units, ctas) with units a list of
    (cta, k, query_head, kv_head, first_row, n0, n1) tuples."""
    lib = load_library()
    ctas = ctypes.c_int(0)
    n = lib.attn_selftest_fused_plan(B, H, H_kv, T, int(bool(causal)), sms, None, 0,
                                     ctypes.byref(ctas))
    if n < 0:
        raise ValueError("bad sizes")
    buf = (ctypes.c_int * (7 * max(n, 1)))()
    n2 = lib.attn_selftest_fused_plan(B, H, H_kv, T, int(bool(causal)), sms, buf, n,
                                      ctypes.byref(ctas))
    assert n2 == n
    return [tuple(buf[7 * i:7 * i + 7]) for i in range(n)], ctas.value


def decode_plan(B: int, H: int, H_kv: int, Tq: int, Tk: int, splits: int, sms: int):
    """Host-side work plan of attn_fwd_decode on a device with ``sms`` SMs
    (no device needed): (segments, nseg, slots, copies) with segments a list of
    (cta_x, cta_y, cta_z, kvbh, row_block, first_tile, tiles, first_slot)
    tuples (a segment fills slots first_slot .. first_slot + copies - 1) and
    nseg[w] the partial slots the merge reads for head w."""
    lib = load_library()
    nrb = ((H // H_kv) * Tq + 127) // 128 if H_kv > 0 and H % H_kv == 0 else 0
    heads = B * H_kv * nrb
    slots, copies = ctypes.c_int(0), ctypes.c_int(0)
    n = lib.attn_selftest_decode_plan(B, H, H_kv, Tq, Tk, splits, sms, None, 0, None, 0,
                                      ctypes.byref(slots), ctypes.byref(copies))
    if n < 0:
        raise ValueError("bad decode sizes")
    segs = (ctypes.c_int * (8 * max(n, 1)))()
    nseg = (ctypes.c_int * max(heads, 1))()
    n2 = lib.attn_selftest_decode_plan(B, H, H_kv, Tq, Tk, splits, sms, segs, n, nseg, heads,
                                       ctypes.byref(slots), ctypes.byref(copies))
    assert n2 == n
    return ([tuple(segs[8 * i:8 * i + 8]) for i in range(n)], list(nseg[:heads]), slots.value,
            copies.value)


def fused_grid_ctas(B: int, H: int, T: int, D: int, causal: bool) -> int:
    return int(load_library().attn_fused_grid_ctas(B, H, T, D, int(bool(causal))))


def selftest_qk_tile(q, k, stream=None):
    lib = load_library()
    D = int(q.shape[-1])
    s = torch.empty((128, 128), dtype=torch.float32, device=q.device)
    _check(lib.attn_selftest_qk_tile(q.data_ptr(), k.data_ptr(), s.data_ptr(), D,
                                     _stream(stream)), "attn_selftest_qk_tile")
    return s


def selftest_pv_tile(p, v, stream=None):
    lib = load_library()
    D = int(v.shape[-1])
    o = torch.empty((128, D), dtype=torch.float32, device=v.device)
    _check(lib.attn_selftest_pv_tile(p.data_ptr(), v.data_ptr(), o.data_ptr(), D,
                                     _stream(stream)), "attn_selftest_pv_tile")
    return o


def selftest_timeout(limit_us: int, stream=None):
    _check(load_library().attn_selftest_timeout(int(limit_us), _stream(stream)),
           "attn_selftest_timeout")
