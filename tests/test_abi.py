"""The C-ABI library (no GPU needed): it builds for sm_100a, loads, exports
every symbol the headers declare, and rejects bad arguments on the host
before any CUDA work.  The product path has no fallback when it is missing."""
import ctypes
import os
import re

import pytest

import exact_attention_124_b200 as attn
from exact_attention_124_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("attn.h", "attn_selftest.h")]


@pytest.fixture(scope="module")
def lib():
    build.build()
    return attn.load_library()


def declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(attn_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_headers_declare_the_boundary():
    names = declared_functions()
    for must in ("attn_fwd", "attn_fwd_unfused", "attn_fwd_host", "attn_last_error",
                 "attn_status_str", "attn_unfused_workspace_bytes"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(_lib.library_path())
    for name in declared_functions():
        assert hasattr(raw, name), name


def declared_parameter_counts():
    """Parameter count of every declared function, from the headers."""
    counts = {}
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        for m in re.finditer(r"\b(attn_\w+)\s*\(([^)]*)\)\s*;", text):
            params = m.group(2).strip()
            counts[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return counts


def test_binding_signatures_match_the_headers(lib):
    """Every ctypes signature the binding sets has the headers' parameter count."""
    counts = declared_parameter_counts()
    assert set(counts) == set(declared_functions())
    checked = 0
    for name, n in counts.items():
        argtypes = getattr(lib, name).argtypes
        if argtypes is not None:
            assert len(argtypes) == n, (name, len(argtypes), n)
            checked += 1
    assert checked >= 15


NULL = None
A = 4096  # a 16-byte aligned fake address: never dereferenced, validation fails first


@pytest.mark.parametrize("args,code", [
    ((NULL, A, A, A, A, 1, 1, 128, 64, 1, 0.125), 1),
    ((A, A, A, A, NULL, 1, 1, 128, 64, 1, 0.125), 1),
    ((A, A, A, A, A, 1, 1, 128, 96, 1, 0.125), 2),
    ((A, A, A, A, A, 1, 1, 128, 32, 1, 0.125), 2),
    ((A, A, A, A, A, 0, 1, 128, 64, 1, 0.125), 3),
    ((A, A, A, A, A, 1, 1, 0, 64, 1, 0.125), 3),
    ((A, A, A, A, A, 65536, 65536, 128, 64, 1, 0.125), 3),
    ((A + 8, A, A, A, A, 1, 1, 128, 64, 1, 0.125), 4),
    ((A, A, A, A, A + 2, 1, 1, 128, 64, 1, 0.125), 4),  # lse needs float alignment
    ((A, A, A, A, A, 1, 1, 128, 64, 1, float("nan")), 5),
    ((A, A, A, A, A, 1, 1, 128, 64, 1, -1.0), 5),
    ((A, A, A, A, A, 1, 1, 128, 64, 1, 0.0), 5),
    ((A, A, A, A, A, 1, 1, 128, 64, 2, 0.125), 9),
])
def test_fused_rejects_bad_arguments_on_host(lib, args, code):
    assert lib.attn_fwd(*args, None) == code


def test_unfused_rejects_bad_arguments_on_host(lib):
    ok = (A, A, A, A, A, A, A, 1, 1, 256, 64, 1, 0.125, None)
    bad_t = ok[:9] + (200,) + ok[10:]
    assert lib.attn_fwd_unfused(*bad_t) == 3
    no_ws = ok[:5] + (None, A) + ok[7:]
    assert lib.attn_fwd_unfused(*no_ws) == 1
    mis = ok[:5] + (A + 2, A) + ok[7:]
    assert lib.attn_fwd_unfused(*mis) == 4


def test_host_variant_rejects_null_host_buffers(lib):
    args = (None, A, A, A, A, A, A, A, A, A, 1, 1, 128, 64, 1, 0.125, None)
    assert lib.attn_fwd_host(*args) == 1


def test_workspace_size_and_status_strings(lib):
    assert attn.unfused_workspace_bytes(8, 16, 4096) == 8 * 16 * 4096 * 4096 * 2
    assert attn.unfused_workspace_bytes(0, 16, 4096) == 0
    assert "timed out" in attn.status_str(7)
    assert attn.status_str(0) == "ok"
    assert re.match(r"^\d+\.\d+\.\d+$", attn.version())


def test_no_fallback_when_library_missing(monkeypatch):
    monkeypatch.setattr(_lib, "_SO", "/nonexistent/libattn_b200.so")
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(ImportError):
        _lib.load_library()


def test_mma_order_switch(lib):
    prev = attn.set_mma_order(1)
    assert attn.set_mma_order(prev) == 1
    with pytest.raises(ValueError):
        attn.set_mma_order(3)


def test_gqa_rejects_bad_head_grouping(lib):
    # H = 6 query heads cannot share H_kv = 4 K/V heads
    assert lib.attn_fwd_gqa(A, A, A, A, A, 1, 6, 4, 128, 64, 1, 0.125, None) == 3
    assert lib.attn_fwd_gqa(A, A, A, A, A, 1, 6, 0, 128, 64, 1, 0.125, None) == 3
    assert lib.attn_fwd_gqa(None, A, A, A, A, 1, 6, 3, 128, 64, 1, 0.125, None) == 1


def test_backward_rejects_bad_arguments(lib):
    ok = [A, A, A, A, A, A, A, A, A, A, 1, 4, 2, 256, 128, 1, 0.125, None]
    bad = list(ok); bad[9] = None            # no workspace
    assert lib.attn_bwd(*bad) == 1
    bad = list(ok); bad[12] = 3              # 4 heads over 3 K/V heads
    assert lib.attn_bwd(*bad) == 3
    bad = list(ok); bad[6] = A + 8           # misaligned dq
    assert lib.attn_bwd(*bad) == 4
    bad = list(ok); bad[14] = 80             # unsupported head size
    assert lib.attn_bwd(*bad) == 2
    assert attn.load_library().attn_bwd_workspace_bytes(2, 4, 256) == 2 * 4 * 256 * 8
    # a ragged T is padded to whole 128-row blocks of statistics
    assert attn.load_library().attn_bwd_workspace_bytes(2, 4, 200) == 2 * 4 * 256 * 8


def test_decode_rejects_bad_arguments(lib):
    ok = [A, A, A, A, A, A, 1, 8, 2, 4, 1024, 128, 1, 0.125, 0, None]
    bad = list(ok); bad[5] = None            # no workspace
    assert lib.attn_fwd_decode(*bad) == 1
    bad = list(ok); bad[10] = 2              # cache shorter than the new queries
    assert lib.attn_fwd_decode(*bad) == 3
    bad = list(ok); bad[8] = 3               # 8 heads over 3 K/V heads
    assert lib.attn_fwd_decode(*bad) == 3
    # workspace size with explicit splits needs no device: 4 splits x rows x (d + 1) floats
    # 4 splits x 4 copies of the 16 packed rows (group 4 x Tq 4), B*H*Tq rows of (d_h + 1) floats
    assert lib.attn_decode_workspace_bytes(1, 8, 2, 4, 1024, 128, 4) == 4 * 4 * 1 * 8 * 4 * 129 * 4
    # 80 packed rows (group 4 x Tq 20): one copy
    assert lib.attn_decode_workspace_bytes(1, 8, 2, 20, 1024, 128, 4) == 4 * 1 * 8 * 20 * 129 * 4
