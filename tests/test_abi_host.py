"""Host-side checks of the C ABI: the library loads, exports everything the
header declares, and rejects bad arguments before touching the device.

No test here launches a kernel: every call that reaches the library carries
exactly one invalid argument, which the host-side validation catches first.
"""

import ctypes
import os
import re

import pytest
import torch

from exact_softmax_attention_03_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_expected_entry_points():
    assert header_functions() == sorted([
        "attn_fwd", "attn_fwd_f32o", "attn_fwd_varlen", "attn_bwd", "attn_bwd_workspace_bytes",
        "attn_decode_workspace_bytes", "attn_merge",
        "attn_decode",
        "attn_decode_paged", "attn_decode_noalloc", "attn_last_error", "attn_device_status",
        "attn_launch_count", "attn_debug_checks",
        "attn_selftest_wait_timeout"])


def test_release_build_is_not_the_debug_build(lib):
    assert lib.attn_debug_checks() == 0


def test_debug_build_exports_the_same_symbols_and_reports_itself():
    path = build.build(debug=True)
    dbg = ctypes.CDLL(path)
    for name in header_functions():
        assert hasattr(dbg, name), name
    dbg.attn_debug_checks.restype = ctypes.c_int
    assert dbg.attn_debug_checks() == 1


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
    assert sorted(_lib.SIGNATURES) == header_functions()


def test_status_codes_match_header():
    text = open(HEADER).read()
    for name, val in re.findall(r"(ATTN_[A-Z_]+)\s*=\s*(\d+)", text):
        assert getattr(_lib, name) == int(val)


P = 0x100000          # a 16-byte-aligned non-null address that is never dereferenced


def fwd_args(**over):
    a = dict(q=P, k=P, v=P, o=P, lse=None, B=1, Hq=4, Hkv=2, Nq=128, Nk=128, d=128,
             scale=0.125, causal=1, window_left=-1, stream=None)
    a.update(over)
    return [a[k] for k in ("q", "k", "v", "o", "lse", "B", "Hq", "Hkv", "Nq", "Nk", "d",
                           "scale", "causal", "window_left", "stream")]


BAD_FWD = [
    (dict(q=None), _lib.ATTN_ERR_INVALID_ARG),
    (dict(o=None), _lib.ATTN_ERR_INVALID_ARG),
    (dict(B=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(Nk=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), _lib.ATTN_ERR_INVALID_ARG),
    (dict(d=96), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(d=256), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(scale=0.0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), _lib.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), _lib.ATTN_ERR_INVALID_ARG),
    (dict(causal=2), _lib.ATTN_ERR_INVALID_ARG),
    (dict(k=P + 8), _lib.ATTN_ERR_INVALID_ARG),
    (dict(o=P + 2), _lib.ATTN_ERR_INVALID_ARG),
    (dict(lse=P + 1), _lib.ATTN_ERR_INVALID_ARG),
]


@pytest.mark.parametrize("entry", ["attn_fwd", "attn_fwd_f32o"])
@pytest.mark.parametrize("over,code", BAD_FWD)
def test_fwd_rejects_bad_arguments_without_launch(lib, entry, over, code):
    before = lib.attn_launch_count()
    rc = getattr(lib, entry)(*fwd_args(**over))
    assert rc == code, lib.attn_last_error()
    assert lib.attn_last_error()
    assert lib.attn_launch_count() == before


def dec_args(**over):
    a = dict(q=P, k=P, v=P, o=P, lse=None, seqlens=None, B=2, Hq=8, Hkv=2, Lmax=1000, d=128,
             scale=0.1, window_left=-1, num_splits=0, ws=P, ws_bytes=1 << 30, stream=None)
    a.update(over)
    return [a[k] for k in ("q", "k", "v", "o", "lse", "seqlens", "B", "Hq", "Hkv", "Lmax", "d",
                           "scale", "window_left", "num_splits", "ws", "ws_bytes", "stream")]


BAD_DEC = [
    (dict(q=None), _lib.ATTN_ERR_INVALID_ARG),
    (dict(Lmax=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), _lib.ATTN_ERR_INVALID_ARG),
    (dict(d=80), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(scale=-1.0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(num_splits=-1), _lib.ATTN_ERR_INVALID_ARG),
    (dict(v=P + 4), _lib.ATTN_ERR_INVALID_ARG),
    (dict(seqlens=P + 2), _lib.ATTN_ERR_INVALID_ARG),
    (dict(ws=None), _lib.ATTN_ERR_WORKSPACE),
    (dict(ws_bytes=16), _lib.ATTN_ERR_WORKSPACE),
    (dict(ws=P + 16), _lib.ATTN_ERR_INVALID_ARG),
]


@pytest.mark.parametrize("over,code", BAD_DEC)
def test_decode_rejects_bad_arguments_without_launch(lib, over, code):
    before = lib.attn_launch_count()
    rc = lib.attn_decode(*dec_args(**over))
    assert rc == code, lib.attn_last_error()
    assert lib.attn_launch_count() == before


def bwd_args(**over):
    a = dict(q=P, k=P, v=P, o=P, do=P, lse=P, dq=P, dk=P, dv=P, B=2, Hq=8, Hkv=2, Nq=256, Nk=256,
             d=128, scale=0.1, causal=1, window_left=-1, ws=P, ws_bytes=1 << 30, stream=None)
    a.update(over)
    return [a[k] for k in ("q", "k", "v", "o", "do", "lse", "dq", "dk", "dv", "B", "Hq", "Hkv",
                           "Nq", "Nk", "d", "scale", "causal", "window_left", "ws", "ws_bytes",
                           "stream")]


BAD_BWD = [
    (dict(do=None), _lib.ATTN_ERR_INVALID_ARG),
    (dict(lse=None), _lib.ATTN_ERR_INVALID_ARG),
    (dict(dk=None), _lib.ATTN_ERR_INVALID_ARG),
    (dict(dq=P + 8), _lib.ATTN_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), _lib.ATTN_ERR_INVALID_ARG),
    (dict(d=80), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(Nk=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(ws=None), _lib.ATTN_ERR_WORKSPACE),
    (dict(ws_bytes=1000), _lib.ATTN_ERR_WORKSPACE),
    (dict(ws=P + 16), _lib.ATTN_ERR_INVALID_ARG),
]


@pytest.mark.parametrize("over,code", BAD_BWD)
def test_backward_rejects_bad_arguments_without_launch(lib, over, code):
    before = lib.attn_launch_count()
    rc = lib.attn_bwd(*bwd_args(**over))
    assert rc == code, lib.attn_last_error()
    assert lib.attn_last_error()
    assert lib.attn_launch_count() == before


def test_backward_workspace_bytes(lib):
    f = lib.attn_bwd_workspace_bytes
    assert f(0, 8, 128, 128) == 0 and f(1, 8, 128, 96) == 0
    # fp32 dQ accumulator + per-row sums, each rounded to 256 bytes
    assert f(2, 8, 100, 128) == ((2 * 100 * 8 * 128 * 4 + 255) // 256 * 256
                                 + (2 * 8 * 100 * 4 + 255) // 256 * 256)


def varlen_args(**over):
    a = dict(q=P, k=P, v=P, o=P, lse=None, cq=P, ck=P, B=3, Hq=8, Hkv=2, total_q=900,
             total_k=900, max_q=512, max_k=512, d=128, scale=0.1, causal=1, window_left=-1,
             stream=None)
    a.update(over)
    return [a[k] for k in ("q", "k", "v", "o", "lse", "cq", "ck", "B", "Hq", "Hkv", "total_q",
                           "total_k", "max_q", "max_k", "d", "scale", "causal", "window_left",
                           "stream")]


BAD_VARLEN = [
    (dict(cq=None), _lib.ATTN_ERR_INVALID_ARG),
    (dict(ck=P + 2), _lib.ATTN_ERR_INVALID_ARG),
    (dict(total_q=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(max_q=1000), _lib.ATTN_ERR_INVALID_ARG),        # longer than total_q
    (dict(max_k=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(B=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), _lib.ATTN_ERR_INVALID_ARG),
    (dict(d=48), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(causal=2), _lib.ATTN_ERR_INVALID_ARG),
    (dict(o=P + 8), _lib.ATTN_ERR_INVALID_ARG),
    (dict(total_q=1 << 28, max_q=512, Hq=16, Hkv=2), _lib.ATTN_ERR_INVALID_ARG),
]


@pytest.mark.parametrize("over,code", BAD_VARLEN)
def test_varlen_rejects_bad_arguments_without_launch(lib, over, code):
    before = lib.attn_launch_count()
    rc = lib.attn_fwd_varlen(*varlen_args(**over))
    assert rc == code, lib.attn_last_error()
    assert lib.attn_last_error()
    assert lib.attn_launch_count() == before


def paged_args(**over):
    a = dict(q=P, k=P, v=P, o=P, lse=None, bt=P, seqlens=None, B=2, Hq=8, Hkv=2, num_pages=40,
             page_size=16, pages_per_seq=20, d=128, scale=0.1, window_left=-1, num_splits=0,
             ws=P, ws_bytes=1 << 30, stream=None)
    a.update(over)
    return [a[k] for k in ("q", "k", "v", "o", "lse", "bt", "seqlens", "B", "Hq", "Hkv",
                           "num_pages", "page_size", "pages_per_seq", "d", "scale", "window_left",
                           "num_splits", "ws", "ws_bytes", "stream")]


BAD_PAGED = [
    (dict(bt=None), _lib.ATTN_ERR_INVALID_ARG),
    (dict(bt=P + 2), _lib.ATTN_ERR_INVALID_ARG),
    (dict(k=None), _lib.ATTN_ERR_INVALID_ARG),
    (dict(page_size=8), _lib.ATTN_ERR_INVALID_ARG),
    (dict(page_size=48), _lib.ATTN_ERR_INVALID_ARG),
    (dict(page_size=192), _lib.ATTN_ERR_INVALID_ARG),
    (dict(num_pages=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(pages_per_seq=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), _lib.ATTN_ERR_INVALID_ARG),
    (dict(d=96), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(scale=float("nan")), _lib.ATTN_ERR_INVALID_ARG),
    (dict(pages_per_seq=1 << 27, page_size=256), _lib.ATTN_ERR_INVALID_ARG),
    (dict(ws=None), _lib.ATTN_ERR_WORKSPACE),
    (dict(ws_bytes=100), _lib.ATTN_ERR_WORKSPACE),
    (dict(ws=P + 16), _lib.ATTN_ERR_INVALID_ARG),
]


@pytest.mark.parametrize("over,code", BAD_PAGED)
def test_paged_decode_rejects_bad_arguments_without_launch(lib, over, code):
    before = lib.attn_launch_count()
    rc = lib.attn_decode_paged(*paged_args(**over))
    assert rc == code, lib.attn_last_error()
    assert lib.attn_last_error()
    assert lib.attn_launch_count() == before


def test_workspace_bytes(lib):
    f = lib.attn_decode_workspace_bytes
    assert f(0, 8, 128, 0, 100) == 0
    assert f(2, 8, 96, 0, 100) == 0
    assert f(2, 8, 128, -1, 100) == 0
    one = f(2, 8, 128, 1, 1000)
    # one split: B*Hq*d floats of partial output + B*Hq*2 floats of (max, sum), 256-byte rounded
    assert one == ((2 * 8 * 128 * 4 + 255) // 256 * 256) + ((2 * 8 * 2 * 4 + 255) // 256 * 256)
    assert f(2, 8, 128, 4, 1000) > one
    assert f(64, 32, 128, 0, 8192) > 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_a_device_reports_cuda_error(lib):
    rc = lib.attn_fwd(*fwd_args())
    assert rc == _lib.ATTN_ERR_CUDA
    assert lib.attn_launch_count() == 0


def test_binding_refuses_cpu_tensors():
    import exact_softmax_attention_03_b200 as ea
    q = torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        ea.attn_fwd(q, q, q)
    with pytest.raises(ValueError, match="CUDA"):
        ea.attn_decode(torch.zeros(1, 2, 64, dtype=torch.bfloat16), q, q)
    with pytest.raises(ValueError, match="CUDA"):
        ea.attn_decode_paged(torch.zeros(1, 2, 64, dtype=torch.bfloat16), q, q,
                             torch.zeros(1, 4, dtype=torch.int32))


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libattn.so"))
    with pytest.raises(RuntimeError, match="missing"):
        _lib.load()
