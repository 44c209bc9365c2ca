"""Property tests of the C ABI's host-side checks (CPU, no device).

Random sizes, flags, scales, pointers and alignments, extremes included. Every
entry point must return one of the header's status codes together with a
message, launch nothing, and never bring the process down (an integer overflow
in a size check, a division by zero). The workspace queries must return either
0 (sizes refused) or at least the bytes their layouts need.

Skipped where a GPU is present: there a call that passes every check would
launch kernels on the fake pointers used here.
"""

import ctypes

import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from exact_softmax_attention_03_b200 import _lib, build

pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="a call that passes the checks would launch on fake pointers")

P = 0x100000                      # 16-byte aligned, never dereferenced
CODES = {_lib.ATTN_ERR_INVALID_ARG, _lib.ATTN_ERR_UNSUPPORTED, _lib.ATTN_ERR_CUDA,
         _lib.ATTN_ERR_WORKSPACE}
EDGES = [-2**31, -1, 0, 1, 2, 3, 7, 16, 63, 64, 65, 127, 128, 129, 255, 256, 1000, 4096, 8192,
         65535, 65536, 2**20, 2**30, 2**31 - 128, 2**31 - 127, 2**31 - 1]

i32 = st.one_of(st.sampled_from(EDGES), st.integers(-2**31, 2**31 - 1), st.integers(1, 300))
small = st.one_of(st.sampled_from(EDGES), st.integers(1, 64))
dims = st.sampled_from([-1, 0, 16, 32, 48, 64, 80, 96, 128, 256, 2**31 - 1])
flag = st.sampled_from([-1, 0, 1, 2])
ptr = st.sampled_from([None, P, P + 1, P + 2, P + 4, P + 8, P + 16, P + 256])
fptr = st.sampled_from([None, P, P + 1, P + 2, P + 4, P + 16])
scale = st.one_of(st.sampled_from([0.0, -1.0, float("nan"), float("inf"), 1e-30, 0.088, 1.0, 1e30]),
                  st.floats(allow_nan=True, allow_infinity=True, width=32))
nbytes = st.one_of(st.sampled_from([0, 1, 16, 2**20, 2**40, 2**64 - 1]), st.integers(0, 2**64 - 1))

SETTINGS = settings(max_examples=400, deadline=None,
                    suppress_health_check=[HealthCheck.too_slow, HealthCheck.function_scoped_fixture])


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def _check(lib, rc):
    assert rc in CODES, rc
    msg = lib.attn_last_error()
    assert msg, rc
    assert lib.attn_launch_count() == 0


@SETTINGS
@given(q=ptr, k=ptr, v=ptr, o=ptr, lse=fptr, B=small, Hq=small, Hkv=small, Nq=i32, Nk=i32, d=dims,
       sc=scale, causal=flag, wl=i32, f32=st.booleans())
def test_forward_checks(lib, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, sc, causal, wl, f32):
    fn = lib.attn_fwd_f32o if f32 else lib.attn_fwd
    _check(lib, fn(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, sc, causal, wl, None))


@SETTINGS
@given(q=ptr, k=ptr, v=ptr, o=ptr, lse=fptr, cq=fptr, ck=fptr, B=small, Hq=small, Hkv=small,
       tq=i32, tk=i32, mq=i32, mk=i32, d=dims, sc=scale, causal=flag, wl=i32)
def test_varlen_checks(lib, q, k, v, o, lse, cq, ck, B, Hq, Hkv, tq, tk, mq, mk, d, sc, causal, wl):
    _check(lib, lib.attn_fwd_varlen(q, k, v, o, lse, cq, ck, B, Hq, Hkv, tq, tk, mq, mk, d, sc,
                                    causal, wl, None))


@SETTINGS
@given(q=ptr, k=ptr, v=ptr, o=ptr, do=ptr, lse=fptr, dq=ptr, dk=ptr, dv=ptr, B=small, Hq=small,
       Hkv=small, Nq=i32, Nk=i32, d=dims, sc=scale, causal=flag, wl=i32, ws=ptr, wsb=nbytes)
def test_backward_checks(lib, q, k, v, o, do, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, sc, causal,
                         wl, ws, wsb):
    _check(lib, lib.attn_bwd(q, k, v, o, do, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, sc, causal,
                             wl, ws, wsb, None))


@SETTINGS
@given(q=ptr, k=ptr, v=ptr, o=ptr, lse=fptr, sl=fptr, B=small, Hq=small, Hkv=small, L=i32,
       d=dims, sc=scale, wl=i32, S=i32, ws=ptr, wsb=nbytes, noalloc=st.booleans())
def test_decode_checks(lib, q, k, v, o, lse, sl, B, Hq, Hkv, L, d, sc, wl, S, ws, wsb, noalloc):
    if noalloc:
        rc = lib.attn_decode_noalloc(q, k, v, o, lse, sl, B, Hq, Hkv, L, d, sc, wl, S, None)
    else:
        rc = lib.attn_decode(q, k, v, o, lse, sl, B, Hq, Hkv, L, d, sc, wl, S, ws, wsb, None)
    _check(lib, rc)


@SETTINGS
@given(q=ptr, k=ptr, v=ptr, o=ptr, lse=fptr, bt=fptr, sl=fptr, B=small, Hq=small, Hkv=small,
       npages=i32, ps=st.one_of(st.sampled_from([16, 32, 48, 64, 128, 192, 256, 2**30]), i32),
       pps=i32, d=dims, sc=scale, wl=i32, S=i32, ws=ptr, wsb=nbytes)
def test_paged_decode_checks(lib, q, k, v, o, lse, bt, sl, B, Hq, Hkv, npages, ps, pps, d, sc, wl,
                             S, ws, wsb):
    _check(lib, lib.attn_decode_paged(q, k, v, o, lse, bt, sl, B, Hq, Hkv, npages, ps, pps, d, sc,
                                      wl, S, ws, wsb, None))


@SETTINGS
@given(op=fptr, lp=fptr, R=st.one_of(small, st.integers(60, 70)), o=ptr, lse=fptr, B=small,
       Nq=i32, Hq=small, d=dims)
def test_merge_checks(lib, op, lp, R, o, lse, B, Nq, Hq, d):
    _check(lib, lib.attn_merge(op, lp, R, o, lse, B, Nq, Hq, d, None))


@SETTINGS
@given(B=small, Hq=small, d=dims, S=i32, L=i32)
def test_decode_workspace_query(lib, B, Hq, d, S, L):
    n = lib.attn_decode_workspace_bytes(B, Hq, d, S, L)
    if n:
        assert B >= 1 and Hq >= 1 and d in (64, 128) and S >= 0 and 1 <= L <= 2**31 - 128
        # at least one split: B*Hq rows of d partial outputs and a (max, sum) pair
        assert n >= B * Hq * (d + 2) * 4
        assert n % 256 == 0
        assert n <= 2**62 + 512


@SETTINGS
@given(B=small, Hq=small, Nq=i32, d=dims)
def test_backward_workspace_query(lib, B, Hq, Nq, d):
    n = lib.attn_bwd_workspace_bytes(B, Hq, Nq, d)
    if n:
        def r256(x):
            return (x + 255) // 256 * 256
        assert n == r256(B * Nq * Hq * d * 4) + r256(B * Hq * Nq * 4)
    elif B >= 1 and Hq >= 1 and Nq >= 1 and d in (64, 128):
        # refused only beyond the limits attn_bwd applies
        assert B * Nq > 2**31 - 1 or B * Hq > 2**31 - 1 or B * Nq * Hq * d > (2**31 - 1) * 8
