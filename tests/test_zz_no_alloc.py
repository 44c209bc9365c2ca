"""attn_decode_noalloc: decode for callers that cannot allocate device memory.

Some users of this library run inside a host program that owns all device
memory through its own pool and forbids allocations from outside it, or on a
path where an allocation's possible device synchronisation is not acceptable.
They cannot provide the decode workspace, so attn_decode_noalloc keeps the
partial results in the library's own fixed device scratch instead.

These tests call the entry point through the C ABI (ctypes, raw pointers) and
check its results against the ordinary attn_decode with a caller workspace,
within the tolerances of the other parity tests, on two calls in a row (the
second call finds the first call's leftovers in the shared scratch). Both
calls are also compared with the fp64 oracle directly: the ragged case whole,
the full decode workload on a sample of its sequences. The file is named so
that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

import attn_inputs as ai
from exact_softmax_attention_03_b200 import _lib, build

MAX_ABS, REL_L2, LSE_ABS = 2e-2, 5e-3, 1e-3


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def _close(a, b, la, lb):
    a = a.float().cpu().double().numpy()
    b = b.float().cpu().double().numpy()
    assert np.isfinite(a).all()
    d = a - b
    assert np.abs(d).max() <= MAX_ABS
    assert np.linalg.norm(d) / max(np.linalg.norm(b), 1e-30) <= REL_L2
    la, lb = la.cpu().double().numpy(), lb.cpu().double().numpy()
    assert (np.isneginf(la) == np.isneginf(lb)).all()
    fin = np.isfinite(lb)
    if fin.any():
        assert np.abs(la[fin] - lb[fin]).max() <= LSE_ABS


def test_rejects_sizes_beyond_the_fixed_scratch(lib):
    # 64 sequences x 32 heads x 64 splits x 128 floats is far above the scratch
    need = lib.attn_decode_workspace_bytes(64, 32, 128, 64, 8192)
    assert need > _lib.ATTN_DECODE_NOALLOC_SCRATCH_BYTES
    P = 0x100000
    before = lib.attn_launch_count()
    rc = lib.attn_decode_noalloc(P, P, P, P, None, None, 64, 32, 8, 8192, 128, 0.088,
                                 -1, 64, None)
    assert rc == _lib.ATTN_ERR_WORKSPACE
    assert "scratch" in lib.attn_last_error().decode()
    assert lib.attn_launch_count() == before


def _case(B, Hq, Hkv, L, d, seed, seqlens=None):
    q, kc, vc = ai.make_decode(B, Hq, Hkv, L, d, seed=seed)
    dev = torch.device("cuda")
    t = dict(q=q.to(dev), k=kc.to(dev), v=vc.to(dev),
             sl=None if seqlens is None else seqlens.to(dev))
    return t


def _noalloc_call(lib, t, wl, splits, stream):
    B, Hq, d = t["q"].shape
    _, L, Hkv, _ = t["k"].shape
    o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    rc = lib.attn_decode_noalloc(t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(),
                                 o.data_ptr(), lse.data_ptr(),
                                 t["sl"].data_ptr() if t["sl"] is not None else None,
                                 B, Hq, Hkv, L, d, float(d ** -0.5), wl, splits, stream)
    assert rc == _lib.ATTN_OK, lib.attn_last_error()
    return o, lse


def _reference_call(t, wl, splits):
    import exact_softmax_attention_03_b200 as ea
    B, Hq, d = t["q"].shape
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    o, _ = ea.attn_decode(t["q"], t["k"], t["v"], lse=lse, seqlens=t["sl"], window_left=wl,
                          num_splits=splits)
    return o, lse


@pytest.mark.gpu
def test_noalloc_matches_workspace_decode_on_two_calls_in_a_row(lib):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    stream = torch.cuda.current_stream().cuda_stream
    w = ai.GQA_DECODE
    first = _case(w.B, w.Hq, w.Hkv, w.Nk, w.d, seed=ai.SEED_Q)          # the decode workload
    second = _case(7, 8, 2, 1500, 128, seed=ai.SEED_Q + 50,
                   seqlens=ai.ragged_seqlens(7, 1500))                    # ragged, more splits
    # two calls in a row on one stream, no synchronisation in between
    o1, l1 = _noalloc_call(lib, first, -1, 0, stream)
    o2, l2 = _noalloc_call(lib, second, 300, 5, stream)
    torch.cuda.synchronize()
    assert lib.attn_device_status(stream) == _lib.ATTN_OK
    r1, rl1 = _reference_call(first, -1, 0)
    r2, rl2 = _reference_call(second, 300, 5)
    torch.cuda.synchronize()
    _close(o1, r1, l1, rl1)
    _close(o2, r2, l2, rl2)
    # and against the oracle itself, not only through the other CUDA path
    import oracle
    from parity import assert_close
    sel = [0, 21, 42, 63]                            # sequences of the decode workload
    O1, L1 = oracle.oracle_decode(first["q"][sel].cpu(), first["k"][sel].cpu(),
                                  first["v"][sel].cpu())
    assert_close(o1[sel], O1, l1[sel], L1, what="noalloc decode workload (sampled sequences)")
    O2, L2 = oracle.oracle_decode(second["q"].cpu(), second["k"].cpu(), second["v"].cpu(),
                                  seqlens=second["sl"].cpu(), window_left=300)
    assert_close(o2, O2, l2, L2, what="noalloc ragged, window 300, 5 splits")
