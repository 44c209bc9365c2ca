"""GPU parity of attn_decode_paged (paged KV cache) against the fp64 oracle and
against the contiguous-cache decode on the same logical keys."""

import pytest
import torch

import attn_inputs as ai
import oracle
from parity import assert_close, cuda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from exact_softmax_attention_03_b200 import build
    build.build()


def run_paged(q, kp, vp, bt, seqlens=None, wl=-1, num_splits=0):
    import exact_softmax_attention_03_b200 as ea
    qg, kg, vg, bg = cuda(q, kp, vp, bt)
    B, Hq, d = q.shape
    lse = torch.full((B, Hq), 5.0, device="cuda")
    sl = seqlens.cuda() if seqlens is not None else None
    o, _ = ea.attn_decode_paged(qg, kg, vg, bg, lse=lse, seqlens=sl, window_left=wl,
                                num_splits=num_splits)
    assert ea.attn_device_status() == 0
    return o, lse


def check(B, Hq, Hkv, L, d, page_size, seqlens=None, wl=-1, num_splits=0):
    q, kc, vc = ai.make_decode(B, Hq, Hkv, L, d)
    kp, vp, bt = ai.make_paged(kc, vc, page_size)
    o, lse = run_paged(q, kp, vp, bt, seqlens, wl, num_splits)
    O, Lr = oracle.oracle_decode_paged(q, kp, vp, bt, seqlens, window_left=wl)
    return assert_close(o, O, lse, Lr, what=(B, Hq, Hkv, L, d, page_size, wl, num_splits))


@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
def test_page_sizes_ragged(page_size):
    L = 1024
    check(6, 8, 2, L, 128, page_size, seqlens=ai.ragged_seqlens(6, L))


@pytest.mark.parametrize("Hq,Hkv,d", [(8, 8, 128), (32, 4, 128), (8, 1, 64), (6, 2, 64)])
def test_head_layouts(Hq, Hkv, d):
    check(3, Hq, Hkv, 768, d, 32, seqlens=ai.ragged_seqlens(3, 768))


@pytest.mark.parametrize("wl", [0, 63, 500])
def test_windows(wl):
    check(5, 8, 2, 1280, 128, 16, seqlens=ai.ragged_seqlens(5, 1280), wl=wl)


@pytest.mark.parametrize("page_size,num_splits", [(16, 1), (16, 5), (128, 3), (256, 0)])
def test_bitwise_equal_to_contiguous_decode(page_size, num_splits):
    import exact_softmax_attention_03_b200 as ea
    B, Hq, Hkv, L, d = 4, 16, 4, 1536, 128
    q, kc, vc = ai.make_decode(B, Hq, Hkv, L, d)
    sl = ai.ragged_seqlens(B, L)
    kp, vp, bt = ai.make_paged(kc, vc, page_size)
    o_p, lse_p = run_paged(q, kp, vp, bt, sl, num_splits=num_splits)
    qg, kg, vg = cuda(q, kc, vc)
    lse_c = torch.empty(B, Hq, device="cuda")
    o_c, _ = ea.attn_decode(qg, kg, vg, lse=lse_c, seqlens=sl.cuda(), num_splits=num_splits)
    torch.cuda.synchronize()
    assert torch.equal(o_p, o_c) and torch.equal(lse_p, lse_c)


def test_table_entries_past_the_sequence_are_ignored():
    B, L = 4, 512
    q, kc, vc = ai.make_decode(B, 8, 2, L, 128)
    sl = torch.tensor([512, 100, 1, 300], dtype=torch.int32)
    kp, vp, bt = ai.make_paged(kc, vc, 16)
    o1, l1 = run_paged(q, kp, vp, bt, sl)
    bad = bt.clone()
    for b in range(B):
        first_unused = (int(sl[b]) + 15) // 16
        bad[b, first_unused:] = torch.where(torch.arange(bad.shape[1] - first_unused) % 2 == 0,
                                            torch.tensor(-1, dtype=torch.int32),
                                            torch.tensor(1 << 30, dtype=torch.int32))
    o2, l2 = run_paged(q, kp, vp, bad, sl)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    O, Lr = oracle.oracle_decode_paged(q, kp, vp, bt, sl)
    assert_close(o1, O, l1, Lr)


def test_decode_workload_full_size_paged_16():
    w = ai.GQA_DECODE
    q, kc, vc = ai.make_decode(w.B, w.Hq, w.Hkv, w.Nk, w.d)
    kp, vp, bt = ai.make_paged(kc, vc, 16)
    o, lse = run_paged(q, kp, vp, bt)
    sel = list(range(0, w.B, 8))
    O, Lr = oracle.oracle_decode_paged(q[sel], kp, vp, bt[sel])
    assert_close(o[sel], O, lse[sel], Lr, what="full size, page 16")
