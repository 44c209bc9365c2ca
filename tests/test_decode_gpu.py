"""GPU parity of attn_decode (split-KV + combine) against the fp64 oracle."""

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


def run_dec(q, kc, vc, seqlens=None, wl=-1, num_splits=0):
    import exact_softmax_attention_03_b200 as ea
    qg, kg, vg = cuda(q, kc, vc)
    B, Hq, d = q.shape
    lse = torch.full((B, Hq), 5.0, device="cuda")
    sl = seqlens.cuda() if seqlens is not None else None
    o, _ = ea.attn_decode(qg, kg, vg, lse=lse, seqlens=sl, window_left=wl, num_splits=num_splits)
    assert ea.attn_device_status() == 0
    return o, lse


def check(B, Hq, Hkv, L, d, seqlens=None, wl=-1, num_splits=0, batch_subset=None):
    q, kc, vc = ai.make_decode(B, Hq, Hkv, L, d)
    o, lse = run_dec(q, kc, vc, seqlens, wl, num_splits)
    sel = list(range(B)) if batch_subset is None else batch_subset
    sl = None if seqlens is None else seqlens[sel]
    O, Lr = oracle.oracle_decode(q[sel], kc[sel], vc[sel], sl, window_left=wl)
    return assert_close(o[sel], O, lse[sel], Lr, what=(B, Hq, Hkv, L, d, wl, num_splits))


def test_decode_workload_full_size():
    w = ai.GQA_DECODE
    # all 64 sequences on the GPU, 16 of them through the oracle
    check(w.B, w.Hq, w.Hkv, w.Nk, w.d, batch_subset=list(range(0, 64, 4)))


@pytest.mark.parametrize("num_splits", [1, 2, 3, 7, 0])
def test_decode_split_counts(num_splits):
    check(4, 8, 2, 1000, 128, num_splits=num_splits)


@pytest.mark.parametrize("Hq,Hkv,d", [(8, 8, 128), (8, 1, 128), (6, 2, 128), (8, 4, 64),
                                      (16, 2, 64), (3, 3, 64), (32, 4, 128), (32, 1, 128)])
def test_decode_head_layouts(Hq, Hkv, d):
    check(3, Hq, Hkv, 777, d)


def test_decode_ragged_seqlens():
    B, L = 12, 1500
    sl = ai.ragged_seqlens(B, L)
    check(B, 8, 2, L, 128, seqlens=sl)


@pytest.mark.parametrize("wl", [0, 1, 63, 64, 500, 5000])
def test_decode_window(wl):
    sl = ai.ragged_seqlens(6, 1200)
    check(6, 8, 2, 1200, 128, seqlens=sl, wl=wl)


def test_decode_short_cache_and_empty_sequence():
    sl = torch.tensor([0, 1, 2, 31, 33], dtype=torch.int32)
    q, kc, vc = ai.make_decode(5, 4, 2, 40, 128)
    o, lse = run_dec(q, kc, vc, sl)
    assert (o[0].float() == 0).all() and torch.isneginf(lse[0]).all()
    O, Lr = oracle.oracle_decode(q[1:], kc[1:], vc[1:], sl[1:])
    assert_close(o[1:], O, lse[1:], Lr)


def test_decode_equals_last_row_of_prefill_on_gpu():
    import exact_softmax_attention_03_b200 as ea
    B, H, Hkv, L, d = 2, 8, 2, 600, 128
    q, k, v = ai.make_qkv(B, H, Hkv, L, L, d)
    qg, kg, vg = cuda(q, k, v)
    lse_p = torch.empty(B, H, L, device="cuda")
    o_p, _ = ea.attn_fwd(qg, kg, vg, lse=lse_p, causal=True)
    lse_d = torch.empty(B, H, device="cuda")
    o_d, _ = ea.attn_decode(qg[:, -1].contiguous(), kg, vg, lse=lse_d)
    torch.cuda.synchronize()
    assert (o_p[:, -1].float() - o_d.float()).abs().max().item() <= 1.6e-2
    assert (lse_p[:, :, -1] - lse_d).abs().max().item() <= 1e-3


def test_decode_caller_workspace_and_repeat():
    import exact_softmax_attention_03_b200 as ea
    q, kc, vc = ai.make_decode(4, 8, 2, 900, 128)
    qg, kg, vg = cuda(q, kc, vc)
    need = ea.attn_decode_workspace_bytes(4, 8, 128, 0, 900)
    ws = torch.full((need,), 255, dtype=torch.uint8, device="cuda")    # garbage on entry
    o1, _ = ea.attn_decode(qg, kg, vg, workspace=ws)
    o2, _ = ea.attn_decode(qg, kg, vg, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    O, _ = oracle.oracle_decode(q, kc, vc)
    assert_close(o1, O)


def test_caches_past_4_gib():
    """K and V caches of 4.56 GB each (B4 Lmax131072 Hkv34 d128: more than
    2^31 elements, byte offsets past 2^32), Hq 136 (groups of 4), ragged
    lengths with the last sequence full, so the last keys read lie past 2^32
    bytes. Eight query heads of every sequence are compared with the oracle."""
    import exact_softmax_attention_03_b200 as ea
    B, Hq, Hkv, L, d = 4, 136, 34, 131072, 128
    q, kc, vc = ai.make_decode_on("cuda", B, Hq, Hkv, L, d, seed=ai.SEED_Q + 61)
    assert kc.numel() > 2 ** 31 and kc.numel() * kc.element_size() > 2 ** 32
    sl = torch.tensor([L, 77777, 1, L], dtype=torch.int32)
    lse = torch.empty(B, Hq, device="cuda")
    o, _ = ea.attn_decode(q, kc, vc, lse=lse, seqlens=sl.cuda())
    assert ea.attn_device_status() == 0
    G = Hq // Hkv
    for b, h0 in ((0, 0), (1, 64), (2, 8), (3, Hq - 8)):
        hs = slice(h0, h0 + 8)
        ks = slice(h0 // G, (h0 + 8) // G)
        O, Lr = oracle.oracle_decode(q[b:b + 1, hs].cpu(), kc[b:b + 1, :, ks].cpu(),
                                     vc[b:b + 1, :, ks].cpu(), sl[b:b + 1])
        assert_close(o[b:b + 1, hs], O, lse[b:b + 1, hs], Lr, what=("caches past 4 GiB", b, h0))
    del q, kc, vc, o
    torch.cuda.empty_cache()
