"""GPU parity of attn_fwd_varlen (packed variable-length sequences) against the
fp64 oracle, against attn_fwd on each sequence alone (bit for bit), and for
the device-side check of the sequence offsets."""

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


SENT_O, SENT_L = 7.0, 9.0


def run_varlen(q, k, v, cq, ck, causal, wl, max_q=None, max_k=None, expect_status=0):
    import exact_softmax_attention_03_b200 as ea
    qg, kg, vg, cqg, ckg = cuda(q, k, v, cq, ck)
    total_q, Hq, d = q.shape
    o = torch.full((total_q, Hq, d), SENT_O, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((Hq, total_q), SENT_L, device="cuda")
    lq = (cq[1:] - cq[:-1]).tolist()
    lk = (ck[1:] - ck[:-1]).tolist()
    ea.attn_fwd_varlen(qg, kg, vg, cqg, ckg, max_q if max_q is not None else max(lq),
                       max_k if max_k is not None else max(max(lk), 1), o=o, lse=lse,
                       causal=causal, window_left=wl)
    assert ea.attn_device_status() == expect_status
    return o, lse


def check(lens_q, lens_k, Hq, Hkv, d, causal, wl, q_offset=0, tail=0):
    q, k, v, cq, ck = ai.make_varlen(lens_q, lens_k, Hq, Hkv, d, q_offset=q_offset, tail=tail)
    o, lse = run_varlen(q, k, v, cq, ck, causal, wl)
    O, L = oracle.oracle_attention_varlen(q, k, v, cq, ck, causal=causal, window_left=wl)
    rows = slice(int(cq[0]), int(cq[-1]))
    assert_close(o[rows], O[rows], lse[:, rows], L[:, rows], what=(lens_q, lens_k, causal, wl))
    # rows that belong to no sequence are left untouched
    outside = torch.ones(q.shape[0], dtype=torch.bool)
    outside[rows] = False
    assert (o[outside.cuda()].float() == SENT_O).all()
    assert (lse[:, outside.cuda()] == SENT_L).all()


MIX = [1, 127, 128, 129, 300, 1000, 2, 513]


def test_length_mix_causal_mha():
    check(MIX, MIX, 4, 4, 128, True, -1)


def test_length_mix_window_gqa():
    check(MIX, MIX, 8, 2, 128, False, 100)


def test_query_tails_of_longer_key_sets():
    check([50, 128, 1, 200, 7], [300, 128, 500, 200, 7], 4, 2, 128, True, -1)


def test_odd_group_d64_window_causal():
    check([33, 400, 129, 64], [33, 400, 129, 64], 6, 2, 64, True, 50)


def test_offsets_and_untouched_rows():
    check([100, 1, 260], [100, 1, 260], 4, 4, 128, True, -1, q_offset=3, tail=5)


def test_sequence_without_keys():
    q, k, v, cq, ck = ai.make_varlen([40, 30], [40, 0], 4, 4, 128)
    o, lse = run_varlen(q, k, v, cq, ck, False, -1)
    assert (o[40:70].float() == 0).all() and torch.isneginf(lse[:, 40:70]).all()


def test_bitwise_equal_to_one_call_per_sequence():
    import exact_softmax_attention_03_b200 as ea
    lens = [1, 130, 257, 640]
    Hq, Hkv, d = 8, 2, 128
    q, k, v, cq, ck = ai.make_varlen(lens, lens, Hq, Hkv, d)
    o, lse = run_varlen(q, k, v, cq, ck, True, 200)
    for b, n in enumerate(lens):
        q0, k0 = int(cq[b]), int(ck[b])
        qb = q[q0:q0 + n][None].contiguous().cuda()
        kb = k[k0:k0 + n][None].contiguous().cuda()
        vb = v[k0:k0 + n][None].contiguous().cuda()
        lb = torch.empty(1, Hq, n, device="cuda")
        ob, _ = ea.attn_fwd(qb, kb, vb, lse=lb, causal=True, window_left=200)
        torch.cuda.synchronize()
        assert torch.equal(ob[0], o[q0:q0 + n]), b
        assert torch.equal(lb[0], lse[:, q0:q0 + n]), b


def test_inconsistent_offsets_are_skipped_and_reported():
    from exact_softmax_attention_03_b200 import _lib
    lens = [100, 300, 50]
    q, k, v, cq, ck = ai.make_varlen(lens, lens, 4, 4, 128, tail=8)
    # sequence 1 claims more rows than max_seqlen_q allows; the others are fine
    o, lse = run_varlen(q, k, v, cq, ck, True, -1, max_q=200, max_k=300,
                        expect_status=_lib.ATTN_ERR_INVALID_ARG)
    O, L = oracle.oracle_attention_varlen(q, k, v, cq, ck, causal=True)
    for b in (0, 2):
        r = slice(int(cq[b]), int(cq[b + 1]))
        assert_close(o[r], O[r], lse[:, r], L[:, r], what=b)
    r = slice(int(cq[1]), int(cq[2]))
    assert (o[r].float() == SENT_O).all() and (lse[:, r] == SENT_L).all()
    # offsets beyond the packed tensors
    bad = cq.clone()
    bad[2] = q.shape[0] + 1000
    o2, _ = run_varlen(q, k, v, bad, ck, True, -1, max_q=q.shape[0], max_k=300,
                       expect_status=_lib.ATTN_ERR_INVALID_ARG)
    r0 = slice(int(cq[0]), int(cq[1]))
    assert_close(o2[r0], O[r0], what="sequence 0 beside bad offsets")


def test_bench_mix_sampled():
    lens = ai.varlen_lengths(16, 256, 4096)
    Hq, d = 32, 128
    q, k, v, cq, ck = ai.make_varlen(lens, lens, Hq, Hq, d)
    o, lse = run_varlen(q, k, v, cq, ck, True, -1)
    for b in (0, 7, 15):
        q0, n = int(cq[b]), lens[b]
        rows = sorted({0, n - 1, n // 2, n // 3})
        for h in (0, Hq - 1):
            Ob, Lb = oracle.oracle_attention_rows(q[q0:q0 + n][None], k[q0:q0 + n][None],
                                                  v[q0:q0 + n][None], 0, h, rows, causal=True)
            assert_close(o[[q0 + r for r in rows], h], Ob, lse[h, [q0 + r for r in rows]], Lb,
                         what=(b, h))
