"""Pins of the paged-cache oracle (CPU).

The page lookup ("Inference Engineering", section 2.5 "Optimizing Attention",
PagedAttention paragraph) is checked on a hand-built pool, by a round trip
through the seeded page scatter, and by the fact that paging only moves keys:
decode over the pages equals decode over the contiguous cache exactly.
"""

import numpy as np
import pytest
import torch

import attn_inputs as ai
import oracle


def test_page_lookup_hand_example():
    # 3 pages of 2 keys, Hkv = 1, d = 1; page p holds values 10p and 10p + 1
    pages = np.array([[[[0.0]], [[1.0]]], [[[10.0]], [[11.0]]], [[[20.0]], [[21.0]]]])
    bt = np.array([[2, 0, 1], [1, 1, 0]])
    out = oracle.paged_to_contiguous(pages, bt, seqlens=[6, 3])
    assert out[0, :, 0, 0].tolist() == [20, 21, 0, 1, 10, 11]
    # keys at or past seqlen stay zero: sequence 1 has 3 keys
    assert out[1, :, 0, 0].tolist() == [10, 11, 10, 0, 0, 0]


def test_unread_table_entries_are_not_used():
    pages = np.arange(8, dtype=np.float64).reshape(4, 2, 1, 1)
    bt = np.array([[3, 10**6]])                    # second entry is never needed
    out = oracle.paged_to_contiguous(pages, bt, seqlens=[2])
    assert out[0, :2, 0, 0].tolist() == [6, 7]


@pytest.mark.parametrize("page_size", [16, 64, 128])
def test_scatter_gather_round_trip(page_size):
    q, kc, vc = ai.make_decode(3, 4, 2, 256, 64)
    kp, vp, bt = ai.make_paged(kc, vc, page_size)
    assert kp.shape[0] == 3 * 256 // page_size + 3
    assert len(set(bt.reshape(-1).tolist())) == bt.numel()        # no page used twice
    back = oracle.paged_to_contiguous(kp, bt)
    assert np.array_equal(back, kc.double().numpy())
    back_v = oracle.paged_to_contiguous(vp, bt)
    assert np.array_equal(back_v, vc.double().numpy())


def test_paged_decode_equals_contiguous_decode_exactly():
    q, kc, vc = ai.make_decode(4, 8, 2, 192, 64)
    sl = ai.ragged_seqlens(4, 192)
    kp, vp, bt = ai.make_paged(kc, vc, 32)
    O1, L1 = oracle.oracle_decode(q, kc, vc, sl, window_left=50)
    O2, L2 = oracle.oracle_decode_paged(q, kp, vp, bt, sl, window_left=50)
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)


def test_noise_in_unreferenced_pages_does_not_leak():
    q, kc, vc = ai.make_decode(2, 4, 1, 64, 64)
    kp, vp, bt = ai.make_paged(kc, vc, 16, extra_pages=2)
    used = set(bt.reshape(-1).tolist())
    free = [p for p in range(kp.shape[0]) if p not in used]
    kp[free] = torch.nan
    vp[free] = torch.nan
    O, L = oracle.oracle_decode_paged(q, kp, vp, bt)
    assert np.isfinite(O).all() and np.isfinite(L).all()
