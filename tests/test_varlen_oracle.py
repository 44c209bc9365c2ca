"""Pins of the packed variable-length oracle (CPU).

With Q = 0 every allowed score is 0, so each row's softmax is uniform over its
allowed keys: O is the mean of those V rows and LSE = ln(count). The expected
values below are computed from the sequence offsets and the mask rule
directly, so a wrong offset, a key taken from the neighbouring sequence or a
misaligned per-sequence mask changes them.
"""

import math

import numpy as np
import pytest
import torch

import attn_inputs as ai
import oracle

CASES = [
    # (lens_q, lens_k, causal, window_left)
    ([3, 5, 1], [3, 5, 1], True, -1),
    ([3, 5, 1], [3, 5, 1], False, -1),
    ([2, 4], [6, 4], True, -1),            # query tail of a longer key set (bottom-right)
    ([4, 6], [4, 6], True, 1),
    ([5, 2], [5, 3], False, 2),
]


@pytest.mark.parametrize("lens_q,lens_k,causal,wl", CASES)
def test_zero_query_gives_mean_of_allowed_values(lens_q, lens_k, causal, wl):
    Hq, Hkv, d = 2, 1, 3
    q, k, v, cq, ck = ai.make_varlen(lens_q, lens_k, Hq, Hkv, d, q_offset=2, tail=1)
    q = torch.zeros_like(q)
    O, L = oracle.oracle_attention_varlen(q, k, v, cq, ck, causal=causal, window_left=wl)
    vv = v.double().numpy()
    for b in range(len(lens_q)):
        nq, nk = lens_q[b], lens_k[b]
        for i in range(nq):
            qpos = i + nk - nq
            keys = [j for j in range(nk)
                    if (not causal or j <= qpos) and (wl < 0 or j >= qpos - wl)]
            row = int(cq[b]) + i
            for h in range(Hq):
                if not keys:
                    assert np.all(O[row, h] == 0) and L[h, row] == -np.inf
                    continue
                mean = vv[[int(ck[b]) + j for j in keys], 0].mean(axis=0)
                assert np.allclose(O[row, h], mean, rtol=0, atol=1e-12)
                assert math.isclose(L[h, row], math.log(len(keys)), abs_tol=1e-12)
    # rows outside every sequence are not computed
    assert np.isnan(O[:2]).all() and np.isnan(O[-1]).all()


def test_other_sequences_do_not_leak():
    q, k, v, cq, ck = ai.make_varlen([7, 9, 4], [7, 9, 4], 4, 2, 16)
    O1, L1 = oracle.oracle_attention_varlen(q, k, v, cq, ck, causal=True)
    k2, v2 = k.clone(), v.clone()
    k2[int(ck[1]):int(ck[2])] = 3.0            # change sequence 1's keys and values only
    v2[int(ck[1]):int(ck[2])] = -2.0
    O2, L2 = oracle.oracle_attention_varlen(q, k2, v2, cq, ck, causal=True)
    for b in (0, 2):
        r = slice(int(cq[b]), int(cq[b + 1]))
        assert np.array_equal(O1[r], O2[r]) and np.array_equal(L1[:, r], L2[:, r])
    r = slice(int(cq[1]), int(cq[2]))
    assert not np.array_equal(O1[r], O2[r])


def test_empty_key_set_gives_zero_and_minus_inf():
    q, k, v, cq, ck = ai.make_varlen([3, 2], [4, 0], 2, 2, 8)
    O, L = oracle.oracle_attention_varlen(q, k, v, cq, ck, causal=False)
    assert np.all(O[3:5] == 0) and np.all(np.isneginf(L[:, 3:5]))


def test_lengths_generator_is_seeded_and_bounded():
    a = ai.varlen_lengths(50, 128, 4096)
    assert a == ai.varlen_lengths(50, 128, 4096)
    assert min(a) >= 128 and max(a) <= 4096 and len(set(a)) > 10
