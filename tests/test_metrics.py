"""Pins for the work / traffic counts the bench divides by.

The pages print closed-form tables (cache sizes, score-product FLOPs, flash HBM
traffic); the mask-adjusted pair counts are checked against the oracle's mask
by brute force and against closed forms.
"""

import numpy as np
import pytest

import oracle
from exact_softmax_attention_03_b200 import metrics


def test_kv_cache_sizes_match_pages(golden):
    for src, L, H, dh, N, s, B, val, unit in golden("kv_cache_sizes.txt"):
        got = metrics.kv_cache_bytes(int(L), int(H), int(dh), int(N), int(s), int(B))
        got = got / 2**30 if unit == "GiB" else got / 1e9
        digits = len(val.split(".")[1])
        assert round(got, digits) == float(val), (src, H, got, val)


def test_score_flops_table_matches_page(golden):
    for n, t in golden("score_flops_table.txt"):
        got = metrics.score_flops_one_product(int(n), 4096, 32, 32) / 1e12
        assert round(got, 3) == float(t)


def test_flash_traffic_table_matches_page(golden):
    # Q, K, V read once + O written once, all heads and layers (no LSE, as printed)
    for n, gb in golden("flash_traffic_table.txt"):
        n = int(n)
        one_layer = metrics.attn_fwd_bytes(1, 32, 32, n, n, 128, out_bytes=2, with_lse=False)
        assert round(one_layer * 32 / 1e9, 2) == float(gb)


@pytest.mark.parametrize("Nq,Nk,causal,wl", [(8, 8, True, 2), (37, 37, True, -1),
                                             (20, 45, True, 5), (45, 20, True, -1),
                                             (30, 30, False, 4), (17, 33, False, -1),
                                             (64, 64, True, 0), (5, 5, True, 100)])
def test_allowed_pairs_equals_oracle_mask_count(Nq, Nk, causal, wl):
    assert metrics.allowed_pairs(Nq, Nk, causal, wl) == int(oracle.allowed_mask(Nq, Nk, causal, wl).sum())
    assert (metrics.allowed_pairs_per_row(Nq, Nk, causal, wl)
            == oracle.allowed_mask(Nq, Nk, causal, wl).sum(axis=1)).all()


def test_pair_counts_closed_forms():
    # causal: N (N + 1) / 2 ; window w (= window_left + 1 keys): w N - w (w - 1) / 2
    for N in (2048, 8192):
        assert metrics.allowed_pairs(N, N, True, -1) == N * (N + 1) // 2
    N, wl = 32768, 4096
    w = wl + 1
    assert metrics.allowed_pairs(N, N, True, wl) == w * N - w * (w - 1) // 2 == 125_859_840
    assert metrics.allowed_pairs(128, 128, False, -1) == 128 * 128


def test_executed_tiles_counts():
    # one 128-row block per 128 keys up to and including the diagonal
    assert metrics.executed_tiles(2048, 2048, True, -1) == 16 * 17 // 2 == 136
    assert metrics.executed_tiles(8192, 8192, True, -1) == 64 * 65 // 2
    assert metrics.executed_tiles(128, 128, False, -1) == 1
    # sliding window 4096 at 32K: query block i (rows 128i..128i+127) needs key
    # blocks i-32 .. i, clipped at 0: sum(i + 1 for i < 32) + 224 * 33
    t = metrics.executed_tiles(32768, 32768, True, 4096)
    assert t == sum(i + 1 for i in range(32)) + 224 * 33 == 7920


def test_decode_bytes():
    # 64 sequences x 8192 keys x 8 kv heads x 128 x 2 bytes x (K and V)
    assert metrics.decode_kv_bytes([8192] * 64, 8, 128) == 2 * 64 * 8192 * 8 * 128 * 2
    assert metrics.decode_kv_bytes([10, 3], 1, 64, window_left=4) == 2 * (5 + 3) * 64 * 2
    assert np.isclose(metrics.decode_kv_bytes([8192] * 64, 8, 128) / 1e9, 2.147, atol=5e-4)
