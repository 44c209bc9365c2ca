"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics.

Each check compares the oracle with something other than itself: values the
pages print (fixtures under tests/golden/), exact closed forms for scores that
are logs of integers, invariants (rows of P sum to 1, constant V, GQA equals
MHA on repeated K/V, decode equals the last prefill row, window >= N equals
causal), an independent pure-Python loop, a key-chunk merge of separately normalised chunks,
and library routines (torch's float64 SDPA, scipy's logsumexp).

The last test plants plausible mistakes in copies of the oracle (a transposed
operand, a dropped scale, a wrong head map, an off-by-one window, a wrong LSE
base) and shows that at least one pin fails for each.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oa

LN = math.log


# ---------------------------------------------------------------------------
# Pins written as functions of an attention routine, so the planted-mistake
# test can run them against mutated oracles as well.
# ---------------------------------------------------------------------------

def _hand_3x3_inputs():
    # Scores S[i, j] = K[j, i] with Q = I and scale 1, chosen as logs of
    # integers so that P has exact rational entries. S is not symmetric, so a
    # transposed product changes the result.
    W = np.array([[1, 2, 3],
                  [4, 1, 3],
                  [2, 2, 4]], dtype=np.float64)
    S = np.log(W)
    q = np.eye(3)[None, :, None, :]              # [1, 3, 1, 3]
    k = S.T[None, :, None, :]                    # K[j, c] = S[c, j]
    v = np.eye(3)[None, :, None, :]              # one-hot values: O = P
    return q, k, v


HAND_3X3 = {
    # (causal, window_left): (expected P rows, expected LSE), by hand
    (False, -1): ([[1 / 6, 2 / 6, 3 / 6], [4 / 8, 1 / 8, 3 / 8], [2 / 8, 2 / 8, 4 / 8]],
                  [LN(6), LN(8), LN(8)]),
    (True, -1): ([[1, 0, 0], [4 / 5, 1 / 5, 0], [2 / 8, 2 / 8, 4 / 8]],
                 [0.0, LN(5), LN(8)]),
    (True, 1): ([[1, 0, 0], [4 / 5, 1 / 5, 0], [0, 2 / 6, 4 / 6]],
                [0.0, LN(5), LN(6)]),
    # window without causal limits the left side only: row i sees keys j >= i
    (False, 0): ([[1 / 6, 2 / 6, 3 / 6], [0, 1 / 4, 3 / 4], [0, 0, 1]],
                 [LN(6), LN(4), LN(4)]),
}


def pin_hand_3x3(attn):
    q, k, v = _hand_3x3_inputs()
    for (causal, wl), (P, lse) in HAND_3X3.items():
        O, L = attn(q, k, v, causal=causal, window_left=wl, scale=1.0)
        if not np.allclose(O[0, :, 0, :], np.array(P), atol=1e-13, rtol=0):
            return False
        if not np.allclose(L[0, 0], np.array(lse), atol=1e-13, rtol=0):
            return False
    return True


def pin_hand_2x2_scaled(attn):
    # d = 2, scale = 0.5: q0 = [2 ln2, 0], q1 = [0, 2]; k0 = [0, 1], k1 = [1, 0].
    # Scaled scores: row 0 = [0, ln 2] -> P = [1/3, 2/3], LSE = ln 3;
    #                row 1 = [1, 0]    -> P = [e/(e+1), 1/(e+1)], LSE = ln(e+1).
    q = np.array([[2 * LN(2), 0.0], [0.0, 2.0]])[None, :, None, :]
    k = np.array([[0.0, 1.0], [1.0, 0.0]])[None, :, None, :]
    v = np.array([[1.0, 0.0], [0.0, 1.0]])[None, :, None, :]
    O, L = attn(q, k, v, causal=False, window_left=-1, scale=0.5)
    e = math.e
    ok = np.allclose(O[0, :, 0, :], [[1 / 3, 2 / 3], [e / (e + 1), 1 / (e + 1)]], atol=1e-13)
    ok &= np.allclose(L[0, 0], [LN(3), LN(e + 1)], atol=1e-13)
    return bool(ok)


def pin_page_worked_example(attn, golden):
    rows = {r[0]: r[1:] for r in golden("online_softmax_scores_1_3.txt")}
    s = [float(x) for x in rows["scores"]]
    q = np.array([[1.0, 0.0]])[None, :, None, :]
    k = np.array([[s[0], 0.0], [s[1], 0.0]])[None, :, None, :]
    v = np.eye(2)[None, :, None, :]
    O, L = attn(q, k, v, causal=False, window_left=-1, scale=1.0)
    probs = [float(x) for x in rows["prob"]]
    den = float(rows["denominator"][0])
    m = float(rows["final_max"][0])
    ok = np.allclose(O[0, 0, 0], probs, atol=5e-4)
    # LSE = m + ln(denominator); the page prints the denominator to 4 decimals.
    ok &= abs(L[0, 0, 0] - (m + math.log(den))) < 1e-4
    return bool(ok)


def pin_gqa_is_repeated_mha(attn, rng):
    B, N, Hq, Hkv, d = 2, 9, 6, 2, 4
    q = rng.standard_normal((B, N, Hq, d))
    k = rng.standard_normal((B, N, Hkv, d))
    v = rng.standard_normal((B, N, Hkv, d))
    Og, Lg = attn(q, k, v, causal=True, window_left=-1, scale=0.7)
    # "Chapter 3 ...", section 3.3: repeat each K/V group H // G times.
    kr = np.repeat(k, Hq // Hkv, axis=2)
    vr = np.repeat(v, Hq // Hkv, axis=2)
    Om, Lm = attn(q, kr, vr, causal=True, window_left=-1, scale=0.7)
    return bool(np.allclose(Og, Om, atol=1e-13) and np.allclose(Lg, Lm, atol=1e-13))


def pin_window_pattern(mask_fn, golden):
    rows = golden("window_mask_n8_W3.txt")
    hdr = {r[0]: int(r[1]) for r in rows if len(r) == 2}
    pattern = np.array([[c == "X" for c in r] for r in rows if len(r) == hdr["n"]])
    m = mask_fn(hdr["n"], hdr["n"], True, hdr["W"] - 1)
    return (bool((m == pattern).all()) and int(m.sum()) == hdr["allowed"]
            and int(mask_fn(hdr["n"], hdr["n"], True, -1).sum()) == hdr["causal_allowed"])


# ---------------------------------------------------------------------------
# Tests
# ---------------------------------------------------------------------------

def test_online_softmax_worked_example(golden):
    rows = {r[0]: r[1:] for r in golden("online_softmax_scores_1_3.txt")}
    probs, m, den = oracle.online_softmax([float(x) for x in rows["scores"]])
    assert m == float(rows["final_max"][0])
    assert abs(den - float(rows["denominator"][0])) < 5e-5
    assert [round(p, 3) for p in probs] == [float(x) for x in rows["prob"]]
    # exact: e^-2 / (1 + e^-2)
    assert abs(probs[0] - math.exp(-2) / (1 + math.exp(-2))) < 1e-15


def test_oracle_reproduces_worked_example(golden):
    assert pin_page_worked_example(oracle.oracle_attention, golden)


def test_window_mask_matches_page_diagram(golden):
    assert pin_window_pattern(oracle.allowed_mask, golden)


def test_causal_bottom_right_alignment_by_hand():
    # Nq = 2 queries at the end of Nk = 4 keys: row 0 sits at key 2, row 1 at key 3.
    m = oracle.allowed_mask(2, 4, True, -1)
    assert m.tolist() == [[True, True, True, False], [True, True, True, True]]
    m = oracle.allowed_mask(2, 4, True, 1)
    assert m.tolist() == [[False, True, True, False], [False, False, True, True]]
    # window without causal: left limit only
    m = oracle.allowed_mask(2, 4, False, 0)
    assert m.tolist() == [[False, False, True, True], [False, False, False, True]]


def test_hand_3x3_closed_forms():
    assert pin_hand_3x3(oracle.oracle_attention)


def test_hand_2x2_scaled_closed_forms():
    assert pin_hand_2x2_scaled(oracle.oracle_attention)


def test_rows_of_p_sum_to_one():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((1, 37, 2, 8))
    k = rng.standard_normal((1, 41, 1, 8))
    for causal, wl in [(False, -1), (True, -1), (True, 5), (False, 3)]:
        P = oracle.oracle_probabilities(q, k, causal=causal, window_left=wl, hq=1)
        assert np.allclose(P.sum(axis=1), 1.0, atol=1e-12, rtol=0)
        assert (P[~oracle.allowed_mask(37, 41, causal, wl)] == 0).all()


def test_constant_v_returns_constant():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((2, 19, 4, 16))
    k = rng.standard_normal((2, 23, 2, 16))
    v = np.full((2, 23, 2, 16), -1.75)
    O, _ = oracle.oracle_attention(q, k, v, causal=True, window_left=4)
    assert np.allclose(O, -1.75, atol=1e-13, rtol=0)


def test_one_hot_v_column_returns_p_column():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 11, 1, 4))
    k = rng.standard_normal((1, 11, 1, 4))
    v = np.zeros((1, 11, 1, 4))
    v[0, 7, 0, 2] = 1.0                                # key 7 carries a 1 in column 2
    O, _ = oracle.oracle_attention(q, k, v, causal=False)
    P = oracle.oracle_probabilities(q, k, causal=False)
    assert np.allclose(O[0, :, 0, 2], P[:, 7], atol=1e-15)
    assert np.allclose(np.delete(O[0, :, 0, :], 2, axis=1), 0.0)


def test_window_covering_everything_equals_causal():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 30, 2, 8))
    k = rng.standard_normal((1, 30, 2, 8))
    v = rng.standard_normal((1, 30, 2, 8))
    Oc, Lc = oracle.oracle_attention(q, k, v, causal=True)
    for wl in (29, 30, 1000):
        Ow, Lw = oracle.oracle_attention(q, k, v, causal=True, window_left=wl)
        assert np.array_equal(Oc, Ow) and np.array_equal(Lc, Lw)
    Ow, _ = oracle.oracle_attention(q, k, v, causal=True, window_left=28)
    assert not np.allclose(Oc, Ow)


def test_gqa_equals_mha_with_repeated_kv():
    assert pin_gqa_is_repeated_mha(oracle.oracle_attention, np.random.default_rng(4))


def test_decode_equals_last_row_of_causal_prefill():
    rng = np.random.default_rng(5)
    B, L, Hq, Hkv, d = 3, 20, 4, 2, 8
    kc = rng.standard_normal((B, L, Hkv, d))
    vc = rng.standard_normal((B, L, Hkv, d))
    qfull = rng.standard_normal((B, L, Hq, d))
    seqlens = [20, 7, 1]
    for wl in (-1, 3):
        Od, Ld = oracle.oracle_decode(qfull[:, -1], kc, vc, seqlens, window_left=wl)
        for b, s in enumerate(seqlens):
            q_b = qfull[b:b + 1, :s].copy()
            q_b[0, s - 1] = qfull[b, -1]
            Op, Lp = oracle.oracle_attention(q_b, kc[b:b + 1, :s], vc[b:b + 1, :s],
                                             causal=True, window_left=wl)
            assert np.allclose(Od[b], Op[0, s - 1], atol=1e-13)
            assert np.allclose(Ld[b], Lp[0, :, s - 1], atol=1e-13)


def test_key_chunk_merge_equals_materialising_oracle():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((2, 70, 4, 16)) * 3.0
    k = rng.standard_normal((2, 90, 2, 16)) * 3.0
    v = rng.standard_normal((2, 90, 2, 16))
    for causal, wl in [(False, -1), (True, -1), (True, 17), (False, 40)]:
        O1, L1 = oracle.oracle_attention(q, k, v, causal=causal, window_left=wl)
        O2, L2 = oracle.key_chunk_attention(q, k, v, causal=causal, window_left=wl, chunk=32)
        assert np.allclose(O1, O2, atol=1e-12, rtol=0)
        assert np.allclose(L1, L2, atol=1e-12, rtol=0)


@pytest.mark.parametrize("causal,wl,Nq,Nk", [(False, -1, 5, 7), (True, -1, 5, 7),
                                             (True, 2, 6, 6), (False, 1, 4, 6),
                                             (True, -1, 7, 4)])
def test_pure_python_brute_force_matches(causal, wl, Nq, Nk):
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, Nq, 2, 3))
    k = rng.standard_normal((1, Nk, 1, 3))
    v = rng.standard_normal((1, Nk, 1, 3))
    O1, L1 = oracle.oracle_attention(q, k, v, causal=causal, window_left=wl)
    O2, L2 = oracle.brute_force_attention(q.tolist(), k.tolist(), v.tolist(),
                                          causal=causal, window_left=wl)
    assert np.allclose(O1, np.array(O2), atol=1e-13)
    assert np.allclose(L1, np.array(L2), atol=1e-13)


def test_against_torch_float64_sdpa():
    # torch's CPU scaled_dot_product_attention in float64 is an independent
    # implementation of the same definition (mask given explicitly).
    rng = np.random.default_rng(8)
    B, Nq, Nk, Hq, Hkv, d = 2, 33, 47, 4, 2, 16
    q = rng.standard_normal((B, Nq, Hq, d))
    k = rng.standard_normal((B, Nk, Hkv, d))
    v = rng.standard_normal((B, Nk, Hkv, d))
    for causal, wl in [(False, -1), (True, -1), (True, 9), (False, 5)]:
        O, _ = oracle.oracle_attention(q, k, v, causal=causal, window_left=wl, scale=0.3)
        mask = torch.from_numpy(oracle.allowed_mask(Nq, Nk, causal, wl))
        tq = torch.from_numpy(q).transpose(1, 2)
        tk = torch.from_numpy(np.repeat(k, Hq // Hkv, axis=2)).transpose(1, 2)
        tv = torch.from_numpy(np.repeat(v, Hq // Hkv, axis=2)).transpose(1, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(
            tq, tk, tv, attn_mask=mask, scale=0.3).transpose(1, 2).numpy()
        assert np.allclose(O, ref, atol=1e-12, rtol=0)


def test_lse_against_scipy_logsumexp():
    from scipy.special import logsumexp
    rng = np.random.default_rng(9)
    q = rng.standard_normal((1, 12, 1, 8))
    k = rng.standard_normal((1, 15, 1, 8))
    v = rng.standard_normal((1, 15, 1, 8))
    _, L = oracle.oracle_attention(q, k, v, causal=True, window_left=6, scale=0.25)
    mask = oracle.allowed_mask(12, 15, True, 6)
    S = 0.25 * q[0, :, 0] @ k[0, :, 0].T
    ref = [logsumexp(S[i][mask[i]]) for i in range(12)]
    assert np.allclose(L[0, 0], ref, atol=1e-13)


def test_fully_masked_rows_give_zero_and_minus_inf():
    rng = np.random.default_rng(10)
    q = rng.standard_normal((1, 6, 1, 4))
    k = rng.standard_normal((1, 3, 1, 4))
    v = rng.standard_normal((1, 3, 1, 4))
    O, L = oracle.oracle_attention(q, k, v, causal=True)
    # rows 0..2 sit before key 0 (bottom-right alignment): nothing allowed
    assert (O[0, :3] == 0).all() and np.isneginf(L[0, 0, :3]).all()
    assert np.isfinite(L[0, 0, 3:]).all()


def test_merge_of_key_chunks_equals_whole():
    rng = np.random.default_rng(11)
    q = rng.standard_normal((1, 1, 1, 8)) * 2
    k = rng.standard_normal((1, 50, 1, 8)) * 2
    v = rng.standard_normal((1, 50, 1, 8))
    Ofull, Lfull = oracle.oracle_attention(q, k, v)
    parts = []
    for a, b in [(0, 13), (13, 14), (14, 40), (40, 50)]:
        Oc, Lc = oracle.oracle_attention(q, k[:, a:b], v[:, a:b])
        parts.append((Lc[0, 0, 0], 1.0, Oc[0, 0, 0]))   # (m, l, acc) with m = LSE, l = 1
    parts.append((-np.inf, 0.0, np.zeros(8)))             # an empty chunk
    O, L = oracle.merge_partials(parts)
    assert np.allclose(O, Ofull[0, 0, 0], atol=1e-13)
    assert abs(L - Lfull[0, 0, 0]) < 1e-13


def test_rows_helper_matches_full():
    rng = np.random.default_rng(12)
    q = rng.standard_normal((2, 40, 4, 8))
    k = rng.standard_normal((2, 40, 2, 8))
    v = rng.standard_normal((2, 40, 2, 8))
    O, L = oracle.oracle_attention(q, k, v, causal=True, window_left=7)
    rows = [0, 5, 39]
    o, lse = oracle.oracle_attention_rows(q, k, v, 1, 3, rows, causal=True, window_left=7)
    assert np.allclose(o, O[1, rows, 3]) and np.allclose(lse, L[1, 3, rows])


def test_bf16_inputs_are_upcast_exactly():
    t = torch.randn(1, 4, 1, 8).to(torch.bfloat16)
    a = oa._f64(t)
    assert a.dtype == np.float64
    assert np.array_equal(a, t.float().numpy().astype(np.float64))


# ---------------------------------------------------------------------------
# Planted mistakes: each mutated oracle must fail at least one pin.
# ---------------------------------------------------------------------------

def _mutant(kind):
    def head(qh, kh, vh, scale, mask):
        if kind == "transposed" and qh.shape[0] == kh.shape[0]:
            S = scale * (kh @ qh.T)                  # Sᵀ instead of S
        elif kind == "no_scale":
            S = qh @ kh.T
        else:
            S = scale * (qh @ kh.T)
        S = np.where(mask, S, -np.inf)
        m = S.max(axis=1)
        ok = np.isfinite(m)
        ms = np.where(ok, m, 0.0)
        E = np.exp(S - ms[:, None])
        l = E.sum(axis=1)
        P = np.zeros_like(E)
        P[ok] = E[ok] / l[ok, None]
        lse = np.full(m.shape, -np.inf)
        if kind == "log2_lse":
            lse[ok] = m[ok] + np.log2(l[ok])
        else:
            lse[ok] = m[ok] + np.log(l[ok])
        return P @ vh, lse, P

    def mask_fn(Nq, Nk, causal, wl):
        if kind == "window_off_by_one" and wl >= 0:
            wl = wl + 1
        return _orig_mask(Nq, Nk, causal, wl)

    def attn(q, k, v, causal=False, window_left=-1, scale=None):
        q, k, v = oa._f64(q), oa._f64(k), oa._f64(v)
        B, Nq, Hq, d = q.shape
        _, Nk, Hkv, _ = k.shape
        scale = 1 / math.sqrt(d) if scale is None else scale
        mask = mask_fn(Nq, Nk, causal, window_left)
        O = np.zeros((B, Nq, Hq, d))
        L = np.full((B, Hq, Nq), -np.inf)
        for b in range(B):
            for h in range(Hq):
                hk = (h % Hkv) if kind == "head_map_mod" else h // (Hq // Hkv)
                o, lse, _ = head(q[b, :, h], k[b, :, hk], v[b, :, hk], scale, mask)
                O[b, :, h] = o
                L[b, h] = lse
        return O, L

    return attn, mask_fn


_orig_mask = oa.allowed_mask


@pytest.mark.parametrize("kind", ["transposed", "no_scale", "head_map_mod",
                                  "window_off_by_one", "log2_lse"])
def test_planted_mistakes_are_caught(kind, golden):
    attn, mask_fn = _mutant(kind)
    results = [
        pin_hand_3x3(attn),
        pin_hand_2x2_scaled(attn),
        pin_page_worked_example(attn, golden),
        pin_gqa_is_repeated_mha(attn, np.random.default_rng(4)),
        pin_window_pattern(mask_fn, golden),
    ]
    assert not all(results), f"mutant {kind} passed every pin"


def test_unmutated_control_passes_all_pins(golden):
    attn, mask_fn = _mutant("none")
    assert pin_hand_3x3(attn) and pin_hand_2x2_scaled(attn)
    assert pin_page_worked_example(attn, golden)
    assert pin_gqa_is_repeated_mha(attn, np.random.default_rng(4))
    assert pin_window_pattern(mask_fn, golden)


def test_mask_of_selected_rows_is_those_rows_of_the_full_mask():
    rng = np.random.default_rng(11)
    for Nq, Nk, causal, wl in [(37, 37, True, -1), (20, 50, True, 7), (50, 20, True, -1),
                               (30, 30, False, 4), (9, 9, False, -1)]:
        full = oracle.allowed_mask(Nq, Nk, causal, wl)
        rows = sorted(rng.choice(Nq, size=min(Nq, 11), replace=False).tolist())
        assert (oracle.allowed_mask(Nq, Nk, causal, wl, rows=rows) == full[rows]).all()
