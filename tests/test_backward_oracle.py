"""Pins of the backward oracle (CPU).

The gradient formulas are checked against central finite differences of the
forward oracle (which does not use them), and against two exact identities of
softmax attention: the key gradients of a head sum to zero (each row of dS
sums to zero) and the value gradients sum to the sum of the output gradients
(each row of P sums to one).
"""

import numpy as np
import pytest

import oracle


def _fd_grad(f, x, eps=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + eps
        fp = f()
        x[i] = old - eps
        fm = f()
        x[i] = old
        g[i] = (fp - fm) / (2 * eps)
    return g


CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal, window_left
    (1, 2, 1, 4, 5, 3, True, -1),
    (1, 1, 1, 5, 5, 2, False, 1),
    (2, 2, 2, 3, 3, 2, True, 0),
    (1, 2, 1, 6, 4, 2, True, 1),          # leading rows with no key
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal,wl", CASES)
def test_gradients_match_finite_differences(B, Hq, Hkv, Nq, Nk, d, causal, wl):
    rng = np.random.default_rng(5)
    q = rng.standard_normal((B, Nq, Hq, d))
    k = rng.standard_normal((B, Nk, Hkv, d))
    v = rng.standard_normal((B, Nk, Hkv, d))
    w = rng.standard_normal((B, Nq, Hq, d))          # loss = sum(w * O): dO = w
    scale = 0.7

    def loss():
        O, _ = oracle.oracle_attention(q, k, v, causal=causal, window_left=wl, scale=scale)
        return float((w * O).sum())

    dQ, dK, dV = oracle.oracle_attention_backward(q, k, v, w, causal=causal, window_left=wl,
                                                  scale=scale)
    for x, g in ((q, dQ), (k, dK), (v, dV)):
        num = _fd_grad(loss, x)
        assert np.allclose(g, num, rtol=1e-6, atol=1e-7), np.abs(g - num).max()


def test_softmax_identities():
    rng = np.random.default_rng(9)
    B, Hq, Hkv, N, d = 2, 4, 2, 37, 8
    q = rng.standard_normal((B, N, Hq, d))
    k = rng.standard_normal((B, N, Hkv, d))
    v = rng.standard_normal((B, N, Hkv, d))
    do = rng.standard_normal((B, N, Hq, d))
    dQ, dK, dV = oracle.oracle_attention_backward(q, k, v, do, causal=True)
    # sum over keys of dK is zero for every (batch, kv head)
    assert np.abs(dK.sum(axis=1)).max() < 1e-10
    # sum over keys of dV equals the sum of dO over the group's rows
    G = Hq // Hkv
    for h in range(Hkv):
        want = do[:, :, h * G:(h + 1) * G].sum(axis=(1, 2))
        assert np.allclose(dV[:, :, h].sum(axis=1), want, atol=1e-10)


def test_masked_rows_give_zero_query_gradient():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 6, 1, 4))
    k = rng.standard_normal((1, 3, 1, 4))
    v = rng.standard_normal((1, 3, 1, 4))
    do = rng.standard_normal((1, 6, 1, 4))
    dQ, _, _ = oracle.oracle_attention_backward(q, k, v, do, causal=True)
    assert np.all(dQ[0, :3] == 0)           # rows 0-2 see no key (bottom-right alignment)


def test_group_slices_equal_the_full_problem():
    # the full-size GPU parity test checks one (batch, K/V head) group at a time
    from parity import backward_of_group
    rng = np.random.default_rng(5)
    B, Hq, Hkv, Nq, Nk, d = 2, 6, 2, 9, 13, 4
    q = rng.standard_normal((B, Nq, Hq, d))
    k = rng.standard_normal((B, Nk, Hkv, d))
    v = rng.standard_normal((B, Nk, Hkv, d))
    do = rng.standard_normal((B, Nq, Hq, d))
    dQ, dK, dV = oracle.oracle_attention_backward(q, k, v, do, causal=True, window_left=5)
    G = Hq // Hkv
    for b in range(B):
        for hk in range(Hkv):
            gq, gk, gv = backward_of_group(q, k, v, do, b, hk, True, 5)
            assert np.allclose(gq, dQ[b, :, hk * G:(hk + 1) * G], rtol=0, atol=1e-12)
            assert np.allclose(gk, dK[b, :, hk], rtol=0, atol=1e-12)
            assert np.allclose(gv, dV[b, :, hk], rtol=0, atol=1e-12)
