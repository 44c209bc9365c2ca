"""Randomised cross-checks of the fp64 oracle on tiny shapes (CPU).

The fixed-shape pins live in test_oracle_pins.py. Here hypothesis draws
batches, GQA groups, unequal query/key lengths (rows with no allowed key
included), windows down to 0 and random inputs. The NumPy oracle must agree
with the independent formulations the oracle module carries:

- the pure-Python loops;
- the key-chunk merge (section 3.5 rule), with random chunk sizes;
- decode as the last causal row;
- the merge rule over a random split of the keys;
- the backward identities (a head's key gradients sum to zero; its value
  gradients sum to the output gradients of the rows that see a key).
"""

import math

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from oracle import attention as oa

SETTINGS = settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.too_slow])


@st.composite
def problems(draw, max_n=9):
    B = draw(st.integers(1, 2))
    Hkv = draw(st.integers(1, 3))
    G = draw(st.integers(1, 3))
    Nq = draw(st.integers(1, max_n))
    Nk = draw(st.integers(1, max_n))
    d = draw(st.integers(1, 5))
    causal = draw(st.booleans())
    wl = draw(st.one_of(st.just(-1), st.integers(0, max_n + 1)))
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Nq, Hkv * G, d))
    k = rng.standard_normal((B, Nk, Hkv, d))
    v = rng.standard_normal((B, Nk, Hkv, d))
    return q, k, v, causal, wl


def _same(a, b, tol=1e-12):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape
    ninf_a, ninf_b = np.isneginf(a), np.isneginf(b)
    assert (ninf_a == ninf_b).all()
    fin = ~ninf_a
    assert np.allclose(a[fin], b[fin], rtol=0, atol=tol), np.abs(a[fin] - b[fin]).max()


@SETTINGS
@given(problems())
def test_numpy_oracle_equals_pure_python_loops(p):
    q, k, v, causal, wl = p
    O, L = oracle.oracle_attention(q, k, v, causal=causal, window_left=wl)
    Ob, Lb = oa.brute_force_attention(q.tolist(), k.tolist(), v.tolist(), causal=causal,
                                      window_left=wl)
    _same(O, Ob)
    _same(L, Lb)


@SETTINGS
@given(problems(), st.integers(1, 5))
def test_key_chunk_merge_equals_materialised(p, ck):
    q, k, v, causal, wl = p
    O, L = oracle.oracle_attention(q, k, v, causal=causal, window_left=wl)
    Ot, Lt = oa.key_chunk_attention(q, k, v, causal=causal, window_left=wl, chunk=ck)
    _same(O, Ot)
    _same(L, Lt)


@SETTINGS
@given(problems())
def test_rows_without_keys_are_zero_and_rows_with_keys_normalise(p):
    q, k, v, causal, wl = p
    O, L = oracle.oracle_attention(q, k, v, causal=causal, window_left=wl)
    empty = np.isneginf(L)                                   # [B, Hq, Nq]
    assert (O.transpose(0, 2, 1, 3)[empty] == 0).all()
    # constant V returns the constant on every row that sees a key
    Oc, _ = oracle.oracle_attention(q, k, np.full_like(v, 0.375), causal=causal, window_left=wl)
    seen = ~empty
    assert np.allclose(Oc.transpose(0, 2, 1, 3)[seen], 0.375, rtol=0, atol=1e-12)


@SETTINGS
@given(problems())
def test_decode_is_the_last_causal_row(p):
    q, k, v, _, wl = p
    O, L = oracle.oracle_attention(q, k, v, causal=True, window_left=wl)
    Od, Ld = oracle.oracle_decode(q[:, -1], k, v, window_left=wl)
    _same(Od, O[:, -1])
    _same(Ld, L[:, :, -1])


@SETTINGS
@given(problems(), st.data())
def test_merge_of_a_key_split_equals_the_whole(p, data):
    q, k, v, _, _ = p
    Nk = k.shape[1]
    if Nk < 2:
        return
    s = data.draw(st.integers(1, Nk - 1))
    O, L = oracle.oracle_attention(q, k, v)
    O1, L1 = oracle.oracle_attention(q, k[:, :s], v[:, :s])
    O2, L2 = oracle.oracle_attention(q, k[:, s:], v[:, s:])
    B, Nq, Hq, _ = q.shape
    for b in range(B):
        for h in range(Hq):
            for i in range(Nq):
                # a part's state: m = its LSE, l = 1, acc = its normalised output
                Om, Lm = oa.merge_partials([(L1[b, h, i], 1.0, O1[b, i, h]),
                                            (L2[b, h, i], 1.0, O2[b, i, h])])
                assert np.allclose(Om, O[b, i, h], rtol=0, atol=1e-12)
                assert math.isclose(Lm, L[b, h, i], rel_tol=0, abs_tol=1e-12)


@SETTINGS
@given(problems())
def test_backward_identities(p):
    q, k, v, causal, wl = p
    rng = np.random.default_rng(int(abs(q).sum() * 1e6) % (2**32))
    do = rng.standard_normal(q.shape)
    dQ, dK, dV = oracle.oracle_attention_backward(q, k, v, do, causal=causal, window_left=wl)
    _, L = oracle.oracle_attention(q, k, v, causal=causal, window_left=wl)
    G = q.shape[2] // k.shape[2]
    assert np.abs(dK.sum(axis=1)).max() < 1e-10
    seen = ~np.isneginf(L)                                   # [B, Hq, Nq]
    for h in range(k.shape[2]):
        want = np.zeros((q.shape[0], q.shape[3]))
        for g in range(G):
            hq = h * G + g
            want += (do[:, :, hq] * seen[:, hq, :, None]).sum(axis=1)
        assert np.allclose(dV[:, :, h].sum(axis=1), want, rtol=0, atol=1e-10)
    # rows with no allowed key get no query gradient
    assert (dQ.transpose(0, 2, 1, 3)[~seen] == 0).all()
