"""The FMA-pipe exponential of the prefill kernel, emulated bit for bit in
float32 on the CPU: range reduction with the 1.5 * 2^23 rounding constant, the
cubic, and the exponent-field add. Checked against the error bound of the fit
and against exact 2^x, and its constants against a fresh fit.
"""

import os
import re

import numpy as np

from exact_softmax_attention_03_b200 import fit_exp2_poly

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "exact_softmax_attention_03_b200", "csrc", "sm100_ptx.cuh")


def kernel_coefficients():
    text = open(SRC).read()
    body = text[text.index("uint64_t exp2_poly_f2"):]
    body = body[:body.index("\n}\n")]
    lits = re.findall(r"(0x1\.[0-9a-f]+p-?\d+)f", body)
    # each literal appears twice (both halves of a pair): c3, c2, c1, c0 in Horner order
    uniq = list(dict.fromkeys(lits))
    return [float.fromhex(x) for x in uniq][::-1]       # -> c0, c1, c2, c3


def emulate(x):
    """float32 emulation of exp2_poly_f2 on an array."""
    c0, c1, c2, c3 = [np.float32(c) for c in kernel_coefficients()]
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    f = (x - r).astype(np.float32)
    q = (f * c3 + c2).astype(np.float32)       # fma vs mul+add differ by < 1 ulp here
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    with np.errstate(over="ignore"):          # the exponent add wraps by design
        e = (q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return e.view(np.float32)


def test_constants_match_a_fresh_fit():
    coef, err = fit_exp2_poly.fit()
    assert err < 8e-5
    assert np.allclose(kernel_coefficients(), coef, rtol=0, atol=2e-7)


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    got = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1)
    assert rel.max() < 1.2e-4          # fit bound 7.5e-5 plus float32 rounding
    assert (got > 0).all()


def test_integer_arguments_and_clamp():
    for j in range(-125, 9):
        assert abs(float(emulate(np.float32(j))) / 2.0 ** j - 1) < 1e-4
    # far below the clamp the result is a tiny positive normal, never a wrapped exponent
    v = float(emulate(np.float32(-1000.0)))
    assert 0 < v < 1e-37
