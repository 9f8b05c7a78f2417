"""The attention softmax and the LM-head epilogue compute part of their
exponentials with their own 2^x (csrc/dg_attn_tc.cu exp2_poly, degree 3;
csrc/dg_lmhead_tc.cu exp2_poly4, degree 4): a round-to-nearest split
x = j + f and a polynomial for 2^f on [-1/2, 1/2]. Their error bounds, checked
on CPU by evaluating the same steps in float32 with the coefficients read from
the sources: relative error within 1e-4 (attention: far below the 2^-9 half-ulp
of the bf16 probabilities) and within 3e-6 (LM head: the entropy then moves by
less than 7e-5 nats) over the ranges they are used on."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coefficients(fname="dg_attn_tc.cu", func="float exp2_poly("):
    """The polynomial's coefficients, highest degree first, as written in the source."""
    src = open(os.path.join(ROOT, "token_canvas_denoising_b200", "csrc", fname)).read()
    body = src[src.index(func):]
    body = body[:body.index("}")]
    return [np.float32(x) for x in re.findall(r"(-?\d+\.\d+(?:e-?\d+)?)f", body) if abs(float(x)) < 1.5]


def _exp2_poly(x, coef=None):
    """The kernels' steps in float32 / int32 (Horner from the highest degree)."""
    coef = _coefficients()[-4:] if coef is None else coef
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0))).astype(np.float32)
    p = np.float32(coef[0]) * np.ones_like(f)
    for c in coef[1:]:
        p = (p * f + np.float32(c)).astype(np.float32)
    j = t.view(np.int32) - np.int32(0x4B400000)
    return (p.view(np.int32) + (j << 23)).view(np.float32)


def test_coefficients_are_the_fitted_polynomial():
    c = _coefficients()[-4:]
    assert len(c) == 4 and abs(float(c[3]) - 1.0) < 1e-3 and abs(float(c[2]) - np.log(2)) < 1e-3


def test_relative_error_bound_over_the_softmax_range():
    x = np.concatenate([np.linspace(-125, 8, 2_000_001, dtype=np.float32),
                        np.arange(-125, 9, dtype=np.float32) + np.float32(0.5),
                        np.arange(-125, 9, dtype=np.float32)])
    got = _exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.max(np.abs(got / ref - 1))
    assert rel < 1e-4, rel
    assert rel < 2.0 ** -9 / 10


def test_masked_keys_give_a_negligible_weight():
    got = _exp2_poly(np.array([-np.inf, -1000.0], np.float32)).astype(np.float64)
    assert np.all(np.abs(got / 2.0 ** -125 - 1) < 1e-4)


def test_lmhead_degree4_bound():
    coef = _coefficients("dg_lmhead_tc.cu", "float exp2_poly4(")[-5:]
    assert len(coef) == 5 and abs(float(coef[-1]) - 1.0) < 1e-5
    x = np.concatenate([np.linspace(-125, 0, 2_000_001, dtype=np.float32), -np.arange(0, 126, dtype=np.float32),
                        -np.arange(0, 125, dtype=np.float32) - np.float32(0.5)])
    rel = np.max(np.abs(_exp2_poly(x, coef).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1))
    assert rel < 3e-6, rel
