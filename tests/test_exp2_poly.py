"""The FMA-pipe exponential of the attention softmax: its polynomial fit, its
binary32 evaluation and the constants compiled into the kernel.

The kernel evaluates part of its 2^x on the FMA pipe as 2^n * p(f) (Cody-Waite
reduction, degree-3 minimax p fitted by ``exp2_poly``).  These CPU tests keep
the three in step: the Remez fit reaches its documented 7.5e-5 relative error,
the bit-level emulation of the device sequence stays within that error (plus
the rounding of the binary32 steps) against ``numpy.exp2`` over the whole input
range the softmax uses, and the four constants in ``csrc/sm100.cuh`` are the
fitted binary32 coefficients bit for bit.
"""

import os
import re

import numpy as np

from chunk_causal_attention_b200 import exp2_poly

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "chunk_causal_attention_b200", "csrc", "sm100.cuh")

FIT_BOUND = 7.5e-5                 # documented relative error of the fit on [-1/2, 1/2]
F32_SLACK = 8 * 2.0 ** -24         # a handful of binary32 roundings in the evaluation


def test_remez_fit_reaches_documented_error_and_equioscillates():
    coef = exp2_poly.remez()
    f = np.linspace(exp2_poly.LO, exp2_poly.HI, 400001)
    e = exp2_poly._err(coef, f)
    emax = np.abs(e).max()
    assert emax <= FIT_BOUND
    # a minimax fit of degree 3 has 5 alternating extrema of equal size
    sgn = np.sign(e)
    runs = 1 + int(np.count_nonzero(sgn[1:] != sgn[:-1]))
    assert runs >= exp2_poly.DEGREE + 2
    # and the equal-error property: the end points hit the bound too
    assert abs(abs(e[0]) - emax) < 1e-3 * emax and abs(abs(e[-1]) - emax) < 1e-3 * emax


def test_binary32_evaluation_against_numpy_exp2():
    c = exp2_poly.coefficients_f32()
    x = np.linspace(-126.0, 0.0, 3_000_001).astype(np.float32)
    x = np.concatenate([x, np.float32([0.0, -0.5, 0.5 - 1.0, -1.0, -125.0, -2.0 ** -20])])
    got = exp2_poly.eval_f32(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    normal = x >= -125.0
    rel = np.abs(got[normal] / ref[normal] - 1.0)
    assert rel.max() <= FIT_BOUND + F32_SLACK, rel.max()
    # below 2^-125 the exponent insertion leaves the normal range: only the
    # absolute size matters there (P is rounded to bf16 next to values >= 1)
    assert np.abs(got[~normal] - ref[~normal]).max() <= 2.0 ** -124
    assert np.all(got >= 0.0)


def test_kernel_constants_equal_the_fit_bit_for_bit():
    src = open(HEADER).read()
    vals = {}
    for name, lit in re.findall(r"\b(kC[0-3])\s*=\s*([0-9.eE+-]+)f", src):
        vals[name] = np.float32(float(lit))
    assert sorted(vals) == ["kC0", "kC1", "kC2", "kC3"], vals
    want = exp2_poly.coefficients_f32()
    got = np.array([vals[f"kC{i}"] for i in range(4)], dtype=np.float32)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), (got, want)
