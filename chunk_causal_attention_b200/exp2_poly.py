"""Minimax polynomial for 2^f on [-1/2, 1/2] (relative error), fitted here.

The attention kernel evaluates part of its exponentials on the FMA pipe instead
of the MUFU unit (whose 16 results/clock/SM would otherwise cap the softmax):

    2^x = 2^n * 2^f,   n = round(x),  f = x - n in [-1/2, 1/2]   (Cody-Waite)

``n`` comes from the round-to-nearest of ``x + 1.5 * 2^23`` (the float's low
mantissa bits then hold n), 2^f from the polynomial below, and the product by 2^n
is an integer add of ``n << 23`` to the bit pattern of p(f).

The coefficients are a Remez-exchange fit (equioscillating relative error) of
degree ``DEGREE``, computed in binary64 and rounded to binary32.  Running this
module prints them in the form used by ``csrc/attn.cu``; ``tests`` check the
fit and the binary32 evaluation against ``numpy.exp2``.
"""

from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _err(coef, x):
    return np.polyval(coef[::-1], x) / np.exp2(x) - 1.0


def remez(degree: int = DEGREE, iters: int = 30) -> np.ndarray:
    """Coefficients c0..c_deg (ascending) minimising max |p(f) / 2^f - 1| on [LO, HI]."""
    n = degree
    k = np.arange(n + 2)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n + 1 - k) / (n + 1))  # Chebyshev extrema
    dense = np.linspace(LO, HI, 20001)
    coef = None
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  (relative error E with alternating sign)
        A = np.zeros((n + 2, n + 2))
        for i in range(n + 2):
            A[i, :n + 1] = x[i] ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * np.exp2(x[i])
        sol = np.linalg.solve(A, np.exp2(x))
        coef = sol[:n + 1]
        e = _err(coef, dense)
        # new reference: the extremum of each sign-alternating run of the error
        idx = []
        start = 0
        sgn = np.sign(e)
        for i in range(1, len(dense) + 1):
            if i == len(dense) or sgn[i] != sgn[start]:
                seg = np.arange(start, i)
                idx.append(seg[np.argmax(np.abs(e[seg]))])
                start = i
        if len(idx) < n + 2:
            break
        idx = np.array(idx)
        while len(idx) > n + 2:  # drop the smallest end extremum
            if abs(e[idx[0]]) < abs(e[idx[-1]]):
                idx = idx[1:]
            else:
                idx = idx[:-1]
        x = dense[idx]
    return coef


def coefficients_f32(degree: int = DEGREE) -> np.ndarray:
    return remez(degree).astype(np.float32)


def eval_f32(x: np.ndarray, coef: np.ndarray) -> np.ndarray:
    """Binary32 emulation of the device sequence (clamp at -126 so the exponent
    add can never borrow into the sign bit, magic round, Horner with
    fused multiply-adds, exponent insertion by integer add)."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)  # 1.5 * 2^23
    t = (x + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    f = (x - r).astype(np.float32)
    p = np.full_like(f, coef[-1], dtype=np.float64)
    for c in coef[-2::-1]:  # fma in binary64 then one rounding == fused multiply-add
        p = (p * f.astype(np.float64) + np.float64(c)).astype(np.float32).astype(np.float64)
    p = p.astype(np.float32)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    c = coefficients_f32()
    d = np.linspace(LO, HI, 200001)
    print("max rel err (binary64 coefs):", np.abs(_err(remez().astype(np.float64), d)).max())
    print("coefficients (ascending, binary32):")
    for i, v in enumerate(c):
        print(f"  c{i} = {float(v)!r}f  // {np.float32(v).view(np.uint32):#010x}")
