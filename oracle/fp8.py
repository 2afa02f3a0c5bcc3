"""Oracle: FP8 e4m3 encoding and per-head absmax quantisation.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages say only that FP8 quantisation is applied across the deployed
pipeline ["JoyAI-Video-Edit 소개", section 30 FPS를 만드는 실시간 배포
파이프라인; "論文解説: JoyAI-Video-Edit", §5].  Format and granularity are left
open; the reading used here is:

* format: OCP "e4m3fn" -- 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits,
  subnormals, no infinities, 0x7F/0xFF are NaN, largest finite value 448;
* rounding: round-to-nearest-even, saturating to +-448 (never NaN for finite in);
  the sign of zero is kept (a negative value that rounds to zero gives 0x80);
* scale per (tensor, head): ``s = fl32(absmax / 448)`` with ``s = 1`` when the
  head is all zeros, and the code of ``x`` is ``e4m3(fl32(x / s))`` where both
  divisions are IEEE-754 binary32 divisions (correctly rounded);
* dequantised value ``x_hat = decode(code) * s``.

The encoder is written from the format's definition (value = 2^(e-7)(1+m/8) for
normal codes, 2^-6 (m/8) for subnormal codes).  Pins: every one of the 254
finite codes round-trips; hand-checked codes (1.0 -> 0x38, 448 -> 0x7E,
2^-9 -> 0x01, ties to even); and agreement with ``torch.float8_e4m3fn``
conversion (a library routine) on in-range values.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
_MIN_NORMAL = 2.0 ** -6
_SUBNORMAL_QUANTUM = 2.0 ** -9


def _positive_code_values() -> np.ndarray:
    """Value of each non-negative code 0x00..0x7E (index = code)."""
    vals = np.empty(127, dtype=np.float64)
    for code in range(127):
        e = code >> 3
        m = code & 7
        if e == 0:
            vals[code] = (m / 8.0) * _MIN_NORMAL
        else:
            vals[code] = 2.0 ** (e - 7) * (1.0 + m / 8.0)
    return vals


_POS_VALUES = _positive_code_values()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """uint8 codes -> fp64 values (NaN for 0x7F / 0xFF)."""
    codes = np.asarray(codes, dtype=np.uint8)
    mag = codes & 0x7F
    out = np.where(mag == 0x7F, np.nan, _POS_VALUES[np.minimum(mag, 126)])
    return np.where(codes & 0x80, -out, out)


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Round finite values to the nearest e4m3 value (ties to even), saturating."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    # spacing of the e4m3 grid at |a|: 2^-9 below 2^-6, else 2^(floor(log2 a) - 3)
    _, e2 = np.frexp(np.where(a > 0, a, 1.0))  # a = m * 2^e2, m in [0.5, 1): exact
    quantum = np.where(a < _MIN_NORMAL, _SUBNORMAL_QUANTUM, np.ldexp(1.0, e2 - 1 - 3))
    r = np.rint(a / quantum) * quantum  # np.rint rounds half to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Finite values -> uint8 e4m3 codes (round-to-nearest-even, saturating)."""
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("e4m3_encode expects finite inputs")
    r = e4m3_round(x)
    mag = np.searchsorted(_POS_VALUES, np.abs(r)).astype(np.uint8)
    assert np.array_equal(_POS_VALUES[mag], np.abs(r)), "value not on the e4m3 grid"
    sign = np.where(np.signbit(r), 0x80, 0).astype(np.uint8)  # zero keeps its sign
    return (mag | sign).astype(np.uint8)


def head_scales(x: np.ndarray) -> np.ndarray:
    """Per-head scale s_h = fl32(absmax_h / 448) (1 for an all-zero head).

    x: [n_tok, H, D], float values exactly representable in binary32.
    """
    x32 = np.asarray(x, dtype=np.float32)
    absmax = np.abs(x32).max(axis=(0, 2)) if x32.shape[0] > 0 else np.zeros(x32.shape[1], np.float32)
    s = (absmax / np.float32(E4M3_MAX)).astype(np.float32)
    return np.where(absmax > 0, s, np.float32(1.0)).astype(np.float32)


def quantize_per_head(x: np.ndarray):
    """Per-head absmax quantisation of x [n_tok, H, D] -> (codes uint8, scale fp32 [H])."""
    x32 = np.asarray(x, dtype=np.float32)
    s = head_scales(x32)
    y = (x32 / s[None, :, None]).astype(np.float32)  # binary32 division, per element
    return e4m3_encode(y.astype(np.float64)), s


def dequantize_per_head(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """x_hat = decode(code) * s_h in fp64."""
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[None, :, None]
