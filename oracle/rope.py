"""Oracle: rotary position encoding with a fused 3D + 1D angle.

TEST INFRASTRUCTURE ONLY (see the package docstring).

["JoyAI-Video-Edit 소개", section 세 부품으로 이루어진 아키텍처]: the position
encoding builds its rotation angles by fusing a 3D spatio-temporal RoPE with a
1D source RoPE, so source and generated tokens in one sequence play different
roles.  The formula is not on the pages; the reading used here:

* every token has integer coordinates (t, h, w, s): latent frame, row, column
  and a source index;
* the head's D elements form D/2 planes, plane i = elements (2i, 2i+1), read as
  the complex number z_i = x_{2i} + 1j x_{2i+1};
* the 3D part gives plane i the angle p_a * f_a(i) of the one coordinate a whose
  section holds i (sections t, h, w in that order, frequencies base^(-j/sec_a)
  inside a section of sec_a planes); the 1D source part gives every plane the
  angle s * base^(-2i/D);
* both rotate the same plane, so the angles add:  z_i -> z_i * exp(1j theta_i).

Computed in fp64 with complex arithmetic.  Pins (``tests/test_oracle_rope.py``):
the relative-position property (scores depend only on coordinate differences),
norm preservation, section separation (a coordinate moves only its planes and the
source index moves all), and hand-computed angles at small positions.
"""

from __future__ import annotations

import numpy as np


def sections_default(head_dim: int) -> tuple[int, int, int]:
    """Planes per coordinate (t, h, w): a third each, the remainder to t."""
    p = head_dim // 2
    return (p - 2 * (p // 3), p // 3, p // 3)


def frequencies(head_dim: int, sections=None, base: float = 10000.0) -> np.ndarray:
    """[4, D/2] angular frequencies: rows t, h, w (zero outside their section), s."""
    if sections is None:
        sections = sections_default(head_dim)
    p = head_dim // 2
    if sum(sections) != p:
        raise ValueError("sections must cover D/2 planes")
    f = np.zeros((4, p), dtype=np.float64)
    start = 0
    for a, n in enumerate(sections):
        f[a, start:start + n] = base ** (-np.arange(n, dtype=np.float64) / n)
        start += n
    f[3] = base ** (-2.0 * np.arange(p, dtype=np.float64) / head_dim)
    return f


def angles(pos: np.ndarray, freq: np.ndarray) -> np.ndarray:
    """theta [n, D/2] = sum over the four coordinates of position x frequency."""
    return np.asarray(pos, dtype=np.float64) @ np.asarray(freq, dtype=np.float64)


def apply(x: np.ndarray, pos: np.ndarray, freq: np.ndarray) -> np.ndarray:
    """Rotate x [n, H, D] at positions pos [n, 4] (fp64 result)."""
    x = np.asarray(x, dtype=np.float64)
    n, h, d = x.shape
    z = x[..., 0::2] + 1j * x[..., 1::2]
    z = z * np.exp(1j * angles(pos, freq))[:, None, :]
    out = np.empty_like(x)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out
