"""Pins of the rotary-encoding oracle (``oracle.rope``) by what a rotary
encoding must satisfy, independent of its own formula.

* Relative positions: q.k after encoding depends only on the difference of the
  two tokens' coordinates (the defining property of rotary encodings), for every
  coordinate including the source index.
* Each plane is rotated, so per-plane norms are preserved.
* Sections: moving t changes only the t planes (and h, w likewise); moving the
  source index changes every plane.
* Hand-computed values: a unit vector in plane i at (t, 0, 0, 0) comes out as
  (cos t f, sin t f) with f the plane's frequency from the stated recipe.
* Planted mistakes (rotation direction flipped on one operand's pairs, planes
  taken as (i, i + D/2), angles of 3D and 1D multiplied instead of added) break
  one of the pins.
"""

import numpy as np
import pytest

from oracle import rope

D = 64


def _pos(g, n):
    return np.stack([g.integers(0, 8, n), g.integers(0, 30, n), g.integers(0, 54, n), g.integers(0, 3, n)], 1)


def _scores(apply, q, k, pq, pk, f):
    return np.einsum("hd,hd->h", apply(q[None], pq[None], f)[0], apply(k[None], pk[None], f)[0])


def relative_ok(apply, f, seed=0):
    g = np.random.default_rng(seed)
    q, k = g.standard_normal((2, 3, D))
    for _ in range(20):
        pq, pk, shift = _pos(g, 1)[0], _pos(g, 1)[0], _pos(g, 1)[0]
        a = _scores(apply, q, k, pq, pk, f)
        b = _scores(apply, q, k, pq + shift, pk + shift, f)
        if np.abs(a - b).max() > 1e-9:
            return False
    return True


def test_relative_position_property():
    f = rope.frequencies(D)
    assert relative_ok(rope.apply, f)


def test_plane_norms_preserved():
    g = np.random.default_rng(1)
    x = g.standard_normal((50, 2, D))
    y = rope.apply(x, _pos(g, 50), rope.frequencies(D))
    nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    assert np.abs(nx - ny).max() < 1e-12


def test_sections_move_only_their_planes():
    f = rope.frequencies(D)
    st, sh, sw = rope.sections_default(D)
    g = np.random.default_rng(2)
    x = g.standard_normal((1, 1, D))
    p0 = np.array([[1, 2, 3, 0]])
    base = rope.apply(x, p0, f)
    spans = {0: range(0, st), 1: range(st, st + sh), 2: range(st + sh, st + sh + sw)}
    for a in range(3):
        p = p0.copy()
        p[0, a] += 1
        moved = np.abs(rope.apply(x, p, f) - base)[0, 0].reshape(-1, 2).max(axis=1) > 1e-12
        assert set(np.flatnonzero(moved)) == set(spans[a])
    p = p0.copy()
    p[0, 3] += 1
    moved = np.abs(rope.apply(x, p, f) - base)[0, 0].reshape(-1, 2).max(axis=1) > 1e-12
    assert moved.all()


def test_hand_computed_angles():
    f = rope.frequencies(D, sections=(12, 10, 10), base=10000.0)
    # plane 3 lies in the t section (12 planes): frequency 10000^(-3/12); plane 0 of h (index 12): 1
    for plane, a, freq in [(3, 0, 10000.0 ** (-3 / 12)), (12, 1, 1.0), (25, 2, 10000.0 ** (-3 / 10))]:
        x = np.zeros((1, 1, D))
        x[0, 0, 2 * plane] = 1.0
        p = np.zeros((1, 4), dtype=np.int64)
        p[0, a] = 5
        y = rope.apply(x, p, f)[0, 0]
        assert abs(y[2 * plane] - np.cos(5 * freq)) < 1e-12 and abs(y[2 * plane + 1] - np.sin(5 * freq)) < 1e-12
    # the source index: every plane i at 10000^(-2i/D)
    x = np.zeros((1, 1, D))
    x[0, 0, 2 * 7 + 1] = 1.0  # imaginary part of plane 7
    y = rope.apply(x, np.array([[0, 0, 0, 2]]), f)[0, 0]
    th = 2 * 10000.0 ** (-14 / D)
    assert abs(y[14] + np.sin(th)) < 1e-12 and abs(y[15] - np.cos(th)) < 1e-12


def _planted_half_split(x, pos, freq):
    x = np.asarray(x, dtype=np.float64)
    h = x.shape[-1] // 2
    z = (x[..., :h] + 1j * x[..., h:]) * np.exp(1j * rope.angles(pos, freq))[:, None, :]
    return np.concatenate([z.real, z.imag], axis=-1)


def _planted_product(x, pos, freq):
    p = np.asarray(pos, dtype=np.float64)
    th = (p[:, :3] @ freq[:3]) * (p[:, 3:] @ freq[3:4])
    x = np.asarray(x, dtype=np.float64)
    z = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * th)[:, None, :]
    out = np.empty_like(x)
    out[..., 0::2], out[..., 1::2] = z.real, z.imag
    return out


@pytest.mark.parametrize("plant", ["half_split", "product"])
def test_planted_mistakes_are_caught(plant):
    f = rope.frequencies(D)
    if plant == "half_split":
        # still a rotation, so only the hand-computed plane layout exposes it
        x = np.zeros((1, 1, D))
        x[0, 0, 6] = 1.0
        y = _planted_half_split(x, np.array([[5, 0, 0, 0]]), f)[0, 0]
        assert abs(y[6] - np.cos(5 * f[0, 3])) > 1e-3 or abs(y[7] - np.sin(5 * f[0, 3])) > 1e-3
    else:
        assert not relative_ok(_planted_product, f)


def test_flipped_direction_on_one_side_breaks_relative_property():
    f = rope.frequencies(D)

    def mixed(x, pos, freq, _n=[0]):
        _n[0] += 1
        return rope.apply(x, pos if _n[0] % 2 else -pos, freq)
    assert not relative_ok(mixed, f)
