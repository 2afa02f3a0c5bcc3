"""GPU parity of the fused 3D + 1D rotary encoding: cca_rope_qk on the Q/K
path and cca_kv_append_rope into the ring, against the fp64 oracle
(``oracle.rope``, complex arithmetic on the oracle's own frequency table).

The rotation is computed in fp32 and rounded once to bf16.  The bound per
element is one bf16 ulp of the exact value plus the fp32 error of the
rotation: the angle theta_i = sum_a p_a F_a[i] carries a few fp32 roundings
(the table entry, the products and sums: at most 4 * 2^-24 * sum_a |p_a F_a[i]|
radians), and sincos and the two fused multiply-adds another few 2^-24; either
moves an output by that angle times the norm of its plane (x_2i, x_2i+1).
Where a rotation nearly cancels, this term is many bf16 ulps of the small
result, so it is not folded into the ulp.  V is stored unrotated and
bit-exact.  E4M3 rings store the rotated keys' codes: their
dequantised values must be within half an e4m3 step (at the stored scale) of
the exact rotated keys, and the scales within 1e-5 of absmax / 448.
"""

import numpy as np
import pytest
import torch

import chunk_causal_attention_b200 as cca
from oracle import chunk_attention as oca
from oracle import fp8 as ofp8
from oracle import rope as orope
import synth

from test_gpu_parity import _record_errors, assert_attn_close, bf, check_status, dev, to_np  # noqa: F401

pytestmark = pytest.mark.gpu


def ulp_bf16(x):
    a = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    _, e = np.frexp(a)
    return np.ldexp(1.0, e - 8)


def _freq(D):
    return cca.cca_mrope_freqs(D, device=dev())


def rot_err_bound(x, pos, f):
    """Per-element bound of the fp32 rotation error (radians x plane norm)."""
    x = np.asarray(x, dtype=np.float64)
    th_abs = np.abs(np.asarray(pos, dtype=np.float64)) @ np.abs(f)  # [n, D/2]
    eps = 4 * 2.0 ** -24 * th_abs + 8 * 2.0 ** -24
    r = np.sqrt(x[..., 0::2] ** 2 + x[..., 1::2] ** 2) * eps[:, None, :]
    return np.repeat(r, 2, axis=-1)


def assert_rotated(got, x, pos, f):
    ref = orope.apply(x, pos, f)
    d = np.abs(np.asarray(got, dtype=np.float64) - ref)
    bound = ulp_bf16(ref) + rot_err_bound(x, pos, f)
    assert (d <= bound).all(), float((d / bound).max())


@pytest.mark.parametrize("src", ["bf16", "f32"])
def test_rope_qk_720p(src):
    g = np.random.default_rng(70)
    L, H, D = synth.TOKENS_720P, 24, 128
    q = g.standard_normal((L, H, D)).astype(np.float32)
    k = (3.0 * g.standard_normal((L, H, D))).astype(np.float32)
    if src == "bf16":
        q, k = synth.bf16_round(q), synth.bf16_round(k)
        qt, kt = bf(q), bf(k)
    else:
        qt, kt = torch.from_numpy(q).to(dev()), torch.from_numpy(k).to(dev())
    pos = synth.grid_positions(4, source=1)
    qo, ko = cca.cca_rope_qk(qt, kt, torch.from_numpy(pos).to(dev()), _freq(D))
    f = orope.frequencies(D)
    for got, x in ((qo, q), (ko, k)):
        assert_rotated(to_np(got), x, pos, f)


def test_rope_qk_one_tensor_and_ragged_tokens():
    g = np.random.default_rng(71)
    n, H, D = 333, 3, 64
    k = synth.bf16_round(g.standard_normal((n, H, D)).astype(np.float32))
    pos = np.stack([g.integers(0, 300, n), g.integers(-5, 40, n), g.integers(0, 60, n), g.integers(0, 4, n)],
                   1).astype(np.int32)
    _, ko = cca.cca_rope_qk(None, bf(k), torch.from_numpy(pos).to(dev()), _freq(D))
    assert_rotated(to_np(ko), k, pos, orope.frequencies(D))


@pytest.mark.parametrize("src", ["bf16", "f32"])
def test_append_rope_bf16_ring(src):
    g = np.random.default_rng(72)
    L, H, D, W = 300, 2, 128, 2
    ring = cca.KVRing(H, D, L, W, device=dev())
    f = orope.frequencies(D)
    for t in range(4):
        k = g.standard_normal((L, H, D)).astype(np.float32)
        v = g.standard_normal((L, H, D)).astype(np.float32)
        if src == "bf16":
            k, v = synth.bf16_round(k), synth.bf16_round(v)
            kt, vt = bf(k), bf(v)
        else:
            kt, vt = torch.from_numpy(k).to(dev()), torch.from_numpy(v).to(dev())
        pos = synth.grid_positions(t, grid=(10, 30))
        cca.cca_kv_append_rope(ring, kt, vt, torch.from_numpy(pos).to(dev()), _freq(D))
        n, slots, ids = ring.query()
        torch.cuda.synchronize()
        sl = slots[ids.index(t)]
        assert_rotated(to_np(ring.k_slots[sl]), k, pos, f)
        assert torch.equal(ring.v_slots[sl].cpu(), torch.from_numpy(v).to(torch.bfloat16))
    check_status(ring)


def test_append_rope_e4m3_ring():
    g = np.random.default_rng(73)
    L, H, D, W = 257, 3, 128, 1
    ring = cca.KVRing(H, D, L, W, dtype="e4m3", device=dev())
    k = synth.bf16_round(g.standard_t(4.0, size=(L, H, D)).astype(np.float32))
    v = synth.bf16_round(g.standard_t(4.0, size=(L, H, D)).astype(np.float32))
    pos = synth.grid_positions(0, grid=(1, L))
    cca.cca_kv_append_rope(ring, bf(k), bf(v), torch.from_numpy(pos).to(dev()), _freq(D))
    torch.cuda.synchronize()
    f = orope.frequencies(D)
    rot = orope.apply(k, pos, f)
    s = ring.k_scale[0].cpu().numpy().astype(np.float64)
    s_ref = np.abs(rot).max(axis=(0, 2)) / 448.0
    assert np.abs(s / s_ref - 1).max() < 1e-5
    deq = ofp8.e4m3_decode(ring.k_slots[0].cpu().numpy()) * s[None, :, None]
    err = rot_err_bound(k, pos, f)
    y = (np.abs(rot) + err) / s[None, :, None]  # the largest value the kernel's fp32 rotation can give
    _, e = np.frexp(np.maximum(y, 2.0 ** -6))
    half_step = np.ldexp(1.0, e - 1 - 3) / 2 * s[None, :, None]  # half an e4m3 step there, times the scale
    assert (np.abs(deq - rot) <= half_step * (1 + 1e-4) + err).all()
    vc, vs = ofp8.quantize_per_head(v)  # V is stored unrotated, bit-exact (codes widened to fp16)
    assert np.array_equal(ring.v_slots[0].cpu().numpy(), ofp8.e4m3_decode(vc).astype(np.float16))
    assert np.array_equal(ring.v_scale[0].cpu().numpy(), vs)


def test_rope_then_attention_matches_oracle():
    """The encoded Q/K path in front of the chunk attention, over a ring filled
    by the encoding append, against the oracle's encoding + attention."""
    g = np.random.default_rng(74)
    L, H, D, W, T = 270, 2, 128, 2, 4
    grid = (9, 30)
    f_ref = orope.frequencies(D)
    ring = cca.KVRing(H, D, L, W, device=dev())
    ks, vs = [], []
    for t in range(T):
        k = synth.bf16_round(g.standard_normal((L, H, D)).astype(np.float32))
        v = synth.bf16_round(g.standard_normal((L, H, D)).astype(np.float32))
        pos = synth.grid_positions(t, grid=grid)
        cca.cca_kv_append_rope(ring, bf(k), bf(v), torch.from_numpy(pos).to(dev()), _freq(D))
        ks.append(orope.apply(k, pos, f_ref))
        vs.append(v)
    q = synth.bf16_round(g.standard_normal((L, H, D)).astype(np.float32))
    kc = synth.bf16_round(g.standard_normal((L, H, D)).astype(np.float32))
    vc = synth.bf16_round(g.standard_normal((L, H, D)).astype(np.float32))
    pos = synth.grid_positions(T, grid=grid)
    qr, kr = cca.cca_rope_qk(bf(q), bf(kc), torch.from_numpy(pos).to(dev()), _freq(D))
    o = cca.cca_chunk_attn(ring, qr, kr, bf(vc))
    ref = oca.chunk_attention(orope.apply(q, pos, f_ref), ks, vs, T, W, k_cur=orope.apply(kc, pos, f_ref), v_cur=vc)
    assert_attn_close(to_np(o), ref, what="rope + attention")
    check_status(ring)
