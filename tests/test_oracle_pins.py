"""Pins of the fp64 oracle against things other than itself (CPU only).

Each pin is chosen so that a plausible mistake in the oracle (a dropped sink, a
wrong window bound, a wrong scale, a transposed operand, '>=' for '>', a wrong
tie rule in the FP8 encoder) fails at least one of them; the planted-mistake
tests at the bottom check exactly that, by running the same pin checks against
deliberately broken copies of the oracle functions.

Sources of the rules (page title, section): chunk-causal windowed attention with
a global sink -- "JoyAI-Video-Edit 소개", 청크 단위 자기회귀 적응; the bounded
KV store -- same page, 30 FPS를 만드는 실시간 배포 파이프라인; the mask cache --
"LiveEdit 실시간 Diffusion 기반 스트리밍 비디오 편집", 기술 상세.
"""

import math

import numpy as np
import pytest
import torch

from oracle import chunk_attention as ca
from oracle import fp8
from oracle import kv_ring
from oracle import mask_cache as mc
import synth

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


# --------------------------------------------------------------- helpers
def _stream(seed, n_chunks, L, H, D):
    g = np.random.default_rng(seed)
    q = [g.standard_normal((L, H, D)) for _ in range(n_chunks)]
    k = [g.standard_normal((L, H, D)) for _ in range(n_chunks)]
    v = [g.standard_normal((L, H, D)) for _ in range(n_chunks)]
    return q, k, v


def brute_force_block_causal(q_all, k_all, v_all, chunk_len, scale):
    """Pure-Python attention over the whole packed sequence with the explicit
    element mask M[i, j] = [chunk(j) <= chunk(i)] (full block-causal; the
    packed training-style form of the chunk-causal mask)."""
    n, h_, d_ = len(q_all), len(q_all[0]), len(q_all[0][0])
    out = [[[0.0] * d_ for _ in range(h_)] for _ in range(n)]
    for h in range(h_):
        for i in range(n):
            ci = i // chunk_len
            scores = []
            for j in range(n):
                if j // chunk_len <= ci:
                    s = sum(q_all[i][h][c] * k_all[j][h][c] for c in range(d_)) * scale
                    scores.append((j, s))
            mx = max(s for _, s in scores)
            w = [(j, math.exp(s - mx)) for j, s in scores]
            z = sum(e for _, e in w)
            for c in range(d_):
                out[i][h][c] = sum(e * v_all[j][h][c] for j, e in w) / z
    return np.array(out)


def pin_block_causal(attn_fn=ca.chunk_attention, vis_fn=None):
    """P-a / P-e: window >= t  ==>  equal to brute-force block-causal attention."""
    L, H, D, n = 3, 2, 4, 4
    q, k, v = _stream(11, n, L, H, D)
    ref = brute_force_block_causal(np.concatenate(q).tolist(), np.concatenate(k).tolist(),
                                   np.concatenate(v).tolist(), L, 1 / math.sqrt(D))
    err = 0.0
    for t in range(n):
        o = attn_fn(q[t], k, v, t, window=n) if vis_fn is None else attn_fn(q[t], k, v, t, n, vis_fn)
        err = max(err, np.abs(o - ref[t * L:(t + 1) * L]).max())
    return err


# --------------------------------------------------------------- visible set / ring
def test_visible_chunks_hand_cases():
    # sink + W most recent past chunks + the chunk itself
    assert ca.visible_chunks(0, 3) == [0]
    assert ca.visible_chunks(1, 2) == [0, 1]
    assert ca.visible_chunks(3, 2) == [0, 1, 2, 3]  # window reaches chunk 1: no eviction
    assert ca.visible_chunks(4, 2) == [0, 2, 3, 4]  # chunk 1 evicted
    assert ca.visible_chunks(4, 3) == [0, 1, 2, 3, 4]
    assert ca.visible_chunks(9, 3) == [0, 6, 7, 8, 9]
    assert ca.visible_chunks(5, 0) == [0, 5]


def test_ring_deque_matches_visible_set_over_225_chunks():
    """Two separate restatements of the same rule agree: the deque of cached
    chunks after n appends is the visible set of chunk n minus chunk n."""
    for w in (0, 1, 2, 3, 7):
        ring = kv_ring.KVRing(w)
        for n in range(225):
            assert ring.chunks() == [c for c in ca.visible_chunks(n, w) if c != n] if n > 0 else ring.chunks() == []
            ring.append(n, n)
            assert ring.n_appended == n + 1
            # bounded memory: never more than sink + w chunks
            assert len(ring.chunks()) <= 1 + w


def test_ring_get_and_eviction():
    ring = kv_ring.KVRing(2)
    for n in range(6):
        ring.append(("k", n), ("v", n))
    assert ring.chunks() == [0, 4, 5]
    assert ring.get(0) == (("k", 0), ("v", 0))
    with pytest.raises(KeyError):
        ring.get(3)


# --------------------------------------------------------------- attention pins
def test_pin_block_causal_bruteforce():
    assert pin_block_causal() < 1e-12


def pin_window(attn_fn=ca.chunk_attention, vis_fn=None):
    """Window smaller than history: brute force over the packed sequence with
    an element mask built from the page's prose (key j visible from chunk t iff
    j is in the sink chunk or in one of chunks t-w .. t)."""
    L, H, D, n, w = 2, 2, 4, 7, 2
    q, k, v = _stream(12, n, L, H, D)
    scale = 1 / math.sqrt(D)
    err = 0.0
    for t in range(n):
        keys = [j for j in range(n * L) if (j // L == 0) or (t - w <= j // L <= t)]
        o_bf = np.zeros((L, H, D))
        for i in range(L):
            for h in range(H):
                s = np.array([np.dot(q[t][i, h], k[j // L][j % L, h]) * scale for j in keys])
                p = np.exp(s - s.max())
                p /= p.sum()
                o_bf[i, h] = sum(p[a] * v[j // L][j % L, h] for a, j in enumerate(keys))
        o = attn_fn(q[t], k, v, t, w) if vis_fn is None else attn_fn(q[t], k, v, t, w, vis_fn)
        err = max(err, np.abs(o - o_bf).max())
    return err


def test_pin_window_bruteforce_with_eviction():
    assert pin_window() < 1e-12


def test_pin_causality_future_perturbation():
    L, H, D, n, w = 4, 2, 8, 6, 2
    q, k, v = _stream(13, n, L, H, D)
    base = [ca.chunk_attention(q[t], k, v, t, w) for t in range(n)]
    k2 = [x.copy() for x in k]
    v2 = [x.copy() for x in v]
    for c in range(3, n):  # perturb chunks > 2
        k2[c] += 5.0
        v2[c] -= 3.0
    for t in range(3):
        assert np.array_equal(ca.chunk_attention(q[t], k2, v2, t, w), base[t])


def test_pin_window_evicted_perturbation():
    L, H, D, n, w = 4, 2, 8, 8, 2
    q, k, v = _stream(14, n, L, H, D)
    t = 6  # sees {0, 4, 5, 6}
    base = ca.chunk_attention(q[t], k, v, t, w)
    k2 = [x.copy() for x in k]
    for c in (1, 2, 3, 7):  # evicted and future
        k2[c] = k2[c] * -7.0
    assert np.array_equal(ca.chunk_attention(q[t], k2, v, t, w), base)
    for c in (0, 4, 5):  # sink and window matter
        k3 = [x.copy() for x in k]
        k3[c] = k3[c] * -7.0
        assert np.abs(ca.chunk_attention(q[t], k3, v, t, w) - base).max() > 1e-3


def test_pin_softmax_rows_sum_to_one():
    L, H, D, n, w = 5, 3, 8, 5, 2
    q, k, v = _stream(15, n, L, H, D)
    o, p = ca.chunk_attention(q[4], k, v, 4, w, return_probs=True)
    assert np.all(p >= 0)
    assert np.abs(p.sum(axis=-1) - 1.0).max() < 1e-13
    kk = np.concatenate([k[c] for c in ca.visible_chunks(4, w)])
    vv = np.concatenate([v[c] for c in ca.visible_chunks(4, w)])
    for h in range(H):
        assert np.abs(p[h] @ vv[:, h] - o[:, h]).max() < 1e-12
        # probabilities are a softmax of the scaled scores: log-ratios match
        s = q[4][:, h] @ kk[:, h].T / math.sqrt(D)
        lr = np.log(p[h]) - np.log(p[h][:, :1])
        assert np.abs(lr - (s - s[:, :1])).max() < 1e-9


def test_pin_closed_forms():
    g = np.random.default_rng(16)
    # one key: output is that key's value
    q = g.standard_normal((1, 2, 8)); k = g.standard_normal((1, 2, 8)); v = g.standard_normal((1, 2, 8))
    assert np.abs(ca.chunk_attention(q, [k], [v], 0, 3) - v).max() < 1e-15
    # all keys equal, or zero query: uniform average of the visible values
    L, H, D, n, w = 4, 2, 8, 6, 2
    qs, ks, vs = _stream(17, n, L, H, D)
    same = [np.broadcast_to(ks[0][:1], ks[0].shape).copy() for _ in range(n)]
    t = 5
    vis = ca.visible_chunks(t, w)
    mean_v = np.concatenate([vs[c] for c in vis]).mean(axis=0)
    o1 = ca.chunk_attention(qs[t], same, vs, t, w)
    o2 = ca.chunk_attention(np.zeros_like(qs[t]), ks, vs, t, w)
    assert np.abs(o1 - mean_v[None]).max() < 1e-12
    assert np.abs(o2 - mean_v[None]).max() < 1e-12


def test_pin_single_chunk_equals_library_sdpa():
    g = np.random.default_rng(18)
    L, H, D = 16, 3, 64
    q, k, v = (g.standard_normal((L, H, D)) for _ in range(3))
    o = ca.chunk_attention(q, [k], [v], 0, 2)
    tq, tk, tv = (torch.from_numpy(x).permute(1, 0, 2)[None] for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0].permute(1, 0, 2).numpy()
    assert np.abs(o - ref).max() < 1e-12


def test_pin_permuting_visible_chunks():
    L, H, D = 6, 2, 8
    q, k, v = _stream(19, 5, L, H, D)
    o = ca.softmax_attention(q[4], np.concatenate(k), np.concatenate(v))
    perm = [3, 0, 4, 1, 2]
    o2 = ca.softmax_attention(q[4], np.concatenate([k[i] for i in perm]), np.concatenate([v[i] for i in perm]))
    assert np.abs(o - o2).max() < 1e-13


def test_k_cur_overrides_cached_current_chunk():
    L, H, D = 4, 2, 8
    q, k, v = _stream(20, 3, L, H, D)
    kc, vc = k[2] * 0.5, v[2] + 1.0
    k2 = list(k); v2 = list(v)
    k2[2], v2[2] = kc, vc
    assert np.array_equal(ca.chunk_attention(q[2], k, v, 2, 1, k_cur=kc, v_cur=vc),
                          ca.chunk_attention(q[2], k2, v2, 2, 1))


def test_flops_720p():
    assert ca.flops_per_call(1620, 8100, 24, 128) == pytest.approx(1.612e11, rel=1e-3)


# --------------------------------------------------------------- mask pins
def test_mask_equals_library_norm_threshold():
    m = synth.mask_chunk()
    mask, d, tau = mc.token_mask(m.src, m.edit, tau=3.0)
    ref = np.linalg.norm(m.edit.astype(np.float64) - m.src.astype(np.float64), axis=1)
    assert np.abs(d - ref).max() < 1e-12
    assert np.array_equal(mask, (ref > 3.0).astype(np.uint8))


def test_mask_dynamic_quantile_counts():
    m = synth.mask_chunk()
    mask, d, tau = mc.token_mask(m.src, m.edit, prune_quantile=0.70)
    n = d.shape[0]
    k = mc.prune_count(n, 0.70)
    assert n == 1620 and k == 1134
    assert int(mask.sum()) == n - k == 486
    # ~70 % pruned and the active set is (nearly) the edited region
    assert abs(m.region.mean() - 0.30) <= 0.02
    assert (mask.astype(bool) == m.region).mean() > 0.97


def test_mask_hand_cases():
    src = np.zeros((5, 4))
    edit = np.array([[0.5, 0, 0, 0], [3, 0, 0, 0], [1, 0, 0, 0], [0, 2, 0, 0], [0, 0, 0.6, 0.8]])
    # distances 0.5, 3, 1, 2, 1 ; strict '>' keeps d == tau inactive
    mask, d, tau = mc.token_mask(src, edit, tau=1.0)
    assert list(mask) == [0, 1, 0, 1, 0]
    mask, d, tau = mc.token_mask(src, edit, prune_quantile=0.4)  # k = 2 -> tau = 1
    assert tau == 1.0 and list(mask) == [0, 1, 0, 1, 0]
    mask, _, tau = mc.token_mask(src, src, tau=0.0)  # identical latents: nothing active
    assert tau == 0.0 and mask.sum() == 0
    mask, _, _ = mc.token_mask(src, edit, prune_quantile=1.0)
    assert mask.sum() == 0


def test_compact_and_scatter():
    g = np.random.default_rng(21)
    mask = (g.random(300) < 0.3).astype(np.uint8)
    idx, n = mc.compact(mask)
    assert np.array_equal(idx, np.flatnonzero(mask).astype(np.int32)) and n == mask.sum()
    cache = g.standard_normal((300, 3, 4)).astype(np.float32)
    oc = g.standard_normal((n, 3, 4)).astype(np.float32)
    out = mc.scatter(oc, idx, n, cache)
    assert np.array_equal(out[mask == 0], cache[mask == 0])
    assert np.array_equal(out[idx], oc)
    empty_idx, n0 = mc.compact(np.zeros(10, np.uint8))
    assert n0 == 0 and empty_idx.size == 0
    assert np.array_equal(mc.scatter(oc[:0], empty_idx, 0, cache[:10]), cache[:10])


# --------------------------------------------------------------- fp8 pins
def test_e4m3_codes_round_trip():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert codes.size == 254
    assert np.array_equal(fp8.e4m3_encode(fp8.e4m3_decode(codes)), codes)


def test_e4m3_hand_values():
    cases = [(1.0, 0x38), (448.0, 0x7E), (-448.0, 0xFE), (2.0 ** -9, 0x01), (2.0 ** -6, 0x08),
             (0.0, 0x00), (-0.0, 0x80), (1.0625, 0x38), (1.1875, 0x3A), (1.5 * 2 ** -9, 0x02),
             (0.5 * 2 ** -9, 0x00), (-0.5 * 2 ** -9, 0x80), (460.0, 0x7E), (1000.0, 0x7E),
             (-1e6, 0xFE), (240.0, 0x77), (0.75, 0x34), (0.5, 0x30), (3.5, 0x46)]
    for x, c in cases:
        assert fp8.e4m3_encode(np.array([x]))[0] == c, (x, hex(c))


def test_e4m3_matches_torch_float8():
    g = np.random.default_rng(22)
    y = np.concatenate([g.standard_normal(20000) * s for s in (1e-3, 0.05, 1.0, 30.0, 200.0)])
    y = np.clip(y, -448, 448).astype(np.float32)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(fp8.e4m3_encode(y.astype(np.float64)), ref)


def test_head_scales_and_dequant_error():
    g = np.random.default_rng(23)
    x = g.standard_t(4.0, size=(200, 3, 16)).astype(np.float32)
    x[:, 1] = 0.0
    codes, s = fp8.quantize_per_head(x)
    amax = np.abs(x).max(axis=(0, 2))
    assert s[1] == 1.0 and s[0] == np.float32(amax[0] / np.float32(448))
    xh = fp8.dequantize_per_head(codes, s)
    assert np.all(np.abs(xh) <= 448 * s[None, :, None] * (1 + 1e-6))
    # relative error of e4m3 (3 mantissa bits) is at most 2^-4 for normal values
    big = np.abs(x) > 2 ** -6 * s[None, :, None] * 2
    assert np.all(np.abs(xh - x)[big] <= np.abs(x)[big] * 2.0 ** -4 * 1.0001)


def _absmax_uses_full_range(quantize):
    """What the e4m3fn format fixes for an absmax scale: in every non-zero head
    the largest magnitude lands on the largest finite code (0x7E = 448), no code
    exceeds it, and an all-zero head gives only zero codes.  `quantize` maps
    x [n, H, D] to (codes, scale)."""
    g = np.random.default_rng(31)
    heads = [g.standard_normal((300, 4, 32)), g.standard_t(4.0, size=(300, 4, 32)),
             g.uniform(-1e-3, 1e-3, size=(300, 4, 32)), g.standard_t(1.5, size=(300, 4, 32)) * 1e3]
    for x in heads:
        x = x.astype(np.float32)
        x[:, 2] = 0.0
        codes, _ = quantize(x)
        mag = codes & 0x7F
        if np.any(mag > 0x7E):
            return False
        for h in range(x.shape[1]):
            xh, ch = np.abs(x[:, h]), mag[:, h]
            if not xh.any():
                if np.any(ch != 0):
                    return False
                continue
            if not np.all(ch[xh == xh.max()] == 0x7E):
                return False
    return True


def test_head_scales_pin_absmax_encodes_to_largest_code():
    assert _absmax_uses_full_range(fp8.quantize_per_head)


def test_planted_scale_divisor_240_is_caught():
    def planted(x):  # the e4m3fnuz maximum (240) as divisor: the range is left unused
        amax = np.abs(x).max(axis=(0, 2))
        s = np.where(amax > 0, (amax / np.float32(240.0)).astype(np.float32), np.float32(1.0)).astype(np.float32)
        y = (x / s[None, :, None]).astype(np.float32)
        return fp8.e4m3_encode(y.astype(np.float64)), s
    assert not _absmax_uses_full_range(planted)


def test_head_scale_of_power_of_two_range_is_exact():
    # absmax = 448 * 2^k gives s = 2^k exactly, and grid values times s come back unchanged
    grid = fp8.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    for k in (-12, -3, 0, 5):
        x = np.zeros((grid.size, 1, 2), dtype=np.float32)
        x[:, 0, 0] = (grid * 2.0 ** k).astype(np.float32)
        x[:, 0, 1] = -x[:, 0, 0]
        codes, s = fp8.quantize_per_head(x)
        assert s[0] == np.float32(2.0 ** k)
        assert np.array_equal(fp8.dequantize_per_head(codes, s), x.astype(np.float64))


# --------------------------------------------------------------- planted mistakes
def _vis_no_sink(t, window):
    return [c for c in ca.visible_chunks(t, window) if c != 0 or t == 0]


def _attn_with_vis(q_t, k, v, t, window, vis_fn):
    vis = vis_fn(t, window)
    return ca.softmax_attention(q_t, np.concatenate([k[c] for c in vis]), np.concatenate([v[c] for c in vis]))


def test_planted_dropped_sink_is_caught():
    assert pin_block_causal(_attn_with_vis, ca.visible_chunks) < 1e-12
    assert pin_block_causal(_attn_with_vis, _vis_no_sink) > 1e-3


def test_planted_window_off_by_one_is_caught():
    def vis_short(t, window):  # one history chunk too few
        return sorted({0, t} | set(range(max(1, t - window + 1), t)))
    assert pin_window(_attn_with_vis, ca.visible_chunks) < 1e-12
    assert pin_window(_attn_with_vis, vis_short) > 1e-3
    assert pin_window(_attn_with_vis, _vis_no_sink) > 1e-3


def test_planted_wrong_scale_or_transpose_is_caught():
    g = np.random.default_rng(24)
    L, H, D = 16, 2, 64
    q, k, v = (g.standard_normal((L, H, D)) for _ in range(3))
    tq, tk, tv = (torch.from_numpy(x).permute(1, 0, 2)[None] for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0].permute(1, 0, 2).numpy()
    wrong_scale = ca.softmax_attention(q, k, v, scale=1.0 / D)
    assert np.abs(wrong_scale - ref).max() > 1e-3
    # transposed operand: use k in place of v
    assert np.abs(ca.softmax_attention(q, k, k) - ref).max() > 1e-3


def test_planted_non_strict_mask_is_caught():
    src = np.zeros((3, 2))
    edit = np.array([[1.0, 0], [2, 0], [0.5, 0]])
    d = mc.l2_distance(src, edit)
    assert list((d >= 1.0).astype(np.uint8)) != list(mc.token_mask(src, edit, tau=1.0)[0])


def test_planted_round_half_away_is_caught():
    def enc_half_away(x):
        a = np.abs(x)
        _, e2 = np.frexp(a)
        qn = np.ldexp(1.0, e2 - 4)
        return np.copysign(np.floor(a / qn + 0.5) * qn, x)
    tie = np.array([1.0625])
    assert enc_half_away(tie)[0] != fp8.e4m3_decode(fp8.e4m3_encode(tie))[0]


def test_mask_frames_is_thresholded_norm_over_frames_and_channels():
    g = np.random.default_rng(41)
    F, N, C = 3, 200, 16
    src = g.standard_normal((F, N, C)).astype(np.float32)
    edit = (src + g.normal(0, 1, (F, N, C))).astype(np.float32)
    m, d, tau = mc.token_mask_frames(src, edit, tau=5.0)
    # library routine on the position-major layout [N, F * C]
    ref = np.linalg.norm((edit.astype(np.float64) - src).transpose(1, 0, 2).reshape(N, F * C), axis=1)
    assert np.allclose(d, ref, rtol=1e-14, atol=0)
    assert np.array_equal(m, np.tile((ref > 5.0).astype(np.uint8), F))
    m2, _, tau2 = mc.token_mask_frames(src, edit, prune_quantile=0.7)
    assert m2.reshape(F, N).sum(axis=1).tolist() == [N - math.ceil(0.7 * N)] * F
    # a one-frame chunk is the per-token mask
    m1, d1, _ = mc.token_mask_frames(src[:1], edit[:1], tau=3.0)
    t1, e1, _ = mc.token_mask(src[0], edit[0], tau=3.0)
    assert np.array_equal(m1, t1) and np.allclose(d1, e1, rtol=1e-15, atol=0)
