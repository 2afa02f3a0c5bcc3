"""GPU parity of the token-group step (cca_chunk_attn_groups) and the packed
block-causal forward (cca_block_attn) against the fp64 oracle
(``oracle.token_groups``, an explicit element mask over group labels).

Bars as for the other attention calls: max-abs 2e-2 on top of the bf16 output
rounding and relative L2 1e-2 (BF16), 6e-2 / 3e-2 against the
quantisation-aware oracle (e4m3).  Shapes span several 128-row tiles with
ragged tails; the 720p cases compare sampled query rows, which the oracle
computes one by one over all their keys.
"""

import numpy as np
import pytest
import torch

import chunk_causal_attention_b200 as cca
from oracle import chunk_attention as oca
from oracle import fp8 as ofp8
from oracle import token_groups as otg
import synth

from test_gpu_parity import (BF16_MAX_ABS, BF16_REL_L2, FP8_MAX_ABS, FP8_REL_L2, _record_errors,  # noqa: F401
                             assert_attn_close, bf, check_status, dev, to_np)

pytestmark = pytest.mark.gpu


def _ring(n_heads, head_dim, chunk_len, window, ks, vs, dtype="bf16"):
    ring = cca.KVRing(n_heads, head_dim, chunk_len, window, dtype=dtype, device=dev())
    for k, v in zip(ks, vs):
        ring.append(bf(k), bf(v))
    return ring


def _packed(groups, order=("N", "S", "C")):
    names = [n for n in order if n in groups]
    return names, [np.concatenate([groups[n][i] for n in names]) for i in range(3)]


# ------------------------------------------------------------------ token groups (one step)
@pytest.mark.parametrize("D,L,H,W,n_src,n_cond,n_ref,t", [
    (128, 300, 2, 2, 300, 77, 150, 4),   # all groups, window evicting chunk 1
    (64, 200, 3, 1, 129, 1, 0, 3),       # no reference group
    (128, 130, 1, 3, 0, 0, 257, 2),      # N and R only, window reaching the sink
    (128, 100, 2, 2, 50, 13, 33, 0),     # first chunk: no history at all
])
def test_groups_step_ragged(D, L, H, W, n_src, n_cond, n_ref, t):
    s = synth.groups_chunk(seed=50 + t, n_heads=H, head_dim=D, chunk_len=L, window=W, n_prefill=t, n_src=n_src,
                           n_cond=n_cond, n_ref=n_ref)
    ring = _ring(H, D, L, W, s.ring_k, s.ring_v)
    names, (q, k, v) = _packed(s.groups)
    kr = vr = None
    if s.ref is not None:
        kr, vr = bf(s.ref[1]), bf(s.ref[2])
    o = cca.cca_chunk_attn_groups(ring, bf(q), bf(k), bf(v), k_ref=kr, v_ref=vr)
    hist = {c: (s.ring_k[c], s.ring_v[c]) for c in range(t)}
    ref = otg.step_attention(t, W, [(n, *s.groups[n]) for n in names], hist, ref=s.ref)
    assert_attn_close(to_np(o), ref, what=f"groups D{D} L{L} H{H} W{W} t{t}")
    check_status(ring)


def test_groups_step_720p_sampled_rows():
    s = synth.groups_chunk()
    ring = _ring(s.n_heads, s.head_dim, s.chunk_len, s.window, s.ring_k, s.ring_v)
    names, (q, k, v) = _packed(s.groups)
    o = to_np(cca.cca_chunk_attn_groups(ring, bf(q), bf(k), bf(v), k_ref=bf(s.ref[1]), v_ref=bf(s.ref[2])))
    # sampled rows of every group (its tile boundaries and tails included)
    g = np.random.default_rng(51)
    hist = {c: (s.ring_k[c], s.ring_v[c]) for c in range(s.t)}
    active, rows = [], []
    base = 0
    for n in names:
        gq, gk, gv = s.groups[n]
        pick = np.unique(np.concatenate([[0, 127, 128, len(gq) - 1], g.integers(0, len(gq), 40)]))
        active.append((n, gq[pick], gk, gv))
        rows.append(base + pick)
        base += len(gq)
    ref = otg.step_attention(s.t, s.window, active, hist, ref=s.ref)
    assert_attn_close(o[np.concatenate(rows)], ref, what="groups 720p sampled")
    check_status(ring)


def test_groups_without_extra_groups_equal_chunk_attention():
    """N_t alone and no R: the same call as cca_chunk_attn, bit for bit."""
    s = synth.chunk_720p(n_steps=1)
    ring = _ring(s.n_heads, s.head_dim, s.chunk_len, s.window, s.ring_k, s.ring_v)
    q, k, v = bf(s.q[0]), bf(s.k_cur[0]), bf(s.v_cur[0])
    a = cca.cca_chunk_attn(ring, q, k, v)
    b = cca.cca_chunk_attn_groups(ring, q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_groups_step_e4m3():
    H, D, L, W, t = 2, 128, 200, 2, 3
    s = synth.groups_chunk(seed=55, n_heads=H, head_dim=D, chunk_len=L, window=W, n_prefill=t, n_src=150,
                           n_cond=40, n_ref=90)
    ring = _ring(H, D, L, W, s.ring_k, s.ring_v, dtype="e4m3")
    names, (q, k, v) = _packed(s.groups)
    q8, qs = cca.cca_quant_e4m3(bf(q))
    k8, ks = cca.cca_quant_e4m3(bf(k))
    v8, vs = cca.cca_quant_e4m3_f16(bf(v))
    kr8, krs = cca.cca_quant_e4m3(bf(s.ref[1]))
    vr8, vrs = cca.cca_quant_e4m3_f16(bf(s.ref[2]))
    o = cca.cca_chunk_attn_groups(ring, q8, k8, v8, k_ref=kr8, v_ref=vr8, q_scale=qs, kcur_scale=ks, vcur_scale=vs,
                                  kref_scale=krs, vref_scale=vrs)
    deq = lambda x: ofp8.dequantize_per_head(*ofp8.quantize_per_head(x))
    # the packed block is quantised as one tensor (per head over all its rows)
    qd, kd, vd = deq(q), deq(k), deq(v)
    hist = {c: (deq(s.ring_k[c]), deq(s.ring_v[c])) for c in range(t)}
    ref = otg.step_attention(t, W, [("N", qd, kd, vd)], hist,
                             ref=(deq(s.ref[0]), deq(s.ref[1]), deq(s.ref[2])))
    assert_attn_close(to_np(o), ref, FP8_MAX_ABS, FP8_REL_L2, what="groups e4m3")
    check_status(ring)


# ------------------------------------------------------------------ packed block-causal forward
@pytest.mark.parametrize("T,L,H,D,W,n_ref,same", [
    (6, 200, 2, 128, 2, 0, False),   # clean history and noisy chunks differ
    (5, 129, 1, 64, 4, 0, True),     # plain block-causal (full window)
    (4, 100, 2, 128, 1, 77, False),  # with a reference group
    (40, 20, 1, 64, 3, 0, False),    # more chunks than one launch holds
])
def test_block_attn_ragged(T, L, H, D, W, n_ref, same):
    p = synth.packed_sequence(seed=60 + T, n_chunks=T, n_heads=H, head_dim=D, chunk_len=L, window=W)
    kh, vh = (p.k_cur, p.v_cur) if same else (p.k_hist, p.v_hist)
    ref_t = None
    if n_ref:
        g = np.random.default_rng(61)
        ref_t = tuple(synth.bf16_round(g.standard_normal((n_ref, H, D)).astype(np.float32)) for _ in range(3))
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    o = cca.cca_block_attn(bf(p.q), bf(p.k_cur), bf(p.v_cur), W,
                           k_hist=None if same else bf(kh), v_hist=None if same else bf(vh),
                           k_ref=bf(ref_t[1]) if ref_t else None, v_ref=bf(ref_t[2]) if ref_t else None,
                           status=status)
    want = otg.packed_forward(p.q, p.k_cur, p.v_cur, kh, vh, W, ref=ref_t)
    got = to_np(o)
    for c in range(T):
        assert_attn_close(got[c], want[c], what=f"block T{T} L{L} W{W} chunk {c}")
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_block_attn_ref_self_attention():
    """R's own queries (see R only) as a one-chunk call without history."""
    g = np.random.default_rng(62)
    R = [synth.bf16_round(g.standard_normal((300, 2, 128)).astype(np.float32)) for _ in range(3)]
    o = cca.cca_block_attn(bf(R[0])[None], bf(R[1])[None], bf(R[2])[None], 0)
    assert_attn_close(to_np(o)[0], otg.ref_self_attention(*R), what="R self")


def test_block_attn_720p_sampled_rows():
    p = synth.packed_sequence()
    T = p.q.shape[0]
    o = to_np(cca.cca_block_attn(bf(p.q), bf(p.k_cur), bf(p.v_cur), p.window, k_hist=bf(p.k_hist),
                                 v_hist=bf(p.v_hist)))
    g = np.random.default_rng(63)
    L = p.q.shape[1]
    for c in range(T):
        pick = np.unique(np.concatenate([[0, 255, 256, L - 1], g.integers(0, L, 24)]))
        want = oca.chunk_attention(p.q[c][pick], list(p.k_hist), list(p.v_hist), c, p.window,
                                   k_cur=p.k_cur[c], v_cur=p.v_cur[c])
        assert_attn_close(o[c][pick], want, what=f"block 720p chunk {c}")


def test_block_attn_e4m3():
    T, L, H, D, W = 5, 160, 2, 128, 2
    p = synth.packed_sequence(seed=64, n_chunks=T, n_heads=H, head_dim=D, chunk_len=L, window=W, heavy_tailed=True)
    qz = [cca.cca_quant_e4m3(bf(p.q[c])) for c in range(T)]
    kz = [cca.cca_quant_e4m3(bf(p.k_cur[c])) for c in range(T)]
    vz = [cca.cca_quant_e4m3_f16(bf(p.v_cur[c])) for c in range(T)]
    khz = [cca.cca_quant_e4m3(bf(p.k_hist[c])) for c in range(T)]
    vhz = [cca.cca_quant_e4m3_f16(bf(p.v_hist[c])) for c in range(T)]
    st = lambda z, i: torch.stack([x[i] for x in z]).contiguous()
    o = cca.cca_block_attn(st(qz, 0), st(kz, 0), st(vz, 0), W, k_hist=st(khz, 0), v_hist=st(vhz, 0),
                           q_scale=st(qz, 1), kcur_scale=st(kz, 1), vcur_scale=st(vz, 1), khist_scale=st(khz, 1),
                           vhist_scale=st(vhz, 1))
    deq = lambda x: ofp8.dequantize_per_head(*ofp8.quantize_per_head(x))
    dq = lambda a: np.stack([deq(x) for x in a])
    want = otg.packed_forward(dq(p.q), dq(p.k_cur), dq(p.v_cur), dq(p.k_hist), dq(p.v_hist), W)
    got = to_np(o)
    for c in range(T):
        assert_attn_close(got[c], want[c], FP8_MAX_ABS, FP8_REL_L2, what=f"block e4m3 chunk {c}")


def test_block_attn_future_chunks_never_read():
    """Chunk c's output is bitwise unchanged when chunks > c hold NaN."""
    T, L, H, D, W = 6, 140, 2, 128, 2
    p = synth.packed_sequence(seed=65, n_chunks=T, n_heads=H, head_dim=D, chunk_len=L, window=W)
    args = [bf(x) for x in (p.q, p.k_cur, p.v_cur, p.k_hist, p.v_hist)]
    a = cca.cca_block_attn(args[0], args[1], args[2], W, k_hist=args[3], v_hist=args[4]).clone()
    for x in args[1:]:
        x[4:] = float("nan")
    b = cca.cca_block_attn(args[0], args[1], args[2], W, k_hist=args[3], v_hist=args[4])
    torch.cuda.synchronize()
    assert torch.equal(a[:4], b[:4])
