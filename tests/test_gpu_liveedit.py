"""GPU parity on the LiveEdit-shaped workload: chunks of 3 latent frames (4860
tokens of the 30x54 grid), 4 denoising steps, the mask cache over a multi-frame
chunk ["LiveEdit 실시간 Diffusion 기반 스트리밍 비디오 편집", 기술 상세].

Bars: bit-exact mask (one decision per position, written for every frame) and
compaction; attention within max-abs 2e-2 (beyond bf16 output rounding) and
relative L2 1e-2 of the fp64 oracle on sampled query rows, which the oracle
computes one by one over all 19440 visible keys; inactive cache rows bitwise
unchanged.
"""

import numpy as np
import pytest
import torch

import chunk_causal_attention_b200 as cca
from oracle import chunk_attention as oca
from oracle import mask_cache as omask
import synth

from test_gpu_parity import _record_errors, assert_attn_close, bf, check_status, dev, to_np  # noqa: F401

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def le():
    return synth.liveedit_chunk(n_steps=2)


@pytest.fixture(scope="module")
def le_ring(le):
    ring = cca.KVRing(le.n_heads, le.head_dim, le.chunk_len, le.window, device=dev())
    for t in range(le.t):
        ring.append(bf(le.ring_k[t]), bf(le.ring_v[t]))
    return ring


def _ambiguity_guard(d2_ref, tau2, rel=1e-5):
    assert np.all(np.abs(d2_ref - tau2) > rel * max(tau2, 1e-30)), "seeded input too close to tau"


def test_mask_frames_dynamic_tau_bit_exact(le):
    src, edit = torch.from_numpy(le.src).to(dev()), torch.from_numpy(le.edit).to(dev())
    dist2 = torch.empty(src.shape[1], dtype=torch.float32, device=dev())
    tau = torch.empty(1, dtype=torch.float32, device=dev())
    m = cca.cca_token_mask_l2_frames(src, edit, prune_quantile=le.prune_quantile, dist2=dist2, tau_out=tau)
    ref, d, tau_ref = omask.token_mask_frames(le.src, le.edit, prune_quantile=le.prune_quantile)
    d2 = np.sort(d * d)
    k = omask.prune_count(len(d), le.prune_quantile)
    # the k-th and (k+1)-th distances are apart by more than fp32 can blur, so
    # the fp32 order statistic splits the tokens exactly as the fp64 one
    assert (d2[k] - d2[k - 1]) > 1e-5 * d2[k - 1]
    torch.cuda.synchronize()
    assert np.array_equal(m.cpu().numpy(), ref)
    assert abs(tau.item() - tau_ref) <= 1e-5 * tau_ref
    assert int(ref.sum()) == le.n_frames * (src.shape[1] - k)


@pytest.mark.parametrize("F,N,C,tau", [(3, 1620, 16, 7.0), (2, 777, 4, 1.5), (1, 300, 8, 2.0), (5, 33, 12, 3.0)])
def test_mask_frames_fixed_tau_bit_exact(F, N, C, tau):
    g = np.random.default_rng(80 + F)
    src = g.standard_normal((F, N, C)).astype(np.float32)
    edit = (src + g.normal(0, 1, (F, N, C))).astype(np.float32)
    m = cca.cca_token_mask_l2_frames(torch.from_numpy(src).to(dev()), torch.from_numpy(edit).to(dev()), tau=tau)
    ref, d, _ = omask.token_mask_frames(src, edit, tau=tau)
    _ambiguity_guard(d * d, tau * tau)
    torch.cuda.synchronize()
    assert np.array_equal(m.cpu().numpy(), ref)


def test_liveedit_full_chunk_attention_sampled_rows(le, le_ring):
    g = np.random.default_rng(81)
    past_k = {c: le.ring_k[c] for c in range(le.t)}
    past_v = {c: le.ring_v[c] for c in range(le.t)}
    for s in range(2):
        o = to_np(cca.cca_chunk_attn(le_ring, bf(le.q[s]), bf(le.k_cur[s]), bf(le.v_cur[s])))
        pick = np.unique(np.concatenate([[0, 1619, 1620, 4859], g.integers(0, le.chunk_len, 60)]))
        ref = oca.chunk_attention(le.q[s][pick], past_k, past_v, le.t, le.window, k_cur=le.k_cur[s],
                                  v_cur=le.v_cur[s])
        assert_attn_close(o[pick], ref, what=f"liveedit step {s}")
    check_status(le_ring)


def test_liveedit_mask_cached_chunk_end_to_end(le, le_ring):
    """mask over the 3-frame chunk -> compaction of its 4860 tokens -> active
    queries with the scatter-back fused -> cache: active rows recomputed, the
    rest bitwise unchanged."""
    src, edit = torch.from_numpy(le.src).to(dev()), torch.from_numpy(le.edit).to(dev())
    m = cca.cca_token_mask_l2_frames(src, edit, prune_quantile=le.prune_quantile)
    idx, n = cca.cca_compact(m)
    cache = bf(le.o_cache)
    before = cache.clone()
    cca.cca_chunk_attn_scatter(le_ring, bf(le.q[0]), bf(le.k_cur[0]), bf(le.v_cur[0]), idx, cache, n_q_dev=n,
                               n_q_max=le.chunk_len)
    torch.cuda.synchronize()
    mref, _, _ = omask.token_mask_frames(le.src, le.edit, prune_quantile=le.prune_quantile)
    idx_ref, n_ref = omask.compact(mref)
    assert int(n.item()) == n_ref and np.array_equal(idx[:n_ref].cpu().numpy(), idx_ref)
    got = to_np(cache)
    inactive = np.flatnonzero(mref == 0)
    assert torch.equal(cache[torch.from_numpy(inactive).to(dev())], before[torch.from_numpy(inactive).to(dev())])
    g = np.random.default_rng(82)
    pick = np.unique(np.concatenate([idx_ref[:3], idx_ref[-3:], g.choice(idx_ref, 50, replace=False)]))
    ref = oca.chunk_attention(le.q[0][pick], {c: le.ring_k[c] for c in range(le.t)},
                              {c: le.ring_v[c] for c in range(le.t)}, le.t, le.window, k_cur=le.k_cur[0],
                              v_cur=le.v_cur[0])
    assert_attn_close(got[pick], ref, what="liveedit mask-cached rows")
    check_status(le_ring)
