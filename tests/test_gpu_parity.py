"""GPU parity: every kernel of libcca.so against the fp64 oracle.

Bars: bit-exact for the KV ring contents, e4m3 codes/scales, the mask,
compaction indices and scatter; attention within max-abs 2e-2 and relative L2
1e-2 (BF16) or 6e-2 / 3e-2 (e4m3) of the oracle run on the same inputs.  The
output is bf16, so the max-abs bar is applied on top of the rounding to that
format (half a bf16 ulp at the oracle's value): at |O| >= 16 that rounding alone
is 0.0625, above the e4m3 bar, and no bf16 output could meet the bar without it.
"""

import math
import os

import numpy as np
import pytest
import torch

import chunk_causal_attention_b200 as cca
from oracle import chunk_attention as oca
from oracle import fp8 as ofp8
from oracle import kv_ring as oring
from oracle import mask_cache as omask
import synth

pytestmark = pytest.mark.gpu

BF16_MAX_ABS, BF16_REL_L2 = 2e-2, 1e-2
FP8_MAX_ABS, FP8_REL_L2 = 6e-2, 3e-2


def dev():
    return torch.device("cuda:0")


def bf(x):
    return synth.as_torch_bf16(x, dev())


def err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    d = got - ref
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))


def half_ulp_bf16(x):
    """Half a unit in the last place of bf16 at |x| (8-bit significand): the
    rounding error any bf16 output of the exact value may carry."""
    a = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    _, e = np.frexp(a)  # a = m 2^e, m in [0.5, 1)
    return np.ldexp(1.0, e - 1 - 8)


_RECORD = None


@pytest.fixture(autouse=True)
def _record_errors(record_property):
    """Every attention comparison records its raw errors (junit properties, and
    one JSON line per comparison in $CCA_PARITY_LOG when that is set)."""
    global _RECORD
    _RECORD = record_property
    yield
    _RECORD = None


def _log_errors(what, ma, excess, rl, max_abs, rel_l2):
    if _RECORD is not None:
        _RECORD(f"{what}|max_abs", ma)
        _RECORD(f"{what}|max_abs_beyond_bf16_rounding", excess)
        _RECORD(f"{what}|rel_l2", rl)
    path = os.environ.get("CCA_PARITY_LOG")
    if path:
        import json
        with open(path, "a") as f:
            f.write(json.dumps({"what": what, "max_abs": ma, "max_abs_beyond_bf16_rounding": excess,
                                "rel_l2": rl, "bar_max_abs": max_abs, "bar_rel_l2": rel_l2}) + "\n")


def assert_attn_close(got, ref, max_abs=BF16_MAX_ABS, rel_l2=BF16_REL_L2, what=""):
    """Element-wise |got - ref| <= max_abs on top of the bf16 output rounding
    (half an ulp of bf16 at |ref|), and relative L2 over the tensor <= rel_l2.
    The raw max-abs, the part beyond the output rounding and the relative L2
    are recorded for every call."""
    got = np.asarray(got, dtype=np.float64)
    d = np.abs(got - ref)
    excess = float((d - half_ulp_bf16(ref)).max())
    ma, rl = err(got, ref)
    _log_errors(what or "attention", ma, excess, rl, max_abs, rel_l2)
    assert excess <= max_abs and rl <= rel_l2, f"{what}: max_abs={ma:.3e} (beyond bf16 rounding {excess:.3e}) rel_l2={rl:.3e}"
    return ma, rl


def to_np(t):
    return t.float().cpu().numpy()


def check_status(ring):
    torch.cuda.synchronize()
    st = int(ring.status.item())
    assert st == cca.CCA_DEV_OK, f"device status {st}"


# ------------------------------------------------------------------ ring
def test_ring_append_bf16_bit_exact_with_eviction():
    s = synth.tiny(n_chunks=8)
    ring = cca.KVRing(s.n_heads, s.head_dim, s.chunk_len, s.window, device=dev())
    oracle = oring.KVRing(s.window)
    for t in range(8):
        ring.append(bf(s.k[t]), bf(s.v[t]))
        oracle.append(s.k[t], s.v[t])
        n, slots, ids = ring.query()
        assert n == t + 1 and ids == oracle.chunks()
        torch.cuda.synchronize()
        for sl, c in zip(slots, ids):
            assert torch.equal(ring.k_slots[sl].cpu(), bf(oracle.get(c)[0]).cpu())
            assert torch.equal(ring.v_slots[sl].cpu(), bf(oracle.get(c)[1]).cpu())
    check_status(ring)


def test_ring_append_f32_source_rounds_to_nearest_even():
    g = np.random.default_rng(5)
    x = g.standard_normal((16, 2, 64)).astype(np.float32)
    ring = cca.KVRing(2, 64, 16, 1, device=dev())
    ring.append(torch.from_numpy(x).to(dev()), torch.from_numpy(-x).to(dev()))
    torch.cuda.synchronize()
    assert torch.equal(ring.k_slots[0].cpu(), torch.from_numpy(x).to(torch.bfloat16))
    assert torch.equal(ring.v_slots[0].cpu(), torch.from_numpy(-x).to(torch.bfloat16))


# ------------------------------------------------------------------ fp8
@pytest.mark.parametrize("src_dtype", [torch.bfloat16, torch.float32])
def test_quant_e4m3_bit_exact(src_dtype):
    g = np.random.default_rng(6)
    x = g.standard_t(4.0, size=(1620, 24, 128)).astype(np.float32)
    x[:, 3] = 0.0  # an all-zero head -> scale 1
    x[5, 7, 9] = -0.0
    if src_dtype == torch.bfloat16:
        x = synth.bf16_round(x)
    xt = torch.from_numpy(x).to(dev()).to(src_dtype)
    codes, scale = cca.cca_quant_e4m3(xt)
    ref_codes, ref_scale = ofp8.quantize_per_head(x)
    torch.cuda.synchronize()
    assert np.array_equal(scale.cpu().numpy(), ref_scale)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)


@pytest.mark.parametrize(
    "n_tok,H,D,src_dtype",
    [
        (7, 3, 64, torch.bfloat16),  # fewer tokens than the CTAs of a head's cluster
        (6400, 2, 128, torch.bfloat16),  # 800 rows of 256 B per CTA: the largest shared-memory staging
        (6408, 2, 128, torch.bfloat16),  # 801 rows: streamed from global memory twice
        (3201, 2, 128, torch.float32),  # fp32 rows of 512 B: streamed
        (3200, 3, 64, torch.float32),
    ],
)
def test_quant_e4m3_staged_and_streamed_sizes(n_tok, H, D, src_dtype):
    g = np.random.default_rng(n_tok + H)
    x = g.standard_t(3.0, size=(n_tok, H, D)).astype(np.float32)
    x[n_tok // 2, H - 1, D - 1] = 900.0  # the absmax sits in one CTA's rows only
    if src_dtype == torch.bfloat16:
        x = synth.bf16_round(x)
    xt = torch.from_numpy(x).to(dev()).to(src_dtype)
    codes, scale = cca.cca_quant_e4m3(xt)
    x16, scale16 = cca.cca_quant_e4m3_f16(xt)
    ref_codes, ref_scale = ofp8.quantize_per_head(x)
    torch.cuda.synchronize()
    assert np.array_equal(scale.cpu().numpy(), ref_scale)
    assert np.array_equal(scale16.cpu().numpy(), ref_scale)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    assert np.array_equal(x16.cpu().numpy(), ofp8.e4m3_decode(ref_codes).astype(np.float16))


def _boundary_head(s0, n_tok, D, g):
    """One head whose quotients x / s sit on and next to every e4m3 rounding
    boundary (midpoints between neighbouring codes) and every code value, up to
    4 units in the last place away, both signs; the absmax fixes s."""
    a = np.float32(448.0 * s0)
    s = np.float32(a / np.float32(448.0))
    vals = ofp8.e4m3_decode(np.arange(127, dtype=np.uint8))
    pts = np.concatenate([(vals[:-1] + vals[1:]) / 2.0, vals])
    xs = []
    for m in pts:
        x = np.float32(m * np.float64(s))
        for k in range(-4, 5):
            y = x
            for _ in range(abs(k)):
                y = np.nextafter(y, np.float32(np.inf if k > 0 else -np.inf), dtype=np.float32)
            xs += [y, -y]
    xs = np.array(xs, dtype=np.float32)
    xs = xs[np.abs(xs) <= a]
    head = (g.standard_normal(n_tok * D) * float(s)).astype(np.float32)
    head = np.clip(head, -a, a)
    head[: len(xs)] = xs
    head[len(xs)] = a
    g.shuffle(head)
    return head.reshape(n_tok, D)


def test_quant_e4m3_quotients_next_to_rounding_boundaries():
    # A quantiser that multiplies by a rounded reciprocal instead of dividing
    # disagrees with the fp32 division on about 1 % of these values.
    g = np.random.default_rng(11)
    n_tok, D = 48, 128
    scales = [3.0, 0.7, 1e-3 * np.pi, 12345.678, 1.0 / 3.0, 7.1e-5]
    x = np.stack([_boundary_head(s0, n_tok, D, g) for s0 in scales], axis=1)  # [n_tok][H][D] fp32
    xt = torch.from_numpy(x).to(dev())
    codes, scale = cca.cca_quant_e4m3(xt)
    x16, _ = cca.cca_quant_e4m3_f16(xt)
    ref_codes, ref_scale = ofp8.quantize_per_head(x)
    torch.cuda.synchronize()
    assert np.array_equal(scale.cpu().numpy(), ref_scale)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    assert np.array_equal(x16.cpu().numpy(), ofp8.e4m3_decode(ref_codes).astype(np.float16))


@pytest.mark.parametrize("n_tok,H,D,src_dtype", [(1620, 24, 128, torch.bfloat16), (301, 3, 64, torch.float32)])
def test_quant_e4m3_qkv_equals_three_quantisations(n_tok, H, D, src_dtype):
    g = np.random.default_rng(n_tok)
    xs = [g.standard_t(4.0, size=(n_tok, H, D)).astype(np.float32) * sc for sc in (1.0, 30.0, 1e-3)]
    xs[1][:, H - 1] = 0.0  # an all-zero head of K -> scale 1
    if src_dtype == torch.bfloat16:
        xs = [synth.bf16_round(x) for x in xs]
    q8, qs, k8, ks, v16, vs = cca.cca_quant_e4m3_qkv(*(torch.from_numpy(x).to(dev()).to(src_dtype) for x in xs))
    refs = [ofp8.quantize_per_head(x) for x in xs]
    torch.cuda.synchronize()
    for (codes, scale), (rc, rs) in zip(((q8, qs), (k8, ks)), refs[:2]):
        assert np.array_equal(scale.cpu().numpy(), rs)
        assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(vs.cpu().numpy(), refs[2][1])
    assert np.array_equal(v16.cpu().numpy(), ofp8.e4m3_decode(refs[2][0]).astype(np.float16))


def test_quant_e4m3_f16_widens_the_codes_exactly():
    g = np.random.default_rng(7)
    x = synth.bf16_round(g.standard_t(4.0, size=(777, 5, 128)).astype(np.float32))
    x[:, 2] = 0.0
    x16, scale = cca.cca_quant_e4m3_f16(synth.as_torch_bf16(x, dev()))
    ref_codes, ref_scale = ofp8.quantize_per_head(x)
    torch.cuda.synchronize()
    assert np.array_equal(scale.cpu().numpy(), ref_scale)
    assert np.array_equal(x16.cpu().numpy(), ofp8.e4m3_decode(ref_codes).astype(np.float16))


def test_ring_append_e4m3_bit_exact():
    s = synth.fp8_720p(n_steps=1, n_prefill=5)
    ring = cca.KVRing(s.n_heads, s.head_dim, s.chunk_len, s.window, dtype="e4m3", device=dev())
    for t in range(5):
        ring.append(bf(s.ring_k[t]), bf(s.ring_v[t]))
    n, slots, ids = ring.query()
    assert ids == [0, 2, 3, 4]
    torch.cuda.synchronize()
    for sl, c in zip(slots, ids):
        kc, ks = ofp8.quantize_per_head(s.ring_k[c])
        vc, vs = ofp8.quantize_per_head(s.ring_v[c])
        assert np.array_equal(ring.k_slots[sl].cpu().numpy(), kc)
        # V is stored as the codes' values widened to fp16 (exact)
        assert np.array_equal(ring.v_slots[sl].cpu().numpy(), ofp8.e4m3_decode(vc).astype(np.float16))
        assert np.array_equal(ring.k_scale[sl].cpu().numpy(), ks)
        assert np.array_equal(ring.v_scale[sl].cpu().numpy(), vs)


# ------------------------------------------------------------------ mask / compact / scatter
def _ambiguity_guard(d2_ref, tau2, rel=1e-5):
    assert np.all(np.abs(d2_ref - tau2) > rel * max(tau2, 1e-30)), "seeded input too close to tau"


def test_mask_fixed_tau_tiny_bit_exact():
    s = synth.tiny()
    m_ref, d_ref, tau = omask.token_mask(s.src, s.edit, tau=s.tau)
    _ambiguity_guard(d_ref ** 2, tau ** 2)
    src, edit = torch.from_numpy(s.src).to(dev()), torch.from_numpy(s.edit).to(dev())
    d2 = torch.empty(16, dtype=torch.float32, device=dev())
    mask = cca.cca_token_mask_l2(src, edit, tau=s.tau, dist2=d2)
    torch.cuda.synchronize()
    assert np.array_equal(mask.cpu().numpy(), m_ref)
    assert 0 < m_ref.sum() < 16
    assert np.allclose(d2.cpu().numpy(), d_ref ** 2, rtol=1e-6)


@pytest.mark.parametrize("n_tok,n_ch", [(0, 16), (1, 4), (1621, 4), (777, 64), (300, 256)])
def test_mask_fixed_tau_channel_counts(n_tok, n_ch):
    """Fixed-tau mask for every supported channel count class and ragged token
    counts (0 included), against the oracle, with the ambiguity guard."""
    g = np.random.default_rng(n_tok * 7 + n_ch)
    src = g.standard_normal((n_tok, n_ch)).astype(np.float32)
    edit = (src + g.normal(0.0, 0.5, size=(n_tok, n_ch))).astype(np.float32)
    tau = float(np.sqrt(0.25 * n_ch)) * 1.01
    m_ref, d_ref, _ = omask.token_mask(src, edit, tau=tau)
    if n_tok:
        _ambiguity_guard(d_ref ** 2, tau ** 2)
    mask = torch.full((max(n_tok, 1),), 9, dtype=torch.uint8, device=dev())[:n_tok]
    cca.cca_token_mask_l2(torch.from_numpy(src).to(dev()), torch.from_numpy(edit).to(dev()), tau=tau, mask=mask)
    idx, n = cca.cca_compact(mask)
    torch.cuda.synchronize()
    assert np.array_equal(mask.cpu().numpy(), m_ref)
    assert n.item() == int(m_ref.sum())


def test_mask_identical_latents_all_inactive():
    s = synth.tiny()
    src = torch.from_numpy(s.src).to(dev())
    mask = cca.cca_token_mask_l2(src, src.clone(), tau=0.0)
    idx, n = cca.cca_compact(mask)
    torch.cuda.synchronize()
    assert mask.sum().item() == 0 and n.item() == 0


@pytest.mark.parametrize("n_tok", [1, 2, 255, 256, 1620, 4097, 32768])
@pytest.mark.parametrize("q", [0.01, 0.5, 0.7, 1.0])
def test_mask_dynamic_tau_with_ties(n_tok, q):
    """Integer-valued latents make every d^2 an exact small integer in both
    precisions, with many ties at the threshold: the kernel's order statistic
    and strict-greater mask must equal the oracle's exactly (ties at tau stay
    inactive; q = 1 leaves every token inactive)."""
    g = np.random.default_rng(1000 + n_tok)
    src = np.zeros((n_tok, 16), dtype=np.float32)
    edit = g.integers(0, 3, size=(n_tok, 16)).astype(np.float32) * (g.random((n_tok, 1)) < 0.8)
    q32 = float(np.float32(q))  # the kernel receives q as fp32
    m_ref, _, tau = omask.token_mask(src, edit, prune_quantile=q32)
    tau_out = torch.empty(1, dtype=torch.float32, device=dev())
    mask = cca.cca_token_mask_l2(torch.from_numpy(src).to(dev()), torch.from_numpy(edit).to(dev()),
                                 prune_quantile=q32, tau_out=tau_out)
    torch.cuda.synchronize()
    assert np.array_equal(mask.cpu().numpy(), m_ref)
    assert tau_out.item() == np.float32(tau)
    if q == 1.0:
        assert m_ref.sum() == 0


def test_mask_dynamic_tau_and_compaction_bit_exact():
    m = synth.mask_chunk()
    m_ref, d_ref, tau = omask.token_mask(m.src, m.edit, prune_quantile=m.prune_quantile)
    d2s = np.sort(d_ref ** 2)
    k = omask.prune_count(len(d_ref), m.prune_quantile)
    assert (d2s[k] - d2s[k - 1]) > 1e-5 * d2s[k - 1], "order statistic gap too small for fp32"
    src, edit = torch.from_numpy(m.src).to(dev()), torch.from_numpy(m.edit).to(dev())
    tau_out = torch.empty(1, dtype=torch.float32, device=dev())
    mask = cca.cca_token_mask_l2(src, edit, prune_quantile=m.prune_quantile, tau_out=tau_out)
    idx, n = cca.cca_compact(mask)
    torch.cuda.synchronize()
    assert np.array_equal(mask.cpu().numpy(), m_ref)
    assert n.item() == 486 == len(d_ref) - k
    ref_idx, ref_n = omask.compact(m_ref)
    assert np.array_equal(idx[:n.item()].cpu().numpy(), ref_idx)
    assert abs(tau_out.item() - tau) <= 1e-5 * tau


@pytest.mark.parametrize("n_tok,p", [(0, 0.5), (1, 0.5), (17, 0.3), (16384, 0.05), (16385, 0.9), (65536, 0.3),
                                     (65537, 0.3), (100000, 0.3), (8192 * 37 + 5, 0.5), (8192 * 1000, 0.0),
                                     (8192 * 1000 + 1, 1.0), ((1 << 22) + 3, 0.01), ((1 << 26) + 17, 0.3)])
def test_compaction_ragged_sizes(n_tok, p):
    """Both paths (one CTA up to 65536 tokens, look-back scan above) against the
    oracle on small sizes and against the closed form flatnonzero on all."""
    g = np.random.default_rng(n_tok)
    m = (g.random(n_tok) < p).astype(np.uint8)
    mt = torch.from_numpy(m).to(dev())
    idx, n = cca.cca_compact(mt)
    torch.cuda.synchronize()
    want = np.flatnonzero(m).astype(np.int32)
    assert n.item() == want.shape[0]
    assert np.array_equal(idx[:n.item()].cpu().numpy(), want)
    if n_tok <= 200000:
        ref_idx, ref_n = omask.compact(m)
        assert ref_n == n.item() and np.array_equal(ref_idx, want)
    # a second call reuses the same workspace: its status words are re-zeroed
    ws = torch.full((max(cca.cca_compact_workspace_size(n_tok), 16),), 0xFF, dtype=torch.uint8, device=dev())
    idx2, n2 = cca.cca_compact(mt, workspace=ws)
    idx3, n3 = cca.cca_compact(mt, workspace=ws)
    torch.cuda.synchronize()
    assert n2.item() == n3.item() == want.shape[0]
    assert torch.equal(idx2[:n2.item()], idx[:n.item()]) and torch.equal(idx3[:n3.item()], idx[:n.item()])


@pytest.mark.parametrize("ctas", ["2", "8", "64"])
def test_compaction_long_and_short_runs(ctas, monkeypatch):
    """Few CTAs give each a long run of 8192-token sub-tiles: up to 16 sub-tiles
    a CTA keeps its activity bits between the passes, beyond that it reads the
    mask again in the second pass.  (2^20 + 77 tokens: runs of 65, 17 and 3.)"""
    monkeypatch.setenv("CCA_COMPACT_CTAS", ctas)
    n_tok = (1 << 20) + 77
    g = np.random.default_rng(int(ctas))
    m = (g.random(n_tok) < 0.37).astype(np.uint8)
    m[-77:] = 1  # an active ragged tail
    idx, n = cca.cca_compact(torch.from_numpy(m).to(dev()))
    torch.cuda.synchronize()
    want = np.flatnonzero(m).astype(np.int32)
    assert n.item() == want.shape[0]
    assert np.array_equal(idx[:n.item()].cpu().numpy(), want)


@pytest.mark.parametrize("shift", [1, 2, 3])
@pytest.mark.parametrize("p", [0.3, 1.0])
def test_compaction_index_array_at_any_4_byte_offset(shift, p):
    """The write pass stores 16-byte groups where the index array allows: an
    array that starts 4, 8 or 12 bytes past a 16-byte boundary, and warps whose
    1024 tokens are all active (a run too long to shift onto the boundary),
    still give exactly the list of active positions, and nothing outside it is
    written."""
    n_tok = (1 << 20) + 77
    g = np.random.default_rng(100 + shift)
    m = (g.random(n_tok) < p).astype(np.uint8)
    buf = torch.full((n_tok + 8,), -7, dtype=torch.int32, device=dev())
    idx = buf[shift:shift + n_tok]
    _, n = cca.cca_compact(torch.from_numpy(m).to(dev()), idx=idx)
    torch.cuda.synchronize()
    want = np.flatnonzero(m).astype(np.int32)
    got = buf.cpu().numpy()
    assert n.item() == want.shape[0]
    assert np.array_equal(got[shift:shift + want.shape[0]], want)
    assert np.all(got[:shift] == -7) and np.all(got[shift + want.shape[0]:] == -7)


@pytest.mark.parametrize("n_tok", [1000, 16385, 300007])
def test_compaction_counts_any_nonzero_byte(n_tok):
    """A token is active when its mask byte is nonzero, whatever the value."""
    g = np.random.default_rng(7 + n_tok)
    m = g.choice(np.array([0, 1, 2, 17, 128, 255], dtype=np.uint8), size=n_tok, p=[0.6, 0.1, 0.1, 0.1, 0.05, 0.05])
    idx, n = cca.cca_compact(torch.from_numpy(m).to(dev()))
    torch.cuda.synchronize()
    want = np.flatnonzero(m).astype(np.int32)
    ref_idx, ref_n = omask.compact(m)
    assert ref_n == n.item() == want.shape[0]
    assert np.array_equal(idx[:n.item()].cpu().numpy(), ref_idx)


def test_scatter_keeps_inactive_rows():
    g = np.random.default_rng(9)
    mask = (g.random(1620) < 0.3).astype(np.uint8)
    cache = synth.bf16_round(g.normal(0, 0.02, size=(1620, 24, 128)).astype(np.float32))
    ref_idx, ref_n = omask.compact(mask)
    oc = synth.bf16_round(g.standard_normal((ref_n, 24, 128)).astype(np.float32))
    mt = torch.from_numpy(mask).to(dev())
    idx, n = cca.cca_compact(mt)
    cache_t = bf(cache)
    cca.cca_scatter(bf(oc), idx, n, cache_t)
    torch.cuda.synchronize()
    expect = omask.scatter(oc, ref_idx, ref_n, cache)
    assert torch.equal(cache_t.cpu(), synth.as_torch_bf16(expect))
    # empty active set: cache untouched
    zero = torch.zeros(1, dtype=torch.int32, device=dev())
    before = cache_t.clone()
    cca.cca_scatter(bf(oc), idx, zero, cache_t)
    torch.cuda.synchronize()
    assert torch.equal(before, cache_t)


# ------------------------------------------------------------------ attention
def run_stream(s, n_chunks, window, ring=None):
    """Stream chunks 0..n-1: attention of chunk t (current K/V = chunk t) then append."""
    ring = ring or cca.KVRing(s.n_heads, s.head_dim, s.chunk_len, window, device=dev())
    outs = []
    for t in range(n_chunks):
        o = cca.cca_chunk_attn(ring, bf(s.q[t]), bf(s.k[t]), bf(s.v[t]))
        outs.append(to_np(o))
        ring.append(bf(s.k[t]), bf(s.v[t]))
    check_status(ring)
    return outs


@pytest.mark.parametrize("n_chunks", [4, 8])
def test_attention_tiny_stream(n_chunks):
    s = synth.tiny(n_chunks=n_chunks)
    outs = run_stream(s, n_chunks, s.window)
    for t in range(n_chunks):
        ref = oca.chunk_attention(s.q[t], s.k, s.v, t, s.window)
        assert_attn_close(outs[t], ref, what=f"tiny chunk {t}")


@pytest.mark.parametrize("D,L,H,W", [(64, 200, 3, 2), (128, 300, 2, 1), (128, 129, 1, 0), (64, 1, 2, 3),
                                     (64, 72, 2, 15)])
def test_attention_ragged_shapes(D, L, H, W):
    """Ragged chunk lengths, both head dims, no window, one-token chunks and the
    largest window (W = 15, 17 visible chunks) with eviction."""
    g = np.random.default_rng(D * 1000 + L)
    n = W + 3 if W < 15 else 20
    q = [synth.bf16_round(g.standard_normal((L, H, D)).astype(np.float32)) for _ in range(n)]
    k = [synth.bf16_round(g.standard_normal((L, H, D)).astype(np.float32)) for _ in range(n)]
    v = [synth.bf16_round(g.standard_normal((L, H, D)).astype(np.float32)) for _ in range(n)]
    s = synth.TinyStream(H, D, L, W, q, k, v, None, None, 0.0)
    outs = run_stream(s, n, W)
    for t in range(n):
        assert_attn_close(outs[t], oca.chunk_attention(q[t], k, v, t, W), what=f"D{D} L{L} t{t}")


@pytest.fixture(scope="module")
def c1():
    return synth.chunk_720p()


@pytest.fixture(scope="module")
def c1_ring(c1):
    ring = cca.KVRing(c1.n_heads, c1.head_dim, c1.chunk_len, c1.window, device=dev())
    for t in range(c1.t):
        ring.append(bf(c1.ring_k[t]), bf(c1.ring_v[t]))
    return ring


@pytest.fixture(scope="module")
def c1_ref(c1):
    return [oca.chunk_attention(c1.q[s], c1.ring_k, c1.ring_v, c1.t, c1.window, k_cur=c1.k_cur[s],
                                v_cur=c1.v_cur[s]) for s in range(len(c1.q))]


@pytest.mark.parametrize("ctas", ["auto", "37", "200"])
def test_attention_720p_two_steps(c1, c1_ring, c1_ref, ctas, monkeypatch):
    """Default grid (1 CTA per SM: 148 whole items + 20 split items), 37 CTAs
    (4 full rounds + 20 split items), 200 CTAs (more CTAs than items: all split)."""
    if ctas != "auto":
        monkeypatch.setenv("CCA_ATTN_CTAS", ctas)
    for s in range(len(c1.q)):
        o = cca.cca_chunk_attn(c1_ring, bf(c1.q[s]), bf(c1.k_cur[s]), bf(c1.v_cur[s]))
        assert_attn_close(to_np(o), c1_ref[s], what=f"720p step {s} ctas={ctas}")
    check_status(c1_ring)


def test_attention_720p_is_deterministic_and_bounded_memory(c1, c1_ring):
    a = cca.cca_chunk_attn(c1_ring, bf(c1.q[0]), bf(c1.k_cur[0]), bf(c1.v_cur[0]))
    b = cca.cca_chunk_attn(c1_ring, bf(c1.q[0]), bf(c1.k_cur[0]), bf(c1.v_cur[0]))
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_attention_future_chunks_never_read(c1):
    """Causality on the GPU: garbage in ring slots of evicted / not-yet-written
    chunks does not change the output (bitwise)."""
    ring = cca.KVRing(c1.n_heads, c1.head_dim, c1.chunk_len, 5, device=dev())
    ring.k_slots.fill_(float("nan"))
    ring.v_slots.fill_(float("nan"))
    for t in range(2):
        ring.append(bf(c1.ring_k[t]), bf(c1.ring_v[t]))
    o1 = cca.cca_chunk_attn(ring, bf(c1.q[0]), bf(c1.k_cur[0]), bf(c1.v_cur[0]))
    ring.k_slots[3:].fill_(1e4)
    o2 = cca.cca_chunk_attn(ring, bf(c1.q[0]), bf(c1.k_cur[0]), bf(c1.v_cur[0]))
    torch.cuda.synchronize()
    assert torch.isfinite(o1.float()).all() and torch.equal(o1, o2)
    ref = oca.chunk_attention(c1.q[0], c1.ring_k, c1.ring_v, 2, 5, k_cur=c1.k_cur[0], v_cur=c1.v_cur[0])
    assert_attn_close(to_np(o1), ref, what="t=2 W=5")


# ------------------------------------------------------------------ mask-cached chunk (workload 4)
def test_mask_cached_chunk_end_to_end(c1, c1_ring, c1_ref):
    m = synth.mask_chunk()
    src, edit = torch.from_numpy(m.src).to(dev()), torch.from_numpy(m.edit).to(dev())
    mask = cca.cca_token_mask_l2(src, edit, prune_quantile=m.prune_quantile)
    idx, n = cca.cca_compact(mask)
    n_max = 1620
    q = bf(c1.q[0])
    o_c = cca.cca_chunk_attn(c1_ring, q, bf(c1.k_cur[0]), bf(c1.v_cur[0]), q_idx=idx, n_q_dev=n, n_q_max=n_max)
    cache = bf(m.o_cache)
    cca.cca_scatter(o_c, idx, n, cache, n_max=n_max)
    torch.cuda.synchronize()
    check_status(c1_ring)
    m_ref, _, _ = omask.token_mask(m.src, m.edit, prune_quantile=m.prune_quantile)
    ref_idx, ref_n = omask.compact(m_ref)
    assert n.item() == ref_n == 486
    full = c1_ref[0]
    # active rows: attention of those queries over the full KV; inactive rows: cache unchanged
    got = to_np(cache)
    assert_attn_close(got[ref_idx], full[ref_idx], what="active rows")
    assert np.array_equal(got[m_ref == 0], m.o_cache[m_ref == 0])
    # row independence: compacted row i equals the dense path's row idx[i]
    dense = cca.cca_chunk_attn(c1_ring, q, bf(c1.k_cur[0]), bf(c1.v_cur[0]))
    torch.cuda.synchronize()
    diff = (o_c[:ref_n].float() - dense[torch.from_numpy(ref_idx).long().to(dev())].float()).abs().max().item()
    assert diff <= 1e-2


def test_gathered_queries_with_out_of_range_indices(c1, c1_ref):
    """A query index outside [0, L) sets CCA_DEV_BAD_INDEX and that query
    reads as zeros (uniform weights: the mean of the visible values); the
    other queries are unaffected."""
    ring = cca.KVRing(c1.n_heads, c1.head_dim, c1.chunk_len, c1.window, device=dev())
    for t in range(c1.t):
        ring.append(bf(c1.ring_k[t]), bf(c1.ring_v[t]))
    sel = [5, 1619, 99999, 0, -3, 777]
    idx = torch.tensor(sel, dtype=torch.int32, device=dev())
    n = torch.tensor([len(sel)], dtype=torch.int32, device=dev())
    o = cca.cca_chunk_attn(ring, bf(c1.q[0]), bf(c1.k_cur[0]), bf(c1.v_cur[0]), q_idx=idx, n_q_dev=n, n_q_max=16)
    torch.cuda.synchronize()
    assert int(ring.status.item()) == cca.CCA_DEV_BAD_INDEX
    got = to_np(o)[: len(sel)]
    good = [i for i, r in enumerate(sel) if 0 <= r < c1.chunk_len]
    assert_attn_close(got[good], c1_ref[0][[sel[i] for i in good]], what="valid rows beside bad indices")
    zero_q = np.zeros((1, c1.n_heads, c1.head_dim), dtype=np.float32)
    ref0 = oca.chunk_attention(zero_q, c1.ring_k, c1.ring_v, c1.t, c1.window, k_cur=c1.k_cur[0], v_cur=c1.v_cur[0])
    for i, r in enumerate(sel):
        if not 0 <= r < c1.chunk_len:
            assert_attn_close(got[i:i + 1], ref0, what=f"bad index {r} reads as a zero query")


@pytest.mark.parametrize("ctas", ["auto", "37"])
def test_fused_scatter_equals_attention_then_scatter(c1, c1_ring, monkeypatch, ctas):
    """cca_chunk_attn_scatter writes every active query's row straight into the
    cache: bit-identical to cca_chunk_attn on the compact buffer followed by
    cca_scatter (split items included), inactive rows untouched."""
    if ctas != "auto":
        monkeypatch.setenv("CCA_ATTN_CTAS", ctas)
    m = synth.mask_chunk()
    src, edit = torch.from_numpy(m.src).to(dev()), torch.from_numpy(m.edit).to(dev())
    mask = cca.cca_token_mask_l2(src, edit, prune_quantile=m.prune_quantile)
    idx, n = cca.cca_compact(mask)
    q, kc, vc = bf(c1.q[0]), bf(c1.k_cur[0]), bf(c1.v_cur[0])
    o_c = cca.cca_chunk_attn(c1_ring, q, kc, vc, q_idx=idx, n_q_dev=n, n_q_max=1620)
    two_pass = bf(m.o_cache)
    cca.cca_scatter(o_c, idx, n, two_pass, n_max=1620)
    fused = bf(m.o_cache)
    cca.cca_chunk_attn_scatter(c1_ring, q, kc, vc, idx, fused, n_q_dev=n, n_q_max=1620)
    torch.cuda.synchronize()
    check_status(c1_ring)
    assert torch.equal(fused, two_pass)
    m_ref, _, _ = omask.token_mask(m.src, m.edit, prune_quantile=m.prune_quantile)
    assert np.array_equal(to_np(fused)[m_ref == 0], m.o_cache[m_ref == 0])


def test_fused_scatter_fp8_and_empty():
    s = synth.fp8_720p(n_steps=1)
    m = synth.mask_chunk()
    ring = cca.KVRing(s.n_heads, s.head_dim, s.chunk_len, s.window, dtype="e4m3", device=dev())
    for t in range(s.t):
        ring.append(bf(s.ring_k[t]), bf(s.ring_v[t]))
    mask = cca.cca_token_mask_l2(torch.from_numpy(m.src).to(dev()), torch.from_numpy(m.edit).to(dev()),
                                 prune_quantile=m.prune_quantile)
    idx, n = cca.cca_compact(mask)
    q8, qs = cca.cca_quant_e4m3(bf(s.q[0]))
    k8, ks = cca.cca_quant_e4m3(bf(s.k_cur[0]))
    v8, vs = cca.cca_quant_e4m3_f16(bf(s.v_cur[0]))
    o_c = cca.cca_chunk_attn(ring, q8, k8, v8, q_scale=qs, kcur_scale=ks, vcur_scale=vs, q_idx=idx, n_q_dev=n,
                             n_q_max=s.chunk_len)
    two_pass = torch.zeros((s.chunk_len, s.n_heads, s.head_dim), dtype=torch.bfloat16, device=dev())
    cca.cca_scatter(o_c, idx, n, two_pass, n_max=s.chunk_len)
    fused = torch.zeros_like(two_pass)
    cca.cca_chunk_attn_scatter(ring, q8, k8, v8, idx, fused, q_scale=qs, kcur_scale=ks, vcur_scale=vs, n_q_dev=n,
                               n_q_max=s.chunk_len)
    # empty active set: the cache is left as it is
    keep = torch.full_like(two_pass, 3.0)
    n0 = torch.zeros(1, dtype=torch.int32, device=dev())
    cca.cca_chunk_attn_scatter(ring, q8, k8, v8, idx, keep, q_scale=qs, kcur_scale=ks, vcur_scale=vs, n_q_dev=n0,
                               n_q_max=s.chunk_len)
    torch.cuda.synchronize()
    check_status(ring)
    assert torch.equal(fused, two_pass)
    assert (keep == 3.0).all()


def test_mask_cached_full_and_empty_masks(c1, c1_ring, c1_ref):
    q = bf(c1.q[0])
    full_idx = torch.arange(1620, dtype=torch.int32, device=dev())
    n_full = torch.tensor([1620], dtype=torch.int32, device=dev())
    o = cca.cca_chunk_attn(c1_ring, q, bf(c1.k_cur[0]), bf(c1.v_cur[0]), q_idx=full_idx, n_q_dev=n_full)
    torch.cuda.synchronize()
    assert_attn_close(to_np(o), c1_ref[0], what="full mask")
    n0 = torch.zeros(1, dtype=torch.int32, device=dev())
    out = torch.full((1620, 24, 128), 7.0, dtype=torch.bfloat16, device=dev())
    cca.cca_chunk_attn(c1_ring, q, bf(c1.k_cur[0]), bf(c1.v_cur[0]), q_idx=full_idx, n_q_dev=n0, out=out)
    torch.cuda.synchronize()
    assert (out == 7.0).all()


# ------------------------------------------------------------------ long stream (workload 2)
def test_long_stream_ring_and_sampled_attention():
    ls = synth.LongStream(n_chunks=225)
    ring = cca.KVRing(ls.n_heads, ls.head_dim, ls.chunk_len, ls.window, device=dev())
    oracle = oring.KVRing(ls.window)
    sampled = {0, 1, 2, 3, 4, 5, 100, 224}
    q_fixed = bf(ls.query(0, 0))
    for t in range(ls.n_chunks):
        k, v = ls.next_kv()
        if t in sampled:
            q = ls.query(t, 0)
            o = cca.cca_chunk_attn(ring, bf(q), bf(k), bf(v))
            torch.cuda.synchronize()
            past_k = {c: oracle.get(c)[0] for c in oracle.chunks()}
            past_v = {c: oracle.get(c)[1] for c in oracle.chunks()}
            ref = oca.chunk_attention(q, past_k, past_v, t, ls.window, k_cur=k, v_cur=v)
            assert_attn_close(to_np(o), ref, what=f"stream chunk {t}")
        else:
            cca.cca_chunk_attn(ring, q_fixed, bf(k), bf(v))
        ring.append(bf(k), bf(v))
        oracle.append(k, v)
        n, slots, ids = ring.query()
        assert ids == oracle.chunks()
        if t in sampled or t == ls.n_chunks - 1:
            torch.cuda.synchronize()
            for sl, c in zip(slots, ids):
                assert torch.equal(ring.k_slots[sl].cpu(), synth.as_torch_bf16(oracle.get(c)[0]))
    check_status(ring)


# ------------------------------------------------------------------ e4m3 attention (workload 3)
def _fp8_stream_ref(ring_k, ring_v, q, kc, vc, t, window):
    """Quantisation-aware oracle: every tensor quantised per head by the oracle's
    own e4m3 encoder, attention in fp64 on the dequantised values."""
    deq = lambda x: ofp8.dequantize_per_head(*ofp8.quantize_per_head(x))
    past_k = {c: deq(ring_k[c]) for c in range(t)}
    past_v = {c: deq(ring_v[c]) for c in range(t)}
    return oca.chunk_attention(deq(q), past_k, past_v, t, window, k_cur=deq(kc), v_cur=deq(vc))


def _fp8_call(ring, q, kc, vc, **kw):
    q8, qs = cca.cca_quant_e4m3(bf(q))
    k8, ks = cca.cca_quant_e4m3(bf(kc))
    v8, vs = cca.cca_quant_e4m3_f16(bf(vc))
    return cca.cca_chunk_attn(ring, q8, k8, v8, q_scale=qs, kcur_scale=ks, vcur_scale=vs, **kw)


@pytest.mark.parametrize("ctas", ["auto", "24"])
def test_attention_fp8_720p(ctas, monkeypatch, record_property):
    if ctas != "auto":
        monkeypatch.setenv("CCA_ATTN_CTAS", ctas)
    s = synth.fp8_720p()
    ring = cca.KVRing(s.n_heads, s.head_dim, s.chunk_len, s.window, dtype="e4m3", device=dev())
    for t in range(s.t):
        ring.append(bf(s.ring_k[t]), bf(s.ring_v[t]))
    for st in range(len(s.q)):
        o = _fp8_call(ring, s.q[st], s.k_cur[st], s.v_cur[st])
        ref = _fp8_stream_ref(s.ring_k, s.ring_v, s.q[st], s.k_cur[st], s.v_cur[st], s.t, s.window)
        assert_attn_close(to_np(o), ref, FP8_MAX_ABS, FP8_REL_L2, what=f"fp8 720p step {st}")
        if st == 0 and ctas == "auto":
            # information only: the same call against fp64 attention on the
            # unquantised inputs (quantisation error + kernel error)
            raw = oca.chunk_attention(s.q[st], {c: s.ring_k[c] for c in range(s.t)},
                                      {c: s.ring_v[c] for c in range(s.t)}, s.t, s.window,
                                      k_cur=s.k_cur[st], v_cur=s.v_cur[st])
            d = to_np(o) - raw
            record_property("fp8_vs_unquantised_max_abs", float(np.abs(d).max()))
            record_property("fp8_vs_unquantised_rel_l2", float(np.linalg.norm(d) / np.linalg.norm(raw)))
    check_status(ring)


def test_attention_fp8_ragged_stream_with_eviction():
    g = np.random.default_rng(31)
    L, H, D, W, n = 200, 2, 128, 2, 6
    draw = lambda: synth.bf16_round(g.standard_t(4.0, size=(L, H, D)).astype(np.float32))
    q = [draw() for _ in range(n)]
    k = [draw() for _ in range(n)]
    v = [draw() for _ in range(n)]
    ring = cca.KVRing(H, D, L, W, dtype="e4m3", device=dev())
    for t in range(n):
        o = _fp8_call(ring, q[t], k[t], v[t])
        ref = _fp8_stream_ref(k, v, q[t], k[t], v[t], t, W)
        assert_attn_close(to_np(o), ref, FP8_MAX_ABS, FP8_REL_L2, what=f"fp8 ragged t={t}")
        ring.append(bf(k[t]), bf(v[t]))
    check_status(ring)


def test_attention_fp8_zero_and_tiny_v_scales():
    """Caller-supplied V scales far apart: a zero scale for the current chunk
    (its values are all zero, its keys still take part in the softmax) and a
    ring chunk whose V scale is 2^-30 of its own absmax scale.  The result is
    the dequantised attention, finite everywhere."""
    g = np.random.default_rng(37)
    L, H, D, W = 200, 2, 128, 2
    draw = lambda: synth.bf16_round(g.standard_t(4.0, size=(L, H, D)).astype(np.float32))
    k = [draw() for _ in range(4)]
    v = [draw() for _ in range(4)]
    q = draw()
    ring = cca.KVRing(H, D, L, W, dtype="e4m3", device=dev())
    for t in range(3):
        ring.append(bf(k[t]), bf(v[t]))
    _, slots, ids = ring.query()
    assert ids == [0, 1, 2]
    ring.v_scale[slots[1]] *= 2.0 ** -30
    q8, qs = cca.cca_quant_e4m3(bf(q))
    k8, ks = cca.cca_quant_e4m3(bf(k[3]))
    v8, vs = cca.cca_quant_e4m3_f16(bf(v[3]))
    o = cca.cca_chunk_attn(ring, q8, k8, v8, q_scale=qs, kcur_scale=ks, vcur_scale=torch.zeros_like(vs))

    def deq(x, f=1.0):
        codes, sc = ofp8.quantize_per_head(x)
        return ofp8.dequantize_per_head(codes, sc.astype(np.float64) * f)

    past_k = {c: deq(k[c]) for c in range(3)}
    past_v = {0: deq(v[0]), 1: deq(v[1], 2.0 ** -30), 2: deq(v[2])}
    ref = oca.chunk_attention(deq(q), past_k, past_v, 3, W, k_cur=deq(k[3]), v_cur=deq(v[3], 0.0))
    got = to_np(o)
    assert np.all(np.isfinite(got))
    assert_attn_close(got, ref, FP8_MAX_ABS, FP8_REL_L2, what="fp8 zero / tiny V scales")
    check_status(ring)


def test_attention_fp8_gathered_queries():
    s = synth.fp8_720p(n_steps=1)
    m = synth.mask_chunk()
    ring = cca.KVRing(s.n_heads, s.head_dim, s.chunk_len, s.window, dtype="e4m3", device=dev())
    for t in range(s.t):
        ring.append(bf(s.ring_k[t]), bf(s.ring_v[t]))
    mask_ref, _, _ = omask.token_mask(m.src, m.edit, prune_quantile=m.prune_quantile)
    idx_ref, n_ref = omask.compact(mask_ref)
    idx = torch.from_numpy(idx_ref).to(dev())
    n = torch.tensor([n_ref], dtype=torch.int32, device=dev())
    o = _fp8_call(ring, s.q[0], s.k_cur[0], s.v_cur[0], q_idx=idx, n_q_dev=n, n_q_max=s.chunk_len)
    ref = _fp8_stream_ref(s.ring_k, s.ring_v, s.q[0], s.k_cur[0], s.v_cur[0], s.t, s.window)
    assert_attn_close(to_np(o)[:n_ref], ref[idx_ref], FP8_MAX_ABS, FP8_REL_L2, what="fp8 gathered")
