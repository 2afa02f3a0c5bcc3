"""The seeded synthetic inputs follow the recipe the design states (CPU only).

Each workload's generator is checked for the statistical property it is meant
to have, on reduced shapes so the suite stays fast: bf16 rounding, per-head RMS
1 for the 720p draws, Student-t(4) scale for the e4m3 workload, the AR(1)
variance of the long stream, the edit offset of the tiny latents, and the
independence / reproducibility of the seeded streams.
"""

import numpy as np
import pytest

import synth


def _is_bf16(x):
    bits = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return np.all((bits & 0xFFFF) == 0)


def test_tiny_shapes_rounding_and_edit_offset():
    s = synth.tiny()
    assert len(s.q) == 4 and s.q[0].shape == (16, 1, 64) and s.window == 2
    assert all(_is_bf16(x) for x in s.q + s.k + s.v)
    d = s.edit - s.src
    assert abs(d.std() - 0.25) < 0.05 and abs(d.mean()) < 0.06


def test_chunk_draws_have_unit_head_rms():
    c = synth.chunk_720p(n_heads=3, head_dim=32, chunk_len=200, n_steps=1, n_prefill=2)
    assert c.t == 2 and len(c.ring_k) == 2 and len(c.q) == 1
    for x in c.ring_k + c.ring_v + c.q + c.k_cur + c.v_cur:
        assert _is_bf16(x)
        rms = np.sqrt(np.mean(x.astype(np.float64) ** 2, axis=(0, 2)))
        assert np.all(np.abs(rms - 1.0) < 4e-3)  # exact before bf16 rounding


def test_fp8_workload_is_student_t4_at_raw_scale():
    c = synth.fp8_720p(n_heads=4, head_dim=64, chunk_len=400, n_steps=1, n_prefill=1)
    x = np.abs(np.concatenate([a.ravel() for a in c.ring_k + c.q]))
    # median |t_4| = 0.7407 (quantile 0.75 of Student-t with 4 degrees of freedom)
    assert abs(np.median(x) - 0.7407) < 0.02
    assert x.max() > 10.0  # heavy tail present at this sample size


def test_long_stream_ar1_variance_and_lazy_queries():
    ls = synth.LongStream(n_heads=2, head_dim=32, chunk_len=256, n_chunks=60)
    var = []
    for t in range(60):
        k, v = ls.next_kv()
        var.append(float(np.var(k.astype(np.float64))))
    # x_0 ~ N(0,1); x_t = 0.9 x_{t-1} + 0.44 n_t  =>  var_1 = 0.81 + 0.1936 = 1.0036,
    # stationary 0.1936 / 0.19 = 1.0189
    assert abs(var[1] - 1.0036) < 0.03
    assert abs(np.mean(var[40:]) - 0.1936 / 0.19) < 0.03
    # consecutive chunks are correlated with coefficient 0.9 (per element)
    ls2 = synth.LongStream(n_heads=2, head_dim=32, chunk_len=256, n_chunks=3)
    a, _ = ls2.next_kv()
    b, _ = ls2.next_kv()
    rho = np.corrcoef(a.ravel(), b.ravel())[0, 1]
    assert abs(rho - 0.9 / np.sqrt(1.0036)) < 0.02
    # queries are reproducible and independent of the K/V stream position
    assert np.array_equal(ls.query(5, 0), ls2.query(5, 0))
    assert not np.array_equal(ls.query(5, 0), ls.query(5, 1))


def test_seeded_streams_are_reproducible_and_distinct():
    a = synth.rng(2, 7, 0).standard_normal(8)
    b = synth.rng(2, 7, 0).standard_normal(8)
    c = synth.rng(2, 7, 1).standard_normal(8)
    assert np.array_equal(a, b) and not np.array_equal(a, c)


def test_mask_chunk_recipe():
    m = synth.mask_chunk()
    assert m.src.shape == (1620, 16) and m.edit.shape == (1620, 16)
    assert abs(m.region.mean() - 0.30) <= 0.02
    off = m.edit - m.src
    inside, outside = off[m.region], off[~m.region]
    assert abs(inside.mean() - 2.0) < 0.05 and abs(inside.std() - 1.0) < 0.05
    assert abs(outside.mean()) < 0.01 and abs(outside.std() - 0.1) < 0.01
    assert m.prune_quantile == pytest.approx(0.70)
    assert _is_bf16(m.o_cache) and abs(float(m.o_cache.std()) - 0.02) < 0.002
