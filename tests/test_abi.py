"""C-ABI checks that need no GPU: the library builds and loads, exports every
entry point declared in include/cca.h, and its host-side logic (argument
validation, ring slot bookkeeping) behaves as documented.  No kernel runs here.
"""

import ctypes
import os
import re

import pytest

import chunk_causal_attention_b200 as cca
from chunk_causal_attention_b200 import build as cca_build
from oracle import kv_ring

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    cca_build.build(quiet=True)
    return cca.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "cca.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cca_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_symbols() == sorted(cca.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
    assert L.cca_version() == (0 << 16) | 1
    assert L.cca_last_error() is not None


def _desc(**kw):
    d = dict(n_heads=2, head_dim=64, chunk_len=16, window=2, dtype=cca.CCA_BF16, k_slots=0x100000,
             v_slots=0x200000, k_scale=None, v_scale=None, dev_status=None)
    d.update(kw)
    return cca._RingDesc(**d)


def _create(L, d):
    h = ctypes.c_void_p()
    st = L.cca_kv_ring_create(ctypes.byref(d), ctypes.byref(h))
    return st, h


@pytest.mark.parametrize("bad", [dict(head_dim=96), dict(n_heads=0), dict(chunk_len=0), dict(window=-1),
                                 dict(window=16), dict(k_slots=None), dict(v_slots=0x200001),
                                 dict(dtype=cca.CCA_E4M3), dict(k_scale=0x300000), dict(dtype=7)])
def test_ring_create_rejects_bad_descriptors(L, bad):
    st, h = _create(L, _desc(**bad))
    assert st == 1 and not h.value  # CCA_ERR_INVALID_ARG, no handle
    assert L.cca_last_error().decode()


def test_ring_slot_bookkeeping_matches_oracle_deque(L):
    """Logical content reported by cca_kv_ring_query after n appends (set with
    cca_kv_ring_restore, no device work) equals the oracle deque."""
    for w in (0, 1, 2, 3, 7, 15):
        st, h = _create(L, _desc(window=w))
        assert st == 0
        ring = kv_ring.KVRing(w)
        for n in range(225):
            assert L.cca_kv_ring_restore(h, n) == 0
            na = ctypes.c_int64()
            cnt = ctypes.c_int32()
            slots = (ctypes.c_int32 * (1 + w))()
            ids = (ctypes.c_int64 * (1 + w))()
            assert L.cca_kv_ring_query(h, ctypes.byref(na), slots, ids, ctypes.byref(cnt)) == 0
            assert na.value == n
            assert list(ids[:cnt.value]) == ring.chunks()
            got_slots = list(slots[:cnt.value])
            # every cached chunk has its own slot, the sink is in slot 0
            assert len(set(got_slots)) == len(got_slots)
            assert all(0 <= s <= w for s in got_slots)
            if cnt.value:
                assert got_slots[0] == 0
            ring.append(n, n)
        # a chunk keeps its slot until it is evicted: slot of chunk c is stable
        assert L.cca_kv_ring_reset(h) == 0
        assert L.cca_kv_ring_query(h, ctypes.byref(na), None, None, ctypes.byref(cnt)) == 0
        assert na.value == 0 and cnt.value == 0
        assert L.cca_kv_ring_destroy(h) == 0


def test_slots_stable_until_eviction(L):
    w = 3
    st, h = _create(L, _desc(window=w))
    where = {}
    for n in range(1, 40):
        L.cca_kv_ring_restore(h, n)
        cnt = ctypes.c_int32()
        slots = (ctypes.c_int32 * (1 + w))()
        ids = (ctypes.c_int64 * (1 + w))()
        L.cca_kv_ring_query(h, None, slots, ids, ctypes.byref(cnt))
        for s, c in zip(slots[:cnt.value], ids[:cnt.value]):
            if c in where:
                assert where[c] == s
            where[c] = s
    L.cca_kv_ring_destroy(h)


def test_call_validation_without_device_work(L):
    st, h = _create(L, _desc())
    vp = ctypes.c_void_p
    # attention: n_q_max out of range, NULL / misaligned pointers, scales on a BF16 ring
    assert L.cca_chunk_attn(h, vp(0x1000), vp(0x1000), vp(0x1000), None, None, None, None, None, 17, 0.0,
                            vp(0x1000), None, 0, None) == 1
    assert L.cca_chunk_attn(h, None, vp(0x1000), vp(0x1000), None, None, None, None, None, 16, 0.0,
                            vp(0x1000), None, 0, None) == 1
    assert L.cca_chunk_attn(h, vp(0x1008), vp(0x1000), vp(0x1000), None, None, None, None, None, 16, 0.0,
                            vp(0x1000), None, 0, None) == 1
    assert L.cca_chunk_attn(h, vp(0x1000), vp(0x1000), vp(0x1000), vp(0x2000), None, None, None, None, 16,
                            0.0, vp(0x1000), None, 0, None) == 1
    assert L.cca_chunk_attn(h, None, None, None, None, None, None, None, None, 0, 0.0, None, None, 0,
                            None) == 0  # nothing to do
    assert L.cca_chunk_attn_scatter(h, vp(0x1000), vp(0x1000), vp(0x1000), None, None, None, None, None, 16,
                                    0.0, vp(0x1000), None, 0, None) == 1  # q_idx names the output rows
    # mask / compact / scatter argument checks
    assert L.cca_token_mask_l2(vp(0x1000), vp(0x1000), 10, 6, 1.0, -1.0, vp(0x1000), None, None, None) == 1
    assert L.cca_token_mask_l2(vp(0x1000), vp(0x1000), 10, 16, 1.0, 1.5, vp(0x1000), None, None, None) == 1
    assert L.cca_token_mask_l2(vp(0x1000), vp(0x1000), 40000, 16, 1.0, 0.7, vp(0x1000), None, None, None) == 1
    assert L.cca_token_mask_l2(vp(0x1000), vp(0x1000), 10, 16, -1.0, -1.0, vp(0x1000), None, None, None) == 1
    assert L.cca_compact(vp(0x1000), -1, vp(0x1000), vp(0x1000), None, 0, None) == 1
    assert L.cca_compact(vp(0x1000), 10, vp(0x1000), None, None, 0, None) == 1
    assert L.cca_compact(vp(0x1000), 100000, vp(0x1000), vp(0x1000), None, 0, None) == 1  # needs a workspace
    assert L.cca_compact(vp(0x1000), 10, vp(0x1002), vp(0x1000), None, 0, None) == 1  # idx not 4-byte aligned
    sz = ctypes.c_size_t()
    assert L.cca_compact_workspace_size(16384, ctypes.byref(sz)) == 0 and sz.value == 0
    assert L.cca_compact_workspace_size(16385, ctypes.byref(sz)) == 0 and sz.value == 4096 * 8 + 16
    assert L.cca_compact(vp(0x1000), 16385, vp(0x1000), vp(0x1000), vp(0x1000), 4096 * 8, None) == 1  # too small
    assert L.cca_compact(vp(0x1000), (1 << 30) + 1, vp(0x1000), vp(0x1000), vp(0x1000), 1 << 30, None) == 1
    assert L.cca_scatter(vp(0x1000), vp(0x1000), vp(0x1000), 4, 20, vp(0x1000), None) == 1
    assert L.cca_scatter(None, None, None, 0, 16, None, None) == 0
    assert L.cca_quant_e4m3(vp(0x1000), cca.CCA_BF16, 4, 2, 80, vp(0x1000), vp(0x1000), None) == 1
    qkv = L.cca_quant_e4m3_qkv
    a = vp(0x1000)
    assert qkv(a, a, a, cca.CCA_BF16, 4, 2, 80, a, a, a, a, a, a, None) == 1  # D not in {64, 128}
    assert qkv(a, None, a, cca.CCA_BF16, 4, 2, 64, a, a, a, a, a, a, None) == 1  # missing k
    assert qkv(a, a, a, cca.CCA_BF16, 4, 2, 64, a, a, a, a, None, a, None) == 1  # missing k_scale
    assert qkv(a, a, vp(0x1008), cca.CCA_BF16, 4, 2, 64, a, a, a, a, a, a, None) == 1  # v misaligned
    assert qkv(a, a, a, cca.CCA_E4M3, 4, 2, 64, a, a, a, a, a, a, None) == 1  # source must be BF16 / F32
    assert qkv(a, a, a, cca.CCA_BF16, 4, 2, 64, a, a, a, a, a, vp(0x1002), None) == 1  # scale misaligned
    assert L.cca_kv_append(h, None, vp(0x1000), cca.CCA_BF16, None) == 1
    assert L.cca_kv_append(h, vp(0x1000), vp(0x1000), cca.CCA_E4M3, None) == 1
    # workspace queries and the allocation-free variant: argument errors come first
    sz = ctypes.c_size_t()
    assert L.cca_chunk_attn_workspace_size(None, 16, ctypes.byref(sz)) == 1
    assert L.cca_chunk_attn_workspace_size(h, 17, ctypes.byref(sz)) == 1
    assert L.cca_chunk_attn_workspace_size(h, 16, None) == 1
    assert L.cca_chunk_attn_noalloc(None, vp(0x1000), vp(0x1000), vp(0x1000), None, None, None, None, None, 16,
                                    0.0, vp(0x1000), None) == 1
    assert L.cca_chunk_attn_noalloc(h, vp(0x1000), vp(0x1000), vp(0x1000), None, None, None, None, None, 17,
                                    0.0, vp(0x1000), None) == 1
    assert L.cca_compact_workspace_size(-1, ctypes.byref(sz)) == 1
    assert L.cca_attn_workspace_size(96, ctypes.byref(sz)) == 1
    assert L.cca_attn_workspace_size(128, None) == 1
    # token groups: NULL ring / tensors, sizes out of range, misalignment, scales on BF16
    g = L.cca_chunk_attn_groups
    assert g(None, vp(0x1000), vp(0x1000), vp(0x1000), 8, None, None, 0, None, None, None, None, None, 0.0,
             vp(0x1000), None, 0, None) == 1
    assert g(h, vp(0x1000), vp(0x1000), vp(0x1000), -1, None, None, 0, None, None, None, None, None, 0.0,
             vp(0x1000), None, 0, None) == 1
    assert g(h, vp(0x1000), vp(0x1000), vp(0x1000), 8, None, None, 4, None, None, None, None, None, 0.0,
             vp(0x1000), None, 0, None) == 1  # n_ref > 0 without k_ref / v_ref
    assert g(h, vp(0x1004), vp(0x1000), vp(0x1000), 8, None, None, 0, None, None, None, None, None, 0.0,
             vp(0x1000), None, 0, None) == 1
    assert g(h, vp(0x1000), vp(0x1000), vp(0x1000), 8, None, None, 0, vp(0x2000), None, None, None, None, 0.0,
             vp(0x1000), None, 0, None) == 1
    assert g(h, None, None, None, 0, None, None, 0, None, None, None, None, None, 0.0, None, None, 0, None) == 0
    # packed block-causal forward: descriptor checks
    def bd(**kw):
        d = dict(n_heads=2, head_dim=64, chunk_len=16, n_chunks=3, window=1, dtype=cca.CCA_BF16,
                 k_cur=0x1000, v_cur=0x2000, k_hist=0x1000, v_hist=0x2000, k_ref=None, v_ref=None, ref_len=0,
                 kcur_scale=None, vcur_scale=None, khist_scale=None, vhist_scale=None, kref_scale=None,
                 vref_scale=None, dev_status=None)
        d.update(kw)
        return cca._BlockDesc(**d)
    b = L.cca_block_attn
    assert b(None, vp(0x1000), None, 0.0, vp(0x1000), None, 0, None) == 1
    for bad in (dict(head_dim=96), dict(n_heads=0), dict(chunk_len=0), dict(window=-1), dict(n_chunks=4096),
                dict(k_hist=None), dict(v_cur=0x2008), dict(ref_len=5), dict(dtype=cca.CCA_E4M3),
                dict(kcur_scale=0x3000), dict(dtype=9)):
        assert b(ctypes.byref(bd(**bad)), vp(0x1000), None, 0.0, vp(0x1000), None, 0, None) != 0, bad
    assert b(ctypes.byref(bd(n_chunks=0)), None, None, 0.0, None, None, 0, None) == 0  # nothing to do
    # ring bookkeeping calls reject bad handles and counts
    assert L.cca_kv_ring_restore(h, -1) == 1
    assert L.cca_kv_ring_restore(None, 3) == 1
    assert L.cca_kv_ring_reset(None) == 1
    assert L.cca_kv_ring_query(None, None, None, None, None) == 1
    assert L.cca_kv_ring_destroy(h) == 0


def test_library_rope_table_follows_the_stated_recipe(L):
    """cca_mrope_freqs is host code: its table equals the oracle's fp64 table
    rounded to fp32 (within an ulp of the pow), and bad sections are refused."""
    import numpy as np
    from oracle import rope as orope
    for D, sec in ((128, (22, 21, 21)), (64, (12, 10, 10)), (128, (64, 0, 0))):
        buf = (ctypes.c_float * (2 * D))()
        assert L.cca_mrope_freqs(D, *sec, ctypes.c_float(10000.0), buf) == 0
        got = np.array(list(buf), dtype=np.float64).reshape(4, D // 2)
        want = orope.frequencies(D, sections=sec)
        assert np.all(np.abs(got - want) <= 2.0 ** -23 * np.abs(want))
    buf = (ctypes.c_float * 256)()
    assert L.cca_mrope_freqs(128, 22, 21, 20, ctypes.c_float(10000.0), buf) == 1
    assert L.cca_mrope_freqs(96, 16, 16, 16, ctypes.c_float(10000.0), buf) == 1
    assert L.cca_mrope_freqs(128, 22, 21, 21, ctypes.c_float(1.0), buf) == 1
    vp = ctypes.c_void_p
    assert L.cca_rope_qk(vp(0x1000), None, cca.CCA_BF16, 10, 2, 64, None, vp(0x2000), vp(0x1000), None, None) == 1
    assert L.cca_rope_qk(vp(0x1000), None, cca.CCA_E4M3, 10, 2, 64, vp(0x3000), vp(0x2000), vp(0x1000), None,
                         None) == 1
    assert L.cca_rope_qk(vp(0x1008), None, cca.CCA_BF16, 10, 2, 64, vp(0x3000), vp(0x2000), vp(0x1000), None,
                         None) == 1
    assert L.cca_rope_qk(None, None, cca.CCA_BF16, 10, 2, 64, None, None, None, None, None) == 0


def test_product_path_has_no_cpu_fallback():
    import torch
    with pytest.raises((ValueError, RuntimeError)):
        cca.cca_token_mask_l2(torch.zeros(4, 16), torch.zeros(4, 16), tau=1.0)
    src = open(os.path.join(ROOT, "chunk_causal_attention_b200", "__init__.py")).read()
    assert "oracle" not in src.replace("no CPU fallback", "")
