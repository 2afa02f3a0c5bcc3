"""Python binding of libcca.so: chunk-wise causal attention over a bounded KV
cache and the L2 token-mask cache, for B200 (sm_100a).

This module only marshals arguments: every step runs in the CUDA kernels of
``libcca.so`` (built in-tree by ``python -m chunk_causal_attention_b200.build``).
PyTorch is used for device memory and streams only.  There is no CPU fallback:
if the library is missing, or a tensor is not on a CUDA device, the calls raise.

The functions carry the names of the C ABI (``include/cca.h``); ``KVRing`` is a
small owner of the ring's device buffers around ``cca_kv_ring_*``.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "CCA_BF16", "CCA_E4M3", "CCA_F32", "CcaError", "KVRing", "lib", "lib_path", "EXPORTED",
    "cca_kv_append", "cca_quant_e4m3", "cca_chunk_attn", "cca_chunk_attn_workspace_size", "cca_chunk_attn_noalloc",
    "cca_chunk_attn_scatter", "cca_attn_workspace_size", "cca_chunk_attn_groups", "cca_block_attn",
    "cca_mrope_freqs", "cca_rope_qk", "cca_kv_append_rope", "cca_token_mask_l2_frames", "cca_quant_e4m3_f16",
    "cca_quant_e4m3_qkv", "cca_token_mask_l2", "cca_compact", "cca_compact_workspace_size", "cca_scatter", "cca_selftest_bounded_wait",
    "cca_version",
    "cca_take_launch_count",
]

CCA_BF16, CCA_E4M3, CCA_F32 = 0, 1, 2
CCA_DEV_OK, CCA_DEV_TIMEOUT, CCA_DEV_BAD_INDEX = 0, 1, 2
_STATUS = {0: "CCA_OK", 1: "CCA_ERR_INVALID_ARG", 2: "CCA_ERR_UNSUPPORTED", 3: "CCA_ERR_STATE",
           4: "CCA_ERR_CUDA", 5: "CCA_ERR_DEVICE_TIMEOUT"}

# Every entry point declared in include/cca.h.
EXPORTED = (
    "cca_kv_ring_create", "cca_kv_ring_destroy", "cca_kv_ring_reset", "cca_kv_ring_query",
    "cca_kv_ring_restore", "cca_kv_append", "cca_quant_e4m3", "cca_quant_e4m3_f16", "cca_quant_e4m3_qkv",
    "cca_chunk_attn",
    "cca_chunk_attn_workspace_size", "cca_chunk_attn_noalloc", "cca_chunk_attn_scatter", "cca_attn_workspace_size",
    "cca_chunk_attn_groups", "cca_block_attn", "cca_mrope_freqs", "cca_rope_qk", "cca_kv_append_rope",
    "cca_token_mask_l2", "cca_token_mask_l2_frames", "cca_compact",
    "cca_compact_workspace_size",
    "cca_scatter", "cca_selftest_bounded_wait", "cca_last_error", "cca_version", "cca_take_launch_count",
)


class CcaError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {_STATUS.get(status, status)}: {msg}")
        self.status = status


class _RingDesc(ctypes.Structure):
    _fields_ = [("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("chunk_len", ctypes.c_int32),
                ("window", ctypes.c_int32), ("dtype", ctypes.c_int), ("k_slots", ctypes.c_void_p),
                ("v_slots", ctypes.c_void_p), ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
                ("dev_status", ctypes.c_void_p)]


class _BlockDesc(ctypes.Structure):
    _fields_ = [("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("chunk_len", ctypes.c_int32),
                ("n_chunks", ctypes.c_int32), ("window", ctypes.c_int32), ("dtype", ctypes.c_int),
                ("k_cur", ctypes.c_void_p), ("v_cur", ctypes.c_void_p), ("k_hist", ctypes.c_void_p),
                ("v_hist", ctypes.c_void_p), ("k_ref", ctypes.c_void_p), ("v_ref", ctypes.c_void_p),
                ("ref_len", ctypes.c_int32),
                ("kcur_scale", ctypes.c_void_p), ("vcur_scale", ctypes.c_void_p), ("khist_scale", ctypes.c_void_p),
                ("vhist_scale", ctypes.c_void_p), ("kref_scale", ctypes.c_void_p), ("vref_scale", ctypes.c_void_p),
                ("dev_status", ctypes.c_void_p)]


def lib_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcca.so")


_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded libcca.so (raises if it has not been built)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = lib_path()
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m chunk_causal_attention_b200.build`")
    L = ctypes.CDLL(path)
    vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sigs = {
        "cca_kv_ring_create": [ctypes.POINTER(_RingDesc), ctypes.POINTER(vp)],
        "cca_kv_ring_destroy": [vp],
        "cca_kv_ring_reset": [vp],
        "cca_kv_ring_query": [vp, ctypes.POINTER(i64), ctypes.POINTER(i32), ctypes.POINTER(i64),
                              ctypes.POINTER(i32)],
        "cca_kv_ring_restore": [vp, i64],
        "cca_kv_append": [vp, vp, vp, ctypes.c_int, vp],
        "cca_quant_e4m3": [vp, ctypes.c_int, i32, i32, i32, vp, vp, vp],
        "cca_quant_e4m3_f16": [vp, ctypes.c_int, i32, i32, i32, vp, vp, vp],
        "cca_quant_e4m3_qkv": [vp, vp, vp, ctypes.c_int, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp],
        "cca_chunk_attn": [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, f32, vp, vp, sz, vp],
        "cca_chunk_attn_workspace_size": [vp, i32, ctypes.POINTER(sz)],
        "cca_chunk_attn_noalloc": [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, f32, vp, vp],
        "cca_chunk_attn_scatter": [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, f32, vp, vp, sz, vp],
        "cca_attn_workspace_size": [i32, ctypes.POINTER(sz)],
        "cca_mrope_freqs": [i32, i32, i32, i32, f32, vp],
        "cca_rope_qk": [vp, vp, ctypes.c_int, i32, i32, i32, vp, vp, vp, vp, vp],
        "cca_kv_append_rope": [vp, vp, vp, ctypes.c_int, vp, vp, vp],
        "cca_chunk_attn_groups": [vp, vp, vp, vp, i32, vp, vp, i32, vp, vp, vp, vp, vp, f32, vp, vp, sz, vp],
        "cca_block_attn": [ctypes.POINTER(_BlockDesc), vp, vp, f32, vp, vp, sz, vp],
        "cca_token_mask_l2": [vp, vp, i32, i32, f32, f32, vp, vp, vp, vp],
        "cca_token_mask_l2_frames": [vp, vp, i32, i32, i32, f32, f32, vp, vp, vp, vp],
        "cca_compact": [vp, i32, vp, vp, vp, sz, vp],
        "cca_compact_workspace_size": [i32, ctypes.POINTER(sz)],
        "cca_scatter": [vp, vp, vp, i32, i32, vp, vp],
        "cca_selftest_bounded_wait": [vp, i64, i32, vp],
    }
    for name, args in sigs.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    L.cca_last_error.restype = ctypes.c_char_p
    L.cca_last_error.argtypes = []
    L.cca_version.restype = ctypes.c_int32
    L.cca_take_launch_count.restype = ctypes.c_int64
    _LIB = L
    return L


def _check(status: int, where: str) -> None:
    if status != 0:
        raise CcaError(status, where, lib().cca_last_error().decode())


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _src_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return CCA_BF16
    if t.dtype == torch.float32:
        return CCA_F32
    raise ValueError(f"unsupported source dtype {t.dtype} (bf16 or fp32)")


def cca_version() -> int:
    return int(lib().cca_version())


def cca_take_launch_count() -> int:
    return int(lib().cca_take_launch_count())


class KVRing:
    """Bounded KV cache: sink slot + W window slots per tensor, on one device.

    Owns the device buffers (allocated with torch) and the C handle.
    k_slots / v_slots: [(1+W), L, H, D] (bf16; e4m3: uint8 codes for K and
    fp16-widened e4m3 values for V);
    k_scale / v_scale: [(1+W), H] fp32 (e4m3 only); status: int32[1].
    """

    def __init__(self, n_heads: int, head_dim: int, chunk_len: int, window: int,
                 dtype: str = "bf16", device="cuda"):
        self.n_heads, self.head_dim, self.chunk_len, self.window = n_heads, head_dim, chunk_len, window
        self.dtype = dtype
        device = torch.device(device)
        if device.type != "cuda":
            raise ValueError("KVRing lives on a CUDA device")
        shape = (1 + window, chunk_len, n_heads, head_dim)
        if dtype == "bf16":
            self.k_slots = torch.empty(shape, dtype=torch.bfloat16, device=device)
            self.v_slots = torch.empty(shape, dtype=torch.bfloat16, device=device)
            self.k_scale = self.v_scale = None
            cdt = CCA_BF16
        elif dtype == "e4m3":
            self.k_slots = torch.empty(shape, dtype=torch.uint8, device=device)
            self.v_slots = torch.empty(shape, dtype=torch.float16, device=device)  # widened e4m3 values
            self.k_scale = torch.ones((1 + window, n_heads), dtype=torch.float32, device=device)
            self.v_scale = torch.ones((1 + window, n_heads), dtype=torch.float32, device=device)
            cdt = CCA_E4M3
        else:
            raise ValueError("dtype must be 'bf16' or 'e4m3'")
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        d = _RingDesc(n_heads, head_dim, chunk_len, window, cdt, self.k_slots.data_ptr(),
                      self.v_slots.data_ptr(),
                      self.k_scale.data_ptr() if self.k_scale is not None else None,
                      self.v_scale.data_ptr() if self.v_scale is not None else None,
                      self.status.data_ptr())
        h = ctypes.c_void_p()
        _check(lib().cca_kv_ring_create(ctypes.byref(d), ctypes.byref(h)), "cca_kv_ring_create")
        self.handle = h

    def __del__(self):
        h = getattr(self, "handle", None)
        if h and _LIB is not None:
            _LIB.cca_kv_ring_destroy(h)
            self.handle = None

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None) -> None:
        cca_kv_append(self, k_new, v_new, stream=stream)

    def reset(self) -> None:
        _check(lib().cca_kv_ring_reset(self.handle), "cca_kv_ring_reset")

    def restore(self, n_appended: int) -> None:
        _check(lib().cca_kv_ring_restore(self.handle, int(n_appended)), "cca_kv_ring_restore")

    def query(self):
        """(n_appended, [slot per cached chunk], [chunk id per cached chunk])."""
        n = ctypes.c_int64()
        cnt = ctypes.c_int32()
        slots = (ctypes.c_int32 * (1 + self.window))()
        ids = (ctypes.c_int64 * (1 + self.window))()
        _check(lib().cca_kv_ring_query(self.handle, ctypes.byref(n), slots, ids, ctypes.byref(cnt)),
               "cca_kv_ring_query")
        return n.value, list(slots[:cnt.value]), list(ids[:cnt.value])

    @property
    def n_appended(self) -> int:
        return self.query()[0]


def cca_kv_append(ring: KVRing, k_new: torch.Tensor, v_new: torch.Tensor, stream=None) -> None:
    shape = (ring.chunk_len, ring.n_heads, ring.head_dim)
    if tuple(k_new.shape) != shape or tuple(v_new.shape) != shape:
        raise ValueError(f"k_new/v_new must be {shape}")
    if k_new.dtype != v_new.dtype:
        raise ValueError("k_new and v_new must share a dtype")
    _check(lib().cca_kv_append(ring.handle, _ptr(k_new, "k_new"), _ptr(v_new, "v_new"), _src_dtype(k_new),
                               _stream(stream)), "cca_kv_append")


def cca_mrope_freqs(head_dim: int, sections=None, base: float = 10000.0, device=None) -> torch.Tensor:
    """Default [4, D/2] fp32 frequency table (t, h, w sections, then the 1D source row)."""
    if sections is None:
        p = head_dim // 2
        sections = (p - 2 * (p // 3), p // 3, p // 3)
    buf = (ctypes.c_float * (2 * head_dim))()
    _check(lib().cca_mrope_freqs(int(head_dim), int(sections[0]), int(sections[1]), int(sections[2]),
                                 float(base), buf), "cca_mrope_freqs")
    t = torch.tensor(list(buf), dtype=torch.float32).reshape(4, head_dim // 2)
    return t if device is None else t.to(device)


def cca_rope_qk(q: Optional[torch.Tensor], k: Optional[torch.Tensor], pos: torch.Tensor, freq: torch.Tensor,
                q_out: Optional[torch.Tensor] = None, k_out: Optional[torch.Tensor] = None, stream=None):
    """(rope(q), rope(k)) as bf16 [n, H, D]; pos int32 [n, 4], freq fp32 [4, D/2] on the device."""
    x = q if q is not None else k
    n, h, d = x.shape
    if q is not None and q_out is None:
        q_out = torch.empty((n, h, d), dtype=torch.bfloat16, device=x.device)
    if k is not None and k_out is None:
        k_out = torch.empty((n, h, d), dtype=torch.bfloat16, device=x.device)
    _check(lib().cca_rope_qk(_ptr(q, "q"), _ptr(k, "k"), _src_dtype(x), n, h, d, _ptr(pos, "pos", torch.int32),
                             _ptr(freq, "freq", torch.float32), _ptr(q_out, "q_out", torch.bfloat16),
                             _ptr(k_out, "k_out", torch.bfloat16), _stream(stream)), "cca_rope_qk")
    return q_out, k_out


def cca_kv_append_rope(ring: KVRing, k_new: torch.Tensor, v_new: torch.Tensor, pos: torch.Tensor,
                       freq: torch.Tensor, stream=None) -> None:
    shape = (ring.chunk_len, ring.n_heads, ring.head_dim)
    if tuple(k_new.shape) != shape or tuple(v_new.shape) != shape or k_new.dtype != v_new.dtype:
        raise ValueError(f"k_new/v_new must be {shape} of one dtype")
    _check(lib().cca_kv_append_rope(ring.handle, _ptr(k_new, "k_new"), _ptr(v_new, "v_new"), _src_dtype(k_new),
                                    _ptr(pos, "pos", torch.int32), _ptr(freq, "freq", torch.float32),
                                    _stream(stream)), "cca_kv_append_rope")


def cca_quant_e4m3(x: torch.Tensor, x8: Optional[torch.Tensor] = None, scale: Optional[torch.Tensor] = None,
                   stream=None):
    """Per-head absmax e4m3 quantisation of x [n, H, D] -> (codes uint8, scale fp32 [H])."""
    n, h, d = x.shape
    if x8 is None:
        x8 = torch.empty((n, h, d), dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty(h, dtype=torch.float32, device=x.device)
    _check(lib().cca_quant_e4m3(_ptr(x, "x"), _src_dtype(x), n, h, d, _ptr(x8, "x8", torch.uint8),
                                _ptr(scale, "scale", torch.float32), _stream(stream)), "cca_quant_e4m3")
    return x8, scale


def cca_quant_e4m3_f16(x: torch.Tensor, x16: Optional[torch.Tensor] = None, scale: Optional[torch.Tensor] = None,
                       stream=None):
    """Per-head absmax e4m3 quantisation of x [n, H, D] returning the codes' values
    widened to fp16 (the V-side form of E4M3 attention) and the scales."""
    n, h, d = x.shape
    if x16 is None:
        x16 = torch.empty((n, h, d), dtype=torch.float16, device=x.device)
    if scale is None:
        scale = torch.empty(h, dtype=torch.float32, device=x.device)
    _check(lib().cca_quant_e4m3_f16(_ptr(x, "x"), _src_dtype(x), n, h, d, _ptr(x16, "x16", torch.float16),
                                    _ptr(scale, "scale", torch.float32), _stream(stream)), "cca_quant_e4m3_f16")
    return x16, scale


def cca_quant_e4m3_qkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, stream=None):
    """The three inputs of an E4M3 attention call quantised in one launch:
    returns (q8, q_scale, k8, k_scale, v16, v_scale), the same values as
    cca_quant_e4m3(q), cca_quant_e4m3(k) and cca_quant_e4m3_f16(v)."""
    n, h, d = q.shape
    if k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("cca_quant_e4m3_qkv: q, k and v must share shape and dtype")
    q8 = torch.empty((n, h, d), dtype=torch.uint8, device=q.device)
    k8 = torch.empty_like(q8)
    v16 = torch.empty((n, h, d), dtype=torch.float16, device=q.device)
    qs, ks, vs = (torch.empty(h, dtype=torch.float32, device=q.device) for _ in range(3))
    _check(lib().cca_quant_e4m3_qkv(_ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _src_dtype(q), n, h, d,
                                    _ptr(q8, "q8", torch.uint8), _ptr(k8, "k8", torch.uint8),
                                    _ptr(v16, "v16", torch.float16), _ptr(qs, "q_scale", torch.float32),
                                    _ptr(ks, "k_scale", torch.float32), _ptr(vs, "v_scale", torch.float32),
                                    _stream(stream)), "cca_quant_e4m3_qkv")
    return q8, qs, k8, ks, v16, vs


def cca_chunk_attn_workspace_size(ring: KVRing, n_q_max: int) -> int:
    out = ctypes.c_size_t()
    _check(lib().cca_chunk_attn_workspace_size(ring.handle, int(n_q_max), ctypes.byref(out)),
           "cca_chunk_attn_workspace_size")
    return int(out.value)


def cca_chunk_attn(ring: KVRing, q: torch.Tensor, k_cur: torch.Tensor, v_cur: torch.Tensor,
                   q_scale=None, kcur_scale=None, vcur_scale=None, q_idx: Optional[torch.Tensor] = None,
                   n_q_dev: Optional[torch.Tensor] = None, n_q_max: Optional[int] = None,
                   softmax_scale: float = 0.0, out: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Attention of the current chunk's queries over sink + window + current chunk.

    q / k_cur / v_cur: [L, H, D] in the ring's dtype (bf16, or uint8 e4m3 codes
    with per-head fp32 scales).  q_idx (int32) selects query rows; n_q_dev
    (int32[1], device) bounds their count without a host sync.  Returns out
    [n_q_max, H, D] bf16.
    """
    if n_q_max is None:
        n_q_max = q_idx.shape[0] if q_idx is not None else q.shape[0]
    if out is None:
        out = torch.empty((n_q_max, ring.n_heads, ring.head_dim), dtype=torch.bfloat16, device=q.device)
    need = cca_chunk_attn_workspace_size(ring, n_q_max)
    if need > 0 and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().cca_chunk_attn(ring.handle, _ptr(q, "q"), _ptr(k_cur, "k_cur"), _ptr(v_cur, "v_cur"),
                                _ptr(q_scale, "q_scale"), _ptr(kcur_scale, "kcur_scale"),
                                _ptr(vcur_scale, "vcur_scale"), _ptr(q_idx, "q_idx", torch.int32),
                                _ptr(n_q_dev, "n_q_dev", torch.int32), int(n_q_max), float(softmax_scale),
                                _ptr(out, "out", torch.bfloat16), _ptr(workspace, "workspace"), ws_bytes,
                                _stream(stream)), "cca_chunk_attn")
    return out


def cca_chunk_attn_scatter(ring: KVRing, q: torch.Tensor, k_cur: torch.Tensor, v_cur: torch.Tensor,
                           q_idx: torch.Tensor, o_cache: torch.Tensor, q_scale=None, kcur_scale=None,
                           vcur_scale=None, n_q_dev: Optional[torch.Tensor] = None, n_q_max: Optional[int] = None,
                           softmax_scale: float = 0.0, workspace: Optional[torch.Tensor] = None,
                           stream=None) -> torch.Tensor:
    """Active-query attention whose result for query i lands in row q_idx[i] of
    o_cache ([L, H, D] bf16, updated in place); other rows are left as they are."""
    if n_q_max is None:
        n_q_max = q_idx.shape[0]
    need = cca_chunk_attn_workspace_size(ring, n_q_max)
    if need > 0 and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().cca_chunk_attn_scatter(ring.handle, _ptr(q, "q"), _ptr(k_cur, "k_cur"), _ptr(v_cur, "v_cur"),
                                        _ptr(q_scale, "q_scale"), _ptr(kcur_scale, "kcur_scale"),
                                        _ptr(vcur_scale, "vcur_scale"), _ptr(q_idx, "q_idx", torch.int32),
                                        _ptr(n_q_dev, "n_q_dev", torch.int32), int(n_q_max), float(softmax_scale),
                                        _ptr(o_cache, "o_cache", torch.bfloat16), _ptr(workspace, "workspace"),
                                        ws_bytes, _stream(stream)), "cca_chunk_attn_scatter")
    return o_cache


def cca_chunk_attn_noalloc(ring: KVRing, q: torch.Tensor, k_cur: torch.Tensor, v_cur: torch.Tensor,
                           q_scale=None, kcur_scale=None, vcur_scale=None, q_idx: Optional[torch.Tensor] = None,
                           n_q_dev: Optional[torch.Tensor] = None, n_q_max: Optional[int] = None,
                           softmax_scale: float = 0.0, out: Optional[torch.Tensor] = None,
                           stream=None) -> torch.Tensor:
    """cca_chunk_attn without a workspace argument: for callers that cannot give
    the library device scratch memory (see include/cca.h).  Scratch comes from an
    array built into libcca.so that all calls share, so calls must not overlap on
    the GPU.  ``out`` must be provided by callers that may not allocate at all."""
    if n_q_max is None:
        n_q_max = q_idx.shape[0] if q_idx is not None else q.shape[0]
    if out is None:
        out = torch.empty((n_q_max, ring.n_heads, ring.head_dim), dtype=torch.bfloat16, device=q.device)
    _check(lib().cca_chunk_attn_noalloc(ring.handle, _ptr(q, "q"), _ptr(k_cur, "k_cur"), _ptr(v_cur, "v_cur"),
                                        _ptr(q_scale, "q_scale"), _ptr(kcur_scale, "kcur_scale"),
                                        _ptr(vcur_scale, "vcur_scale"), _ptr(q_idx, "q_idx", torch.int32),
                                        _ptr(n_q_dev, "n_q_dev", torch.int32), int(n_q_max), float(softmax_scale),
                                        _ptr(out, "out", torch.bfloat16), _stream(stream)),
           "cca_chunk_attn_noalloc")
    return out


def cca_attn_workspace_size(head_dim: int) -> int:
    out = ctypes.c_size_t()
    _check(lib().cca_attn_workspace_size(int(head_dim), ctypes.byref(out)), "cca_attn_workspace_size")
    return int(out.value)


def _workspace(workspace, head_dim, device):
    need = cca_attn_workspace_size(head_dim)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


def cca_chunk_attn_groups(ring: KVRing, q: torch.Tensor, k_cur: torch.Tensor, v_cur: torch.Tensor,
                          k_ref: Optional[torch.Tensor] = None, v_ref: Optional[torch.Tensor] = None,
                          q_scale=None, kcur_scale=None, vcur_scale=None, kref_scale=None, vref_scale=None,
                          softmax_scale: float = 0.0, out: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One denoising step of the active chunk's token groups (N_t, S_t, C_t packed
    as the n_cur rows of q / k_cur / v_cur) over R (k_ref / v_ref, optional), the
    ring's sink and window, and the block itself.  Returns out [n_cur, H, D] bf16."""
    n_cur = q.shape[0]
    if tuple(k_cur.shape) != tuple(q.shape) or tuple(v_cur.shape) != tuple(q.shape):
        raise ValueError("q, k_cur and v_cur must have the same shape [n_cur, H, D]")
    n_ref = 0 if k_ref is None else k_ref.shape[0]
    if out is None:
        out = torch.empty((n_cur, ring.n_heads, ring.head_dim), dtype=torch.bfloat16, device=q.device)
    workspace, ws_bytes = _workspace(workspace, ring.head_dim, q.device)
    _check(lib().cca_chunk_attn_groups(ring.handle, _ptr(q, "q"), _ptr(k_cur, "k_cur"), _ptr(v_cur, "v_cur"),
                                       int(n_cur), _ptr(k_ref, "k_ref"), _ptr(v_ref, "v_ref"), int(n_ref),
                                       _ptr(q_scale, "q_scale"), _ptr(kcur_scale, "kcur_scale"),
                                       _ptr(vcur_scale, "vcur_scale"), _ptr(kref_scale, "kref_scale"),
                                       _ptr(vref_scale, "vref_scale"), float(softmax_scale),
                                       _ptr(out, "out", torch.bfloat16), _ptr(workspace, "workspace"), ws_bytes,
                                       _stream(stream)), "cca_chunk_attn_groups")
    return out


def cca_block_attn(q: torch.Tensor, k_cur: torch.Tensor, v_cur: torch.Tensor, window: int,
                   k_hist: Optional[torch.Tensor] = None, v_hist: Optional[torch.Tensor] = None,
                   k_ref: Optional[torch.Tensor] = None, v_ref: Optional[torch.Tensor] = None,
                   q_scale=None, kcur_scale=None, vcur_scale=None, khist_scale=None, vhist_scale=None,
                   kref_scale=None, vref_scale=None, softmax_scale: float = 0.0,
                   out: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Packed block-causal forward: q / k_cur / v_cur [T, L, H, D]; chunk c attends
    to R, history chunks {0} U {max(1, c-W) .. c-1} (k_hist / v_hist, default the
    current tensors) and itself.  Returns out [T, L, H, D] bf16."""
    T, L, H, D = q.shape
    fp8 = q.dtype == torch.uint8  # e4m3: q/k codes, v fp16-widened values
    if k_hist is None:
        k_hist, v_hist, khist_scale, vhist_scale = k_cur, v_cur, kcur_scale, vcur_scale
    if out is None:
        out = torch.empty((T, L, H, D), dtype=torch.bfloat16, device=q.device)
    workspace, ws_bytes = _workspace(workspace, D, q.device)
    d = _BlockDesc(H, D, L, T, int(window), CCA_E4M3 if fp8 else CCA_BF16,
                   _ptr(k_cur, "k_cur"), _ptr(v_cur, "v_cur"), _ptr(k_hist, "k_hist"), _ptr(v_hist, "v_hist"),
                   _ptr(k_ref, "k_ref"), _ptr(v_ref, "v_ref"), 0 if k_ref is None else int(k_ref.shape[0]),
                   _ptr(kcur_scale, "kcur_scale"), _ptr(vcur_scale, "vcur_scale"),
                   _ptr(khist_scale, "khist_scale"), _ptr(vhist_scale, "vhist_scale"),
                   _ptr(kref_scale, "kref_scale"), _ptr(vref_scale, "vref_scale"),
                   _ptr(status, "status", torch.int32))
    _check(lib().cca_block_attn(ctypes.byref(d), _ptr(q, "q"), _ptr(q_scale, "q_scale"), float(softmax_scale),
                                _ptr(out, "out", torch.bfloat16), _ptr(workspace, "workspace"), ws_bytes,
                                _stream(stream)), "cca_block_attn")
    return out


def cca_token_mask_l2(src: torch.Tensor, edit: torch.Tensor, tau: float = 0.0, prune_quantile: float = -1.0,
                      mask: Optional[torch.Tensor] = None, dist2: Optional[torch.Tensor] = None,
                      tau_out: Optional[torch.Tensor] = None, stream=None):
    """mask[u] = ||edit_u - src_u||_2 > tau (fixed) or > the ceil(q*N)-th smallest distance."""
    n, c = src.shape
    if mask is None:
        mask = torch.empty(n, dtype=torch.uint8, device=src.device)
    _check(lib().cca_token_mask_l2(_ptr(src, "src", torch.float32), _ptr(edit, "edit", torch.float32), n, c,
                                   float(tau), float(prune_quantile), _ptr(mask, "mask", torch.uint8),
                                   _ptr(dist2, "dist2", torch.float32), _ptr(tau_out, "tau_out", torch.float32),
                                   _stream(stream)), "cca_token_mask_l2")
    return mask


def cca_token_mask_l2_frames(src: torch.Tensor, edit: torch.Tensor, tau: float = 0.0, prune_quantile: float = -1.0,
                             mask: Optional[torch.Tensor] = None, dist2: Optional[torch.Tensor] = None,
                             tau_out: Optional[torch.Tensor] = None, stream=None):
    """Mask of a multi-frame chunk: src / edit [F, N, C]; one decision per position
    from the norm over all frames and channels, written for every frame: [F * N] uint8."""
    f, n, c = src.shape
    if mask is None:
        mask = torch.empty(f * n, dtype=torch.uint8, device=src.device)
    _check(lib().cca_token_mask_l2_frames(_ptr(src, "src", torch.float32), _ptr(edit, "edit", torch.float32), f, n,
                                          c, float(tau), float(prune_quantile), _ptr(mask, "mask", torch.uint8),
                                          _ptr(dist2, "dist2", torch.float32),
                                          _ptr(tau_out, "tau_out", torch.float32), _stream(stream)),
           "cca_token_mask_l2_frames")
    return mask


def cca_compact_workspace_size(n_tok: int) -> int:
    out = ctypes.c_size_t()
    _check(lib().cca_compact_workspace_size(int(n_tok), ctypes.byref(out)), "cca_compact_workspace_size")
    return int(out.value)


def cca_compact(mask: torch.Tensor, idx: Optional[torch.Tensor] = None, n_active: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, stream=None):
    """Ascending active positions (int32 [n_tok], first n valid) and the count (device int32[1])."""
    n = mask.shape[0]
    if idx is None:
        idx = torch.empty(max(n, 1), dtype=torch.int32, device=mask.device)
    if n_active is None:
        n_active = torch.empty(1, dtype=torch.int32, device=mask.device)
    need = cca_compact_workspace_size(n)
    if need > 0 and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=mask.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().cca_compact(_ptr(mask, "mask", torch.uint8), n, _ptr(idx, "idx", torch.int32),
                             _ptr(n_active, "n_active", torch.int32), _ptr(workspace, "workspace"), ws_bytes,
                             _stream(stream)), "cca_compact")
    return idx, n_active


def cca_scatter(o_compact: torch.Tensor, idx: torch.Tensor, n_active: torch.Tensor, o_cache: torch.Tensor,
                n_max: Optional[int] = None, stream=None) -> torch.Tensor:
    """o_cache[idx[i]] = o_compact[i] for i < n_active (in place)."""
    if n_max is None:
        n_max = o_compact.shape[0]
    row_bytes = o_cache[0].numel() * o_cache.element_size()
    if o_compact.dtype != o_cache.dtype or o_compact[0].numel() != o_cache[0].numel():
        raise ValueError("o_compact and o_cache rows must match")
    _check(lib().cca_scatter(_ptr(o_compact, "o_compact"), _ptr(idx, "idx", torch.int32),
                             _ptr(n_active, "n_active", torch.int32), int(n_max), int(row_bytes),
                             _ptr(o_cache, "o_cache"), _stream(stream)), "cca_scatter")
    return o_cache


def cca_selftest_bounded_wait(status: torch.Tensor, budget_cycles: int, arrive_first: bool = False,
                              stream=None) -> None:
    """Run the bounded-wait self-test; status (int32[1], device) gets CCA_DEV_*."""
    _check(lib().cca_selftest_bounded_wait(_ptr(status, "status", torch.int32), int(budget_cycles),
                                           1 if arrive_first else 0, _stream(stream)), "cca_selftest_bounded_wait")
