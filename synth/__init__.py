"""Seeded synthetic workloads for chunk-causal attention and the L2 mask cache.

This package only draws random inputs (numpy ``Generator(PCG64(seed))``); it
holds none of the method's arithmetic.  Both the fp64 oracle side and the CUDA
side of every test, ``bench.py`` and ``__graft_entry__.smoke()`` take their
inputs from here, so parity compares the two implementations on identical
values.  All floating inputs are returned as float32 numpy arrays whose values
are exactly representable in the dtype the GPU consumes (bf16 rounding is done
here, with round-to-nearest-even, via torch's CPU conversion).

Shapes follow the pages' deployment setting where they fix one: a 720x1280 frame
under 24x24 spatial VAE compression gives a 30 x ceil(1280/24) = 30 x 54 = 1620
token latent grid per chunk, one latent frame (8 video frames) per chunk
["JoyAI-Video-Edit 소개", section 세 부품으로 이루어진 아키텍처].  Head count,
head size and window are not on the pages; the workloads use 24 heads of 128 and
a 3-chunk window plus the sink.

Workloads (seed = index):
  0 tiny      H=1, D=64, 16 tokens/chunk, 4 chunks, W=2; 16x16 latents, tau=1.0
  1 720p      H=24, D=128, 1620 tokens, W=3; ring holds chunks 0..3, current t=4,
              2 denoising steps with fresh Q, K_cur, V_cur; per-head RMS 1, bf16
  2 stream    720p shape for 225 chunks; K/V follow AR(1): 0.9 x_{t-1} + 0.44 N(0,1)
  3 fp8       720p shape with Student-t(nu=4) Q/K/V at raw scale
  4 mask      1620x16 fp32 source/edit latents on the 30x54 grid; 1-4 random
              ellipses covering 30 % +- 2 % get offset N(2,1), background N(0,0.1);
              Q/K/V of workload 1; cached outputs N(0, 0.02^2) bf16
  5 groups    the 720p chunk t=4 with its token groups: N_t (1620 noisy tokens),
              S_t (1620 source tokens), C_t (256 condition tokens) and R (1620
              reference tokens); ring = clean chunks 0..3; per-head RMS 1, bf16
  6 packed    T=8 chunks of the 720p shape in one sequence (teacher forcing):
              noisy Q/K/V and clean K/V [T, 1620, 24, 128], per-head RMS 1, bf16
  7 liveedit  LiveEdit-shaped chunk: 3 latent frames of the 30x54 grid = 4860
              tokens, 24 heads x 128, sink + 2-chunk window, current t=3, 4
              denoising steps; mask latents [3, 1620, 16] with the workload-4
              ellipse recipe (the region held over the 3 frames), dynamic tau 70 %
"""

from __future__ import annotations

import dataclasses

import numpy as np
import torch

GRID_H, GRID_W = 30, 54
TOKENS_720P = GRID_H * GRID_W  # 1620


def rng(*seed) -> np.random.Generator:
    """PCG64 generator from an int or a tuple of ints (independent streams)."""
    return np.random.Generator(np.random.PCG64(list(seed) if len(seed) > 1 else seed[0]))


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (RNE) and return them as float32."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def _head_rms_one(x: np.ndarray) -> np.ndarray:
    """Rescale each head of x [L, H, D] to RMS exactly 1 (before bf16 rounding)."""
    x = x.astype(np.float64)
    rms = np.sqrt(np.mean(x * x, axis=(0, 2), keepdims=True))
    return (x / rms).astype(np.float32)


# ---------------------------------------------------------------- workload 0
@dataclasses.dataclass
class TinyStream:
    n_heads: int
    head_dim: int
    chunk_len: int
    window: int
    q: list  # per chunk [L, H, D] (bf16 values as float32)
    k: list
    v: list
    src: np.ndarray  # [16, 16] fp32 latents
    edit: np.ndarray
    tau: float


def tiny(seed: int = 0, n_chunks: int = 4, n_heads: int = 1, head_dim: int = 64,
         chunk_len: int = 16, window: int = 2) -> TinyStream:
    g = rng(seed)
    shape = (chunk_len, n_heads, head_dim)
    q = [bf16_round(g.standard_normal(shape, dtype=np.float32)) for _ in range(n_chunks)]
    k = [bf16_round(g.standard_normal(shape, dtype=np.float32)) for _ in range(n_chunks)]
    v = [bf16_round(g.standard_normal(shape, dtype=np.float32)) for _ in range(n_chunks)]
    src = g.standard_normal((16, 16), dtype=np.float32)
    edit = (src + g.normal(0.0, 0.25, size=(16, 16))).astype(np.float32)
    return TinyStream(n_heads, head_dim, chunk_len, window, q, k, v, src, edit, 1.0)


# ---------------------------------------------------------------- workload 1
@dataclasses.dataclass
class Chunk720p:
    n_heads: int
    head_dim: int
    chunk_len: int
    window: int
    ring_k: list  # chunks 0..3 appended before the measured chunk
    ring_v: list
    t: int  # index of the current chunk (= number of appended chunks)
    q: list  # per denoising step [L, H, D]
    k_cur: list
    v_cur: list


def chunk_720p(seed: int = 1, n_steps: int = 2, n_heads: int = 24, head_dim: int = 128,
               chunk_len: int = TOKENS_720P, window: int = 3, n_prefill: int = 4,
               heavy_tailed: bool = False) -> Chunk720p:
    """Workload 1 (and 3 with ``heavy_tailed``): ring prefilled, one current chunk."""
    g = rng(seed)
    shape = (chunk_len, n_heads, head_dim)

    def draw():
        if heavy_tailed:
            return bf16_round(g.standard_t(4.0, size=shape).astype(np.float32))
        return bf16_round(_head_rms_one(g.standard_normal(shape, dtype=np.float32)))

    ring_k, ring_v = [], []
    for _ in range(n_prefill):
        ring_k.append(draw())
        ring_v.append(draw())
    q, kc, vc = [], [], []
    for _ in range(n_steps):
        q.append(draw())
        kc.append(draw())
        vc.append(draw())
    return Chunk720p(n_heads, head_dim, chunk_len, window, ring_k, ring_v, n_prefill, q, kc, vc)


def fp8_720p(seed: int = 3, **kw) -> Chunk720p:
    """Workload 3: the 720p chunk with Student-t(4) inputs at raw scale."""
    return chunk_720p(seed=seed, heavy_tailed=True, **kw)


# ---------------------------------------------------------------- workload 2
class LongStream:
    """Workload 2: K/V of chunk t = 0.9 x_{t-1} + 0.44 N(0,1) (float32), bf16-cached.

    Chunks are produced in order by ``next_kv()``; queries of any (chunk, step)
    come from their own seeded stream so they can be drawn lazily.
    """

    def __init__(self, seed: int = 2, n_heads: int = 24, head_dim: int = 128,
                 chunk_len: int = TOKENS_720P, window: int = 3, n_chunks: int = 225):
        self.seed = seed
        self.shape = (chunk_len, n_heads, head_dim)
        self.n_heads, self.head_dim, self.chunk_len = n_heads, head_dim, chunk_len
        self.window, self.n_chunks = window, n_chunks
        self._t = 0
        self._xk = None
        self._xv = None

    def next_kv(self):
        g = rng(self.seed, self._t, 0)
        nk = g.standard_normal(self.shape, dtype=np.float32)
        nv = g.standard_normal(self.shape, dtype=np.float32)
        if self._t == 0:
            self._xk, self._xv = nk, nv
        else:
            self._xk = (np.float32(0.9) * self._xk + np.float32(0.44) * nk).astype(np.float32)
            self._xv = (np.float32(0.9) * self._xv + np.float32(0.44) * nv).astype(np.float32)
        self._t += 1
        return bf16_round(self._xk), bf16_round(self._xv)

    def query(self, t: int, step: int) -> np.ndarray:
        return bf16_round(rng(self.seed, t, 1 + step).standard_normal(self.shape, dtype=np.float32))


# ---------------------------------------------------------------- workload 4
@dataclasses.dataclass
class MaskChunk:
    src: np.ndarray  # [1620, 16] fp32, previous chunk's source latents
    edit: np.ndarray  # [1620, 16] fp32, previous chunk's edited latents
    region: np.ndarray  # [1620] bool, union of the ellipses (for reporting only)
    prune_quantile: float
    o_cache: np.ndarray  # [1620, H, D] bf16 values: outputs cached at chunk k-1


def _ellipse_union(centres, axes, angles, lam):
    yy, xx = np.meshgrid(np.arange(GRID_H) + 0.5, np.arange(GRID_W) + 0.5, indexing="ij")
    inside = np.zeros((GRID_H, GRID_W), dtype=bool)
    for (cy, cx), (a, b), th in zip(centres, axes, angles):
        dy, dx = yy - cy, xx - cx
        u = dx * np.cos(th) + dy * np.sin(th)
        w = -dx * np.sin(th) + dy * np.cos(th)
        inside |= (u / (lam * a)) ** 2 + (w / (lam * b)) ** 2 <= 1.0
    return inside.reshape(-1)


def mask_chunk(seed: int = 4, n_ch: int = 16, n_heads: int = 24, head_dim: int = 128,
               coverage: float = 0.30, tol: float = 0.02) -> MaskChunk:
    g = rng(seed)
    n = GRID_H * GRID_W
    src = g.standard_normal((n, n_ch), dtype=np.float32)
    n_ell = int(g.integers(1, 5))
    centres = np.stack([g.uniform(0, GRID_H, n_ell), g.uniform(0, GRID_W, n_ell)], axis=1)
    axes = np.stack([g.uniform(0.3, 1.0, n_ell) * GRID_W / 4, g.uniform(0.3, 1.0, n_ell) * GRID_H / 4], axis=1)
    angles = g.uniform(0, np.pi, n_ell)
    lo, hi = 0.0, 8.0
    region = _ellipse_union(centres, axes, angles, hi)
    for _ in range(60):  # bisection on a common scale of the semi-axes
        mid = 0.5 * (lo + hi)
        region = _ellipse_union(centres, axes, angles, mid)
        cov = region.mean()
        if abs(cov - coverage) <= tol:
            break
        lo, hi = (mid, hi) if cov < coverage else (lo, mid)
    off_in = g.normal(2.0, 1.0, size=(n, n_ch))
    off_out = g.normal(0.0, 0.1, size=(n, n_ch))
    edit = (src + np.where(region[:, None], off_in, off_out)).astype(np.float32)
    o_cache = bf16_round(g.normal(0.0, 0.02, size=(n, n_heads, head_dim)).astype(np.float32))
    return MaskChunk(src, edit, region, 0.70, o_cache)


# ---------------------------------------------------------------- workload 5
@dataclasses.dataclass
class GroupsChunk:
    n_heads: int
    head_dim: int
    chunk_len: int  # tokens of one clean history chunk
    window: int
    ring_k: list  # clean chunks 0..t-1
    ring_v: list
    t: int
    groups: dict  # name -> (q, k, v) [n, H, D] for "N", "S", "C" (packed in that order)
    ref: tuple  # (q, k, v) of R [n_ref, H, D], or None


def groups_chunk(seed: int = 5, n_heads: int = 24, head_dim: int = 128, chunk_len: int = TOKENS_720P,
                 window: int = 3, n_prefill: int = 4, n_src: int = TOKENS_720P, n_cond: int = 256,
                 n_ref: int = TOKENS_720P) -> GroupsChunk:
    """Workload 5: one denoising step of chunk t with all token groups present.
    The MLLM condition tokens count (256) is not on the pages."""
    g = rng(seed)

    def draw(n):
        return bf16_round(_head_rms_one(g.standard_normal((n, n_heads, head_dim), dtype=np.float32)))

    ring_k, ring_v = [], []
    for _ in range(n_prefill):
        ring_k.append(draw(chunk_len))
        ring_v.append(draw(chunk_len))
    groups = {name: (draw(n), draw(n), draw(n)) for name, n in (("N", chunk_len), ("S", n_src), ("C", n_cond))
              if n > 0}
    ref = (draw(n_ref), draw(n_ref), draw(n_ref)) if n_ref > 0 else None
    return GroupsChunk(n_heads, head_dim, chunk_len, window, ring_k, ring_v, n_prefill, groups, ref)


# ---------------------------------------------------------------- workload 6
@dataclasses.dataclass
class PackedSequence:
    window: int
    q: np.ndarray  # [T, L, H, D] queries of the noisy chunks
    k_cur: np.ndarray
    v_cur: np.ndarray
    k_hist: np.ndarray  # clean chunks
    v_hist: np.ndarray


def packed_sequence(seed: int = 6, n_chunks: int = 8, n_heads: int = 24, head_dim: int = 128,
                    chunk_len: int = TOKENS_720P, window: int = 3, heavy_tailed: bool = False) -> PackedSequence:
    """Workload 6: a training-time packed sequence of T chunks."""
    g = rng(seed)
    shape = (n_chunks, chunk_len, n_heads, head_dim)

    def draw():
        if heavy_tailed:
            return bf16_round(g.standard_t(4.0, size=shape).astype(np.float32))
        x = g.standard_normal(shape, dtype=np.float32)
        return bf16_round(np.stack([_head_rms_one(c) for c in x]))

    return PackedSequence(window, draw(), draw(), draw(), draw(), draw())


def grid_positions(t: int, source: int = 0, grid=(GRID_H, GRID_W), n_frames: int = 1) -> np.ndarray:
    """Integer token coordinates (t, h, w, s) of the latent frames t .. t+n_frames-1
    of a chunk on the latent grid, frame-major then row-major: int32 [n, 4]."""
    f, r, c = np.meshgrid(np.arange(n_frames), np.arange(grid[0]), np.arange(grid[1]), indexing="ij")
    n = f.size
    return np.stack([t + f.reshape(n), r.reshape(n), c.reshape(n), np.full(n, source)], axis=1).astype(np.int32)


# ---------------------------------------------------------------- workload 7
@dataclasses.dataclass
class LiveEditChunk:
    n_heads: int
    head_dim: int
    n_frames: int
    chunk_len: int  # n_frames * 1620
    window: int
    ring_k: list
    ring_v: list
    t: int
    q: list  # per denoising step [L, H, D]
    k_cur: list
    v_cur: list
    src: np.ndarray  # [F, 1620, 16] fp32 latents of chunk k-1
    edit: np.ndarray
    prune_quantile: float
    o_cache: np.ndarray  # [L, H, D] bf16 values


def liveedit_chunk(seed: int = 7, n_frames: int = 3, n_steps: int = 4, n_heads: int = 24, head_dim: int = 128,
                   window: int = 2, n_prefill: int = 3, n_ch: int = 16, coverage: float = 0.30,
                   tol: float = 0.02) -> LiveEditChunk:
    """Workload 7.  Chunk size (3 latent frames) and step count (4) are the
    LiveEdit page's; grid, heads, head size, window and channel count are not
    on that page and follow the other workloads."""
    g = rng(seed)
    L = n_frames * TOKENS_720P
    shape = (L, n_heads, head_dim)

    def draw():
        return bf16_round(_head_rms_one(g.standard_normal(shape, dtype=np.float32)))

    ring_k, ring_v = [], []
    for _ in range(n_prefill):
        ring_k.append(draw())
        ring_v.append(draw())
    q, kc, vc = [], [], []
    for _ in range(n_steps):
        q.append(draw())
        kc.append(draw())
        vc.append(draw())
    n = TOKENS_720P
    src = g.standard_normal((n_frames, n, n_ch), dtype=np.float32)
    n_ell = int(g.integers(1, 5))
    centres = np.stack([g.uniform(0, GRID_H, n_ell), g.uniform(0, GRID_W, n_ell)], axis=1)
    axes = np.stack([g.uniform(0.3, 1.0, n_ell) * GRID_W / 4, g.uniform(0.3, 1.0, n_ell) * GRID_H / 4], axis=1)
    angles = g.uniform(0, np.pi, n_ell)
    lo, hi = 0.0, 8.0
    region = _ellipse_union(centres, axes, angles, hi)
    for _ in range(60):
        mid = 0.5 * (lo + hi)
        region = _ellipse_union(centres, axes, angles, mid)
        cov = region.mean()
        if abs(cov - coverage) <= tol:
            break
        lo, hi = (mid, hi) if cov < coverage else (lo, mid)
    off_in = g.normal(2.0, 1.0, size=(n_frames, n, n_ch))
    off_out = g.normal(0.0, 0.1, size=(n_frames, n, n_ch))
    edit = (src + np.where(region[None, :, None], off_in, off_out)).astype(np.float32)
    o_cache = bf16_round(g.normal(0.0, 0.02, size=shape).astype(np.float32))
    return LiveEditChunk(n_heads, head_dim, n_frames, L, window, ring_k, ring_v, n_prefill, q, kc, vc, src, edit,
                         0.70, o_cache)


def as_torch_bf16(x: np.ndarray, device="cpu") -> torch.Tensor:
    """float32 array of bf16 values -> contiguous bf16 tensor (exact)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).to(device)
