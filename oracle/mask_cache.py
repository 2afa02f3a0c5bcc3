"""Oracle: the AR-oriented mask cache (per-token L2 mask, compaction, scatter).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Restated from ["LiveEdit 실시간 Diffusion 기반 스트리밍 비디오 편집", sections
핵심 기여, 방법론 and 기술 상세]:

* for chunk k, the binary edit mask at spatial token (u, v) is 1 exactly when the
  L2 norm of (edited latent - source latent) of chunk k-1 at that token is
  strictly greater than a threshold tau;
* tau is set dynamically from how redundant tokens are between chunks, pruning
  about 70 % of the tokens (the rule itself is not given);
* tokens with mask 1 get the full computation; tokens with mask 0 reuse the
  feature cached for them at chunk k-1; only the self-attention output is cached
  (caching the FFN output degraded quality in the ablation).

Readings where the pages are open:

* the norm runs over all latent channels of a token (one decision per token);
* dynamic tau is the k-th smallest distance with ``k = ceil(q * N)`` computed in
  binary64 (no interpolation), q = 0.70 by default, so exactly ``N - k`` tokens
  are active when distances are distinct; ties at tau stay inactive because the
  comparison is strict;
* the first chunk has no previous latents: every token is active (the caller
  skips the mask);
* compaction lists active positions in ascending order; scatter writes the
  recomputed rows back into the cache, leaving inactive rows untouched.

Pins: the mask equals thresholding ``numpy.linalg.norm`` (a library routine),
also for multi-frame chunks (norm over frames and channels of a position);
with dynamic tau the active count is ``N - k``; ``compact`` equals
``numpy.flatnonzero``; scatter leaves inactive rows bit-identical.
"""

from __future__ import annotations

import math

import numpy as np


def l2_distance(src: np.ndarray, edit: np.ndarray) -> np.ndarray:
    """d_u = sqrt(sum_c (edit[u,c] - src[u,c])^2) in fp64; src/edit: [N, C]."""
    src = np.asarray(src, dtype=np.float64)
    edit = np.asarray(edit, dtype=np.float64)
    if src.shape != edit.shape or src.ndim != 2:
        raise ValueError("src/edit must both be [N, C]")
    diff = edit - src
    return np.sqrt(np.sum(diff * diff, axis=1))


def prune_count(n_tok: int, prune_quantile: float) -> int:
    """k = ceil(q * N) in binary64: number of tokens at or below tau."""
    if not (0.0 < prune_quantile <= 1.0):
        raise ValueError("prune_quantile must lie in (0, 1]")
    return int(math.ceil(prune_quantile * float(n_tok)))


def dynamic_tau(d: np.ndarray, prune_quantile: float) -> float:
    """tau = k-th smallest distance, k = ceil(q * N)."""
    d = np.asarray(d, dtype=np.float64)
    k = prune_count(d.shape[0], prune_quantile)
    return float(np.sort(d)[k - 1])


def token_mask(src: np.ndarray, edit: np.ndarray, tau: float | None = None,
               prune_quantile: float | None = None):
    """Binary mask M_u = [d_u > tau].  Returns (mask uint8 [N], d fp64 [N], tau)."""
    d = l2_distance(src, edit)
    if prune_quantile is not None:
        tau = dynamic_tau(d, prune_quantile)
    if tau is None:
        raise ValueError("give tau or prune_quantile")
    return (d > tau).astype(np.uint8), d, float(tau)


def token_mask_frames(src: np.ndarray, edit: np.ndarray, tau: float | None = None,
                      prune_quantile: float | None = None):
    """Mask of a chunk of several latent frames, src/edit [F, N, C].

    The formula is indexed by spatial position (u, v) only while a chunk holds
    3 latent frames ["LiveEdit ...", section 기술 상세]; the reading used: the
    norm of position p runs over the channels of every frame, and its decision
    applies to the tokens of all frames at p.  Returns (mask uint8 [F * N],
    frame-major; d fp64 [N]; tau).
    """
    src = np.asarray(src, dtype=np.float64)
    edit = np.asarray(edit, dtype=np.float64)
    if src.shape != edit.shape or src.ndim != 3:
        raise ValueError("src/edit must both be [F, N, C]")
    diff = edit - src
    d = np.sqrt(np.sum(diff * diff, axis=(0, 2)))
    if prune_quantile is not None:
        tau = dynamic_tau(d, prune_quantile)
    if tau is None:
        raise ValueError("give tau or prune_quantile")
    m = (d > tau).astype(np.uint8)
    return np.tile(m, src.shape[0]), d, float(tau)


def compact(mask: np.ndarray) -> tuple[np.ndarray, int]:
    """Ascending positions of active tokens and their count."""
    mask = np.asarray(mask)
    idx = [u for u in range(mask.shape[0]) if mask[u] != 0]
    return np.asarray(idx, dtype=np.int32), len(idx)


def scatter(o_compact: np.ndarray, idx: np.ndarray, n_active: int,
            o_cache: np.ndarray) -> np.ndarray:
    """New cache: row idx[i] <- o_compact[i] for i < n_active; other rows kept."""
    out = np.array(o_cache, copy=True)
    for i in range(n_active):
        out[int(idx[i])] = o_compact[i]
    return out
