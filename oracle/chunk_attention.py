"""Oracle: chunk-wise causal attention with a global sink and a sliding window.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Definition restated from ["JoyAI-Video-Edit 소개", section 청크 단위 자기회귀 적응]
and ["論文解説: JoyAI-Video-Edit", step 1 (§4.1)]:

* a video is cut into chunks of ``chunk_len`` latent tokens;
* the tokens of one chunk attend to each other in both directions;
* across chunks attention is causal: chunk ``t`` never sees chunk ``t' > t``;
* to keep the context constant, chunk ``t`` only sees the ``window`` most recent
  history chunks plus chunk 0, which stays visible forever (the global sink).

So the key/value set of chunk ``t`` is the union of the chunks in
``visible_chunks(t, window)``, and attention over that set is ordinary dense
softmax attention (no element mask inside the set).  Readings where the pages
are silent:

* softmax scale ``1/sqrt(head_dim)`` (standard; the pages give none);
* ``window`` counts past non-sink chunks and excludes the current chunk;
* when the window range reaches chunk 0 the sink is counted once (set union);
* Q and K arrive after positional encoding (the M-RoPE formula is not given).

Pins (``tests/test_oracle_pins.py``): a window that covers every past chunk
equals full block-causal attention computed by an independent pure-Python
brute force (explicit element mask); perturbing future or evicted chunks leaves
outputs unchanged; softmax rows sum to one; closed forms (one key, equal keys,
zero query); chunk 0 alone equals ``torch.nn.functional.scaled_dot_product_attention``
in fp64; permuting visible chunks is invariant.
"""

from __future__ import annotations

import math
from typing import Sequence

import numpy as np


def visible_chunks(t: int, window: int) -> list[int]:
    """Chunk indices that chunk ``t`` attends to, ascending.

    {0} (global sink) U {max(1, t - window), ..., t - 1} (recent history)
    U {t} (the chunk itself, bidirectional).
    """
    if t < 0 or window < 0:
        raise ValueError("t and window must be non-negative")
    vis = {0, t}
    vis.update(range(max(1, t - window), t))
    return sorted(vis)


def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                      scale: float | None = None,
                      return_probs: bool = False):
    """Dense multi-head softmax attention in fp64.

    q: [Lq, H, D], k/v: [Lk, H, D] (any float dtype; promoted to fp64).
    Returns o: [Lq, H, D] fp64 (and the probabilities [H, Lq, Lk] if asked).

    Row-wise ``softmax(q k^T * scale) v``.  The row maximum is subtracted before
    ``exp``; softmax is invariant to that shift, so the result is the plain
    definition up to rounding.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if q.ndim != 3 or k.ndim != 3 or v.ndim != 3:
        raise ValueError("expected [L, H, D] arrays")
    lq, h, d = q.shape
    lk = k.shape[0]
    if k.shape != (lk, h, d) or v.shape != (lk, h, d):
        raise ValueError("k/v shape mismatch")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.empty((lq, h, d), dtype=np.float64)
    probs = np.empty((h, lq, lk), dtype=np.float64) if return_probs else None
    for hh in range(h):
        s = (q[:, hh, :] @ k[:, hh, :].T) * scale
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, hh, :] = p @ v[:, hh, :]
        if return_probs:
            probs[hh] = p
    if return_probs:
        return out, probs
    return out


def chunk_attention(q_t: np.ndarray, k_chunks: Sequence[np.ndarray],
                    v_chunks: Sequence[np.ndarray], t: int, window: int,
                    scale: float | None = None,
                    k_cur: np.ndarray | None = None,
                    v_cur: np.ndarray | None = None,
                    return_probs: bool = False):
    """Output of chunk ``t``'s queries under chunk-causal windowed attention.

    ``k_chunks[c]`` / ``v_chunks[c]`` hold chunk ``c``'s keys/values ([L, H, D])
    for every ``c < t`` that exists (entries of chunks outside the visible set
    may be anything, even ``None``: they are never read).  The current chunk's
    keys/values come from ``k_cur``/``v_cur`` when given (at a denoising step
    they are computed from the noisy input), else from ``k_chunks[t]``.
    """
    vis = visible_chunks(t, window)
    ks, vs = [], []
    for c in vis:
        if c == t and k_cur is not None:
            ks.append(np.asarray(k_cur))
            vs.append(np.asarray(v_cur))
        else:
            ks.append(np.asarray(k_chunks[c]))
            vs.append(np.asarray(v_chunks[c]))
    k = np.concatenate(ks, axis=0)
    v = np.concatenate(vs, axis=0)
    return softmax_attention(q_t, k, v, scale=scale, return_probs=return_probs)


def flops_per_call(lq: int, lk: int, n_heads: int, head_dim: int) -> float:
    """Algorithmic FLOPs of one attention call: QK^T and PV, 2 flops per MAC."""
    return 4.0 * lq * lk * n_heads * head_dim
