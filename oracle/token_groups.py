"""Oracle: attention under the token-group mask, one step or a packed sequence.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Restated from ["JoyAI-Video-Edit 소개", section 세 부품으로 이루어진 아키텍처]
(the attention-mask figure: the sequence holds noisy tokens N_t, the global
tokens H_0, history tokens H_{t-1}, MLLM condition tokens C_t, reference VAE
tokens R and source-video VAE tokens S_t; the mask says which group sees which)
and section 청크 단위 자기회귀 적응 (in training the noisy active chunk, its
source tokens S_t, condition tokens C_t, the optional reference tokens R and the
clean history H_{<t} form one sequence; the active chunk sees its own source and
condition tokens in both directions and the windowed history and the global
sink causally; future chunks are masked; only R is open to every query; each
target chunk has its own noise level).

The figure itself is not in the text, so the rule is the plainest reading of
those sentences (each reading is also listed with the others of this build):

* the active block of chunk t is {N_t, S_t, C_t}; every query of it sees every
  key of it (bidirectional);
* it sees the clean history chunks H_c for c in {0} U {max(1, t-W) .. t-1}
  (H_0 is the global sink; W recent chunks besides it);
* every query sees R; R's own queries see R only;
* a clean history chunk H_c, when its queries are computed (the packed
  training sequence), sees H_c' for c' in {0} U {max(1, c-W) .. c-1} U {c};
* nothing else is visible (future chunks, other chunks' N/S/C groups).

Attention over a sequence with that mask is the plain definition: for each
query, softmax over the scores of the keys it may see, times their values.
The functions below build the element mask from the group labels and apply it
to a dense fp64 score matrix; they do not reuse ``chunk_attention``.

Pins (``tests/test_oracle_groups.py``): brute force in pure Python on tiny
inputs; with no S, C and R the step equals the plain chunk-causal attention;
with history equal to the current chunks and a full window the packed forward
equals block-causal attention written as an explicit mask over chunk indices;
invariances (perturbing a masked group changes nothing, perturbing R changes
every row, rows sum to one).
"""

from __future__ import annotations

import math
from typing import Sequence

import numpy as np

ACTIVE = ("N", "S", "C")


def history_of(t: int, window: int) -> list[int]:
    """Clean history chunks the active chunk t sees: {0} U {max(1, t-W) .. t-1}, minus t."""
    if t < 0 or window < 0:
        raise ValueError("t and window must be non-negative")
    if t == 0:
        return []
    return sorted({0} | set(range(max(1, t - window), t)))


def sees(qg: tuple, kg: tuple, window: int) -> bool:
    """Whether a query of group ``qg`` may attend to a key of group ``kg``.

    Groups are tuples: ("N", t), ("S", t), ("C", t) for the active block of
    chunk t, ("H", c) for clean chunk c, ("R",) for the reference tokens.
    """
    if kg[0] == "R":
        return True
    if qg[0] == "R":
        return False
    if qg[0] in ACTIVE:
        t = qg[1]
        if kg[0] in ACTIVE:
            return kg[1] == t
        if kg[0] == "H":
            return kg[1] in history_of(t, window)
        return False
    if qg[0] == "H":
        c = qg[1]
        return kg[0] == "H" and (kg[1] == c or kg[1] in history_of(c, window))
    raise ValueError(f"unknown group {qg}")


def element_mask(q_groups: Sequence[tuple], k_groups: Sequence[tuple], window: int) -> np.ndarray:
    """Boolean [Lq, Lk] mask from per-token group labels."""
    uq = sorted(set(q_groups), key=repr)
    uk = sorted(set(k_groups), key=repr)
    table = {(a, b): sees(a, b, window) for a in uq for b in uk}
    m = np.zeros((len(q_groups), len(k_groups)), dtype=bool)
    for i, a in enumerate(q_groups):
        for b in uk:
            if table[(a, b)]:
                m[i, [j for j, g in enumerate(k_groups) if g == b]] = True
    return m


def masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray,
                     scale: float | None = None) -> np.ndarray:
    """Dense softmax attention with an element mask, fp64.  q [Lq,H,D], k/v [Lk,H,D],
    mask [Lq, Lk] (every row must see at least one key)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    lq, h, d = q.shape
    if not mask.any(axis=1).all():
        raise ValueError("a query sees no key")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.empty((lq, h, d), dtype=np.float64)
    for hh in range(h):
        s = (q[:, hh, :] @ k[:, hh, :].T) * scale
        s = np.where(mask, s, -np.inf)
        s -= s.max(axis=1, keepdims=True)
        p = np.where(mask, np.exp(s), 0.0)
        p /= p.sum(axis=1, keepdims=True)
        out[:, hh, :] = p @ v[:, hh, :]
    return out


def sequence_attention(tokens: Sequence[tuple], window: int, query_groups=None, scale: float | None = None):
    """Attention over a packed sequence given as (group, q, k, v) blocks.

    Every block contributes its keys; the queries of the blocks whose group is
    in ``query_groups`` (all when None) are computed.  Returns the list of
    outputs of those blocks, in order.
    """
    qs, ks, vs, q_lab, k_lab, spans = [], [], [], [], [], []
    for g, q, k, v in tokens:
        ks.append(np.asarray(k))
        vs.append(np.asarray(v))
        k_lab += [g] * len(k)
        if query_groups is None or g in query_groups:
            spans.append((len(q_lab), len(q_lab) + len(q)))
            qs.append(np.asarray(q))
            q_lab += [g] * len(q)
    mask = element_mask(q_lab, k_lab, window)
    o = masked_attention(np.concatenate(qs), np.concatenate(ks), np.concatenate(vs), mask, scale)
    return [o[a:b] for a, b in spans]


def step_attention(t: int, window: int, active: Sequence[tuple], history: dict, ref=None,
                   scale: float | None = None) -> np.ndarray:
    """Outputs of the active block of chunk t at one denoising step.

    active: [(name, q, k, v)] for the groups of chunk t present ("N", "S", "C"),
        in the order their rows are packed; the result rows follow that order.
    history: {c: (k, v)} clean chunks (entries outside the visible set unused).
    ref: (q, k, v) of R or None (R's queries are not computed here).
    """
    toks = []
    if ref is not None:
        toks.append((("R",), ref[0], ref[1], ref[2]))
    for c in history_of(t, window):
        k, v = history[c]
        toks.append((("H", c), np.zeros((0,) + np.shape(k)[1:]), k, v))
    for name, q, k, v in active:
        toks.append(((name, t), q, k, v))
    outs = sequence_attention(toks, window, query_groups={(n, t) for n, _, _, _ in active}, scale=scale)
    return np.concatenate(outs)


def packed_forward(q: np.ndarray, k_cur: np.ndarray, v_cur: np.ndarray, k_hist: np.ndarray, v_hist: np.ndarray,
                   window: int, ref=None, scale: float | None = None) -> np.ndarray:
    """Training-time packed forward of T chunks ([T, L, H, D] arrays): the queries
    of noisy chunk c (group N_c) over R, the clean history H and N_c itself.
    Returns [T, L, H, D]."""
    T = q.shape[0]
    toks = []
    if ref is not None:
        toks.append((("R",), ref[0], ref[1], ref[2]))
    for c in range(T):
        toks.append((("H", c), np.zeros((0,) + q.shape[2:]), k_hist[c], v_hist[c]))
    for c in range(T):
        toks.append((("N", c), q[c], k_cur[c], v_cur[c]))
    outs = sequence_attention(toks, window, query_groups={("N", c) for c in range(T)}, scale=scale)
    return np.stack(outs)


def clean_forward(q: np.ndarray, k: np.ndarray, v: np.ndarray, window: int, ref=None,
                  scale: float | None = None) -> np.ndarray:
    """Outputs of the clean history chunks themselves in the packed sequence:
    H_c over R and H_{c'} for c' in {0} U {max(1, c-W) .. c}."""
    T = q.shape[0]
    toks = []
    if ref is not None:
        toks.append((("R",), ref[0], ref[1], ref[2]))
    for c in range(T):
        toks.append((("H", c), q[c], k[c], v[c]))
    outs = sequence_attention(toks, window, query_groups={("H", c) for c in range(T)}, scale=scale)
    return np.stack(outs)


def ref_self_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float | None = None) -> np.ndarray:
    """R's own queries: they see R only."""
    return sequence_attention([(("R",), q, k, v)], 0, scale=scale)[0]
