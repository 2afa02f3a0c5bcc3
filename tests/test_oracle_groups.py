"""Pins of the token-group oracle (``oracle.token_groups``) against what the
pages and plain mathematics fix, independently of the oracle's own rule.

* A brute force in pure Python whose visibility is a hand-written table for one
  tiny scenario (chunk t = 3, window 1: the active block N3/S3/C3 sees R, the
  sink H0 and the window chunk H2, not the evicted H1), checked element by
  element.
* Without S, C and R the step equals the plain chunk-causal attention
  (``oracle.chunk_attention``, itself pinned by brute force).
* The packed forward with the history equal to the current chunks and a window
  covering every chunk equals block-causal attention written as an explicit
  mask M[i, j] = [chunk(j) <= chunk(i)]; with separate history it equals, chunk
  by chunk, the chunk-causal attention over the clean history plus the noisy
  chunk itself.
* Invariances: masked groups can be perturbed freely, R reaches every row,
  softmax rows sum to one; R's own queries equal torch's SDPA over R alone.
* Planted mistakes in the rule (R hidden from the active block, S_t not
  bidirectional, the evicted chunk kept) are caught.
"""

import math

import numpy as np
import pytest
import torch

from oracle import chunk_attention as ca
from oracle import token_groups as tg

H, D = 2, 8


def _draw(g, n):
    return g.standard_normal((n, H, D))


def _brute_step(q_rows, keys, allowed):
    """q_rows: [(group, q_vec[H][D])]; keys: [(group, k[H][D], v[H][D])];
    allowed: {query group: set of key groups}.  Pure-Python softmax per head."""
    out = []
    for gq, qv in q_rows:
        o = np.zeros((H, D))
        for h in range(H):
            s = []
            for gk, kv, vv in keys:
                if gk in allowed[gq]:
                    s.append((sum(qv[h][d] * kv[h][d] for d in range(D)) / math.sqrt(D), vv[h]))
            m = max(x for x, _ in s)
            den = sum(math.exp(x - m) for x, _ in s)
            for x, vv in s:
                w = math.exp(x - m) / den
                for d in range(D):
                    o[h][d] += w * vv[d]
        out.append(o)
    return np.array(out)


def _scenario(seed=0):
    g = np.random.default_rng(seed)
    groups = {"R": 3, "H0": 4, "H1": 4, "H2": 4, "N3": 5, "S3": 4, "C3": 2}
    data = {name: (_draw(g, n), _draw(g, n), _draw(g, n)) for name, n in groups.items()}
    return data


# Hand-written for t = 3, W = 1: history {0} U {max(1, 2) .. 2} = {H0, H2}.
ALLOWED_T3_W1 = {
    "N3": {"R", "H0", "H2", "N3", "S3", "C3"},
    "S3": {"R", "H0", "H2", "N3", "S3", "C3"},
    "C3": {"R", "H0", "H2", "N3", "S3", "C3"},
    "R": {"R"},
}


def _oracle_step(data, rule=None):
    hist = {0: data["H0"][1:], 1: data["H1"][1:], 2: data["H2"][1:]}
    active = [(n, *data[f"{n}3"]) for n in ("N", "S", "C")]
    if rule is None:
        return tg.step_attention(3, 1, active, hist, ref=data["R"])
    saved = tg.sees
    tg.sees = rule
    try:
        return tg.step_attention(3, 1, active, hist, ref=data["R"])
    finally:
        tg.sees = saved


def _brute(data):
    keys = []
    for name in ("R", "H0", "H1", "H2", "N3", "S3", "C3"):
        _, k, v = data[name]
        keys += [(name, k[i], v[i]) for i in range(len(k))]
    rows = []
    for name in ("N3", "S3", "C3"):
        q = data[name][0]
        rows += [(name, q[i]) for i in range(len(q))]
    return _brute_step(rows, keys, ALLOWED_T3_W1)


def test_step_matches_pure_python_brute_force():
    data = _scenario()
    got = _oracle_step(data)
    want = _brute(data)
    assert got.shape == want.shape == (11, H, D)
    assert np.abs(got - want).max() < 1e-12


def test_ref_queries_see_only_ref():
    data = _scenario(1)
    q, k, v = data["R"]
    got = tg.ref_self_attention(q, k, v)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x.transpose(1, 0, 2)))
    want = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v)).numpy().transpose(1, 0, 2)
    assert np.abs(got - want).max() < 1e-12
    rows = [("R", q[i]) for i in range(len(q))]
    keys = [(n, data[n][1][i], data[n][2][i]) for n in ("R", "N3") for i in range(len(data[n][1]))]
    assert np.abs(got - _brute_step(rows, keys, {"R": {"R"}})).max() < 1e-12


def test_without_s_c_r_the_step_is_plain_chunk_attention():
    g = np.random.default_rng(2)
    L, W, t = 6, 2, 5
    k = {c: _draw(g, L) for c in range(t)}
    v = {c: _draw(g, L) for c in range(t)}
    q, kc, vc = _draw(g, L), _draw(g, L), _draw(g, L)
    got = tg.step_attention(t, W, [("N", q, kc, vc)], {c: (k[c], v[c]) for c in range(t)})
    want = ca.chunk_attention(q, k, v, t, W, k_cur=kc, v_cur=vc)
    assert np.abs(got - want).max() < 1e-12


def _block_causal_explicit(q, k, v):
    """[T, L, H, D] -> softmax over keys j with chunk(j) <= chunk(i), explicit mask."""
    T, L = q.shape[:2]
    qf, kf, vf = (x.reshape(T * L, H, D) for x in (q, k, v))
    chunk = np.repeat(np.arange(T), L)
    m = chunk[None, :] <= chunk[:, None]
    out = np.zeros_like(qf)
    for h in range(H):
        s = qf[:, h] @ kf[:, h].T / math.sqrt(D)
        s = np.where(m, s, -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        out[:, h] = p @ vf[:, h]
    return out.reshape(T, L, H, D)


def test_packed_full_window_equals_block_causal():
    g = np.random.default_rng(3)
    T, L = 5, 4
    q, k, v = (g.standard_normal((T, L, H, D)) for _ in range(3))
    got = tg.packed_forward(q, k, v, k, v, window=T)
    assert np.abs(got - _block_causal_explicit(q, k, v)).max() < 1e-12
    # the clean chunks' own outputs follow the same mask
    assert np.abs(tg.clean_forward(q, k, v, window=T) - _block_causal_explicit(q, k, v)).max() < 1e-12


def test_packed_with_separate_history_is_chunkwise_attention():
    g = np.random.default_rng(4)
    T, L, W = 7, 3, 2
    q, kc, vc, kh, vh = (g.standard_normal((T, L, H, D)) for _ in range(5))
    got = tg.packed_forward(q, kc, vc, kh, vh, window=W)
    for c in range(T):
        want = ca.chunk_attention(q[c], list(kh), list(vh), c, W, k_cur=kc[c], v_cur=vc[c])
        assert np.abs(got[c] - want).max() < 1e-12


def test_masked_groups_do_not_matter_and_ref_reaches_every_row():
    data = _scenario(5)
    base = _oracle_step(data)
    d2 = dict(data)
    d2["H1"] = tuple(x + 7.0 for x in data["H1"])  # evicted history chunk
    assert np.array_equal(_oracle_step(d2), base)
    d3 = dict(data)
    d3["R"] = (data["R"][0], data["R"][1], data["R"][2] + 1.0)  # R's values move every output row
    moved = np.abs(_oracle_step(d3) - base).max(axis=(1, 2))
    assert np.all(moved > 1e-6)


def test_rows_sum_to_one():
    data = _scenario(6)
    ones = {n: (q, k, np.ones_like(v)) for n, (q, k, v) in data.items()}
    assert np.abs(_oracle_step(ones) - 1.0).max() < 1e-12


def test_packed_future_chunks_never_matter():
    g = np.random.default_rng(7)
    T, L, W = 6, 3, 2
    q, kc, vc, kh, vh = (g.standard_normal((T, L, H, D)) for _ in range(5))
    base = tg.packed_forward(q, kc, vc, kh, vh, window=W)
    for arr in (kc, vc, kh, vh):
        arr[4:] += 3.0
    got = tg.packed_forward(q, kc, vc, kh, vh, window=W)
    assert np.array_equal(got[:4], base[:4])


_ORIG_SEES = tg.sees
_ORIG_HISTORY = tg.history_of


@pytest.mark.parametrize("plant", ["ref_hidden", "source_one_way", "evicted_kept"])
def test_planted_rule_mistakes_are_caught(plant, monkeypatch):
    def rule(qg, kg, window):
        if plant == "ref_hidden" and kg[0] == "R" and qg[0] != "R":
            return False
        if plant == "source_one_way" and qg[0] == "S" and kg[0] in ("N", "C"):
            return False
        return _ORIG_SEES(qg, kg, window)

    def history_all(t, window):  # the window forgotten: every past chunk kept
        return list(range(t))

    monkeypatch.setattr(tg, "sees", rule)
    if plant == "evicted_kept":
        monkeypatch.setattr(tg, "history_of", history_all)
    data = _scenario(8)
    assert np.abs(_oracle_step(data) - _brute(data)).max() > 1e-6
