"""Oracle: the bounded KV cache as a logical deque (sink + last W chunks).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Restated from ["JoyAI-Video-Edit 소개", section 30 FPS를 만드는 실시간 배포
파이프라인] and the per-chunk loop of ["論文解説: JoyAI-Video-Edit", §5]: once a
chunk has been generated its clean K/V state is stored for the next chunk; the
store keeps the first chunk as a permanent sink and a sliding window of the most
recent chunks, so memory stays bounded for an unbounded stream.  Eviction is of
the oldest non-sink chunk.

The deque holds *logical* chunk indices only; where the GPU ring puts a chunk
(its slot) is a layout choice of the library, which reports it through
``cca_kv_ring_query``.  Tests compare that report and the slot contents with
this deque.
"""

from __future__ import annotations

from collections import deque


class KVRing:
    """Logical content of the bounded cache after ``n_appended`` appends."""

    def __init__(self, window: int):
        if window < 0:
            raise ValueError("window must be >= 0")
        self.window = window
        self.n_appended = 0
        self.sink: tuple | None = None
        self.recent: deque = deque()

    def append(self, k, v) -> None:
        """Store chunk ``n_appended``; evict the oldest non-sink chunk if full."""
        t = self.n_appended
        if t == 0:
            self.sink = (0, k, v)
        else:
            self.recent.append((t, k, v))
            while len(self.recent) > self.window:
                self.recent.popleft()
        self.n_appended += 1

    def chunks(self) -> list[int]:
        """Cached chunk indices in logical order: sink first, then oldest->newest."""
        out = [] if self.sink is None else [0]
        out.extend(c for c, _, _ in self.recent)
        return out

    def get(self, c: int):
        """(k, v) of cached chunk ``c``; KeyError if it is not (or no longer) cached."""
        if self.sink is not None and c == 0:
            return self.sink[1], self.sink[2]
        for cc, k, v in self.recent:
            if cc == c:
                return k, v
        raise KeyError(c)
