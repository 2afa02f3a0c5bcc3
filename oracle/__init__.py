"""Plain fp64 CPU oracle for chunk-wise causal attention over a bounded KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the ``libcca.so`` C-ABI
library and its Python binding) may import, call, link or execute anything in
this package.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference legs use it.  It shares no code, constant table or
helper with the CUDA path; the only thing both sides consume is the seeded input
generator package ``synth`` (which holds no arithmetic of the method).

What the oracle restates, and from where (page title, section):

* ``chunk_attention``  -- attention is bidirectional inside a chunk and causal
  across chunks; the active chunk sees a fixed number of the most recent history
  chunks plus the first chunk, kept forever as a global sink.
  ["JoyAI-Video-Edit 소개", section 청크 단위 자기회귀 적응 (chunk-wise
  autoregressive adaptation)]; ["論文解説: JoyAI-Video-Edit", step 1 (§4.1)].
* ``kv_ring``          -- after a chunk is generated its clean K/V are cached for
  the next chunk; the cache keeps the first chunk as sink plus a sliding window of
  recent chunks, so memory and per-chunk compute are bounded.
  ["JoyAI-Video-Edit 소개", section 30 FPS를 만드는 실시간 배포 파이프라인
  (deployment pipeline)]; ["論文解説: JoyAI-Video-Edit", §5 per-chunk loop].
* ``fp8``              -- FP8 quantisation is applied across the deployed
  pipeline (same deployment section).  Format and granularity are not given on
  the pages; the reading used is e4m3 with per-head absmax scales.
* ``mask_cache``       -- the AR-oriented mask cache: per-token L2 distance of
  the previous chunk's edited vs. source latents, thresholded by tau; active
  tokens get the full computation, inactive ones reuse the cached feature.
  ["LiveEdit 실시간 Diffusion 기반 스트리밍 비디오 편집", sections 핵심 기여,
  방법론 and 기술 상세 (the mask-cache formula)].

Every function is pinned by ``tests/test_oracle_pins.py`` against closed forms,
invariants, brute force on tiny inputs and library routines.  The pages print no
worked numeric example, so no value-level pin to the pages exists: the pins are
mathematical, as listed in each module.
"""

from . import chunk_attention, fp8, kv_ring, mask_cache  # noqa: F401
