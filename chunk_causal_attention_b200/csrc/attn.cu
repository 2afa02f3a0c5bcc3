// Chunk-wise causal attention over the bounded KV cache, BF16 and FP8 e4m3, sm_100a.
//
// What it computes ["JoyAI-Video-Edit 소개", section 청크 단위 자기회귀 적응;
// "論文解説: JoyAI-Video-Edit", step 1 (§4.1)]: the queries of the current chunk
// t attend, with one dense softmax, to every key of the visible chunks -- the
// sink (chunk 0), the W most recent earlier chunks (from the ring) and chunk t
// itself (bidirectional inside the chunk).  Because visibility is per whole
// chunk, no element mask is needed: the kernel walks a list of KV chunks and
// only masks the zero-filled tail of a chunk whose length is not a multiple of
// the 128-row tile.
//
// Kernel design (sm_100a; the pages give no kernel):
//  * one work item = two 128-row Q tiles (256 queries) of one head x a range
//    of 128-row KV tiles; both Q tiles share every K/V tile loaded into shared
//    memory, halving L2->SM traffic per FLOP;
//  * warp 0 = TMA producer of Q (once per item) and K (3-stage ring); warp 2 =
//    TMA producer of V (2 stages; for e4m3 the fp16-widened values); warp 3 idle;
//    warp 1 = TMEM allocator and the single thread issuing tcgen05.mma;
//    warps 4-7 / 8-11 = softmax warpgroups, one per Q tile, one row per thread;
//  * TMEM (512 columns): S0 | S1 | O0 | O1.  S = Q K^T lands in TMEM; the
//    softmax warps read it, write P (bf16) back over the first half of S, and
//    P is the A operand of O += P V straight from TMEM;
//  * online softmax in base 2 with the scale folded in; the running maximum is
//    only moved (and O rescaled in TMEM) when a row's maximum grows by more
//    than 2^8, so P never exceeds 256 and rescales are rare;
//  * persistent schedule computed on the device from the query count: each CTA
//    first takes whole (query pair, head) items; the remaining items are split
//    evenly over all CTAs along the KV list, their partial (O, m, l) go to the
//    caller's workspace and a small combine kernel merges only those;
//  * every mbarrier wait is bounded; on timeout the CTA sets an abort flag,
//    drains its in-flight TMA loads and MMAs, frees TMEM and reports
//    CCA_DEV_TIMEOUT through the ring's status word.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <initializer_list>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "ring.cuh"
#include "sm100.cuh"

namespace cca {

constexpr int kBM = 128;       // query rows per Q tile (TMEM lanes)
constexpr int kBN = 128;       // key rows per KV tile
constexpr int kNQ = 2;         // Q tiles per work item
// K pipeline stages: 3 for bf16 (what its shared memory holds next to two Q
// tiles and two V stages); the e4m3 K tiles are half the size, so 5.
#ifndef CCA_NSK_FP8
#define CCA_NSK_FP8 5
#endif
constexpr int kNSK = 3;
constexpr int kNSV = 2;        // V pipeline stages
constexpr int kThreads = 384;  // 12 warps
constexpr float kRescaleThreshold = 8.0f;  // log2 units: p <= 2^8 between rescales
// Pairs of score columns whose exponential runs on the FMA pipe (polynomial)
// instead of the MUFU unit: bit k set = pair k of every 8 pairs (2 of 8 here).
#ifndef CCA_EMU_MASK
#define CCA_EMU_MASK 0xC0
#endif
constexpr unsigned kEmuMask = CCA_EMU_MASK;
// Exponentials: 0 = fp32 MUFU ex2 (+ FMA-pipe polynomial on kEmuMask pairs);
// 1 = packed fp16 MUFU ex2 (two results per instruction).
#ifndef CCA_EXP_MODE
#define CCA_EXP_MODE 0
#endif
constexpr int kExpMode = CCA_EXP_MODE;
#ifndef CCA_SETMAXNREG
#define CCA_SETMAXNREG 1
#endif
// Registers: the producer / MMA warpgroup needs few, the softmax warpgroups many
// (4 x 32 x 88 + 8 x 32 x 208 = 384 x 168 = the launch budget of the block).
constexpr bool kUseSetMaxNReg = CCA_SETMAXNREG;  // log2 units: p <= 2^8 between rescales

// Debug-only event trace of CTA 0 (build with -DCCA_TRACE): 64-bit records
// [event:8 | tile:16 | clock64:40], read back with cca_debug_trace_read().
#ifdef CCA_TRACE
// 4 regions of 16K records (producer, MMA, softmax warpgroup 0, 1); each
// recording thread keeps its own counter, so a record is one plain store.
__device__ unsigned long long g_trace[4 << 14];
#define CCA_TRACE_EV(ev, g)                                                                              \
  do {                                                                                                   \
    if (blockIdx.x == 0 && trace_n < (1 << 14))                                                          \
      g_trace[(trace_role << 14) + trace_n++] = (static_cast<unsigned long long>(ev) << 56) |             \
                                                (static_cast<unsigned long long>((g) & 0xFFFF) << 40) |   \
                                                (static_cast<unsigned long long>(clock64()) & 0xFFFFFFFFFFull); \
  } while (0)
#define CCA_TRACE_ROLE(r) \
  int trace_n = 0;        \
  const int trace_role = (r)
#else
#define CCA_TRACE_EV(ev, g) \
  do {                      \
  } while (0)
#define CCA_TRACE_ROLE(r) \
  do {                    \
  } while (0)
#endif

// KV sources of one launch: 0 = the ring (or the packed clean history), 1 = the
// current block (or the packed current chunks), 2 = a globally visible group
// (the reference tokens R).  Each is a [slots][rows][H][D] tensor.
constexpr int kMaxSrc = 3;
constexpr int kMaxProb = 32;   // query blocks ("problems") per launch
constexpr int kMaxSegs = 192;  // visible KV segments over all problems of a launch

// One block of queries with its own list of visible KV segments.  A segment is
// one slot of one source, all of its rows.  Items of a problem are (query
// pair, head); all have the same KV tile count n_kv.  The host lists problems
// by non-increasing n_kv.
struct AttnProb {
  int32_t n_q;        // queries of this problem (problem 0: overridden by *n_q_dev)
  int16_t q_slot;     // slot of the Q tensor holding them (rows 0 .. n_q-1)
  int16_t out_slot;   // slot of the output tensor
  int16_t seg0, n_seg;
  int32_t n_kv;       // KV tiles per item = sum over its segments
};

struct AttnArgs {
  const void *q;           // query rows (gather path): [rows][H][D] of the ring's element type
  const int32_t *q_idx;    // NULL: dense rows
  const int32_t *n_q_dev;  // NULL: problem 0 has prob[0].n_q queries
  __nv_bfloat16 *out;      // [slots][out_rows][H][D], or [out_rows][H][D] rows q_idx[i] with scatter_out
  int scatter_out;         // 1: query i's row goes to out row q_idx[i] (fused scatter-back)
  float *ws_o;             // [2 x grid][256][D] partial O of split items (unnormalised)
  float *ws_ml;            // [2 x grid][256][2] (running max in log2 units, row sum)
  int32_t *dev_status;
  // e4m3 only: per-head dequantisation scales, [slots][H] per tensor.
  const float *q_scale;
  const float *k_scale[kMaxSrc], *v_scale[kMaxSrc];
  int out_rows;            // rows per output slot (scatter: rows of the cache)
  int q_rows;              // rows of the gathered Q tensor (gather path)
  int H;
  float scale_log2;
  long long wait_budget;
  int src_len[kMaxSrc];    // rows per slot of each source
  int n_prob;
  AttnProb prob[kMaxProb];
  uint16_t seg[kMaxSegs];     // (source << 12) | slot
  uint16_t seg_t0[kMaxSegs];  // first KV tile of the segment in its problem's list
};

// Shared-memory plan.  Q/K/V tiles arrive by TMA as 128-row x 128-byte boxes
// with the 128-byte swizzle (two boxes per tile for 16-bit D=128).  V is
// always 16-bit: bf16, or for e4m3 the e4m3 values widened to fp16 (the PV
// product keeps P in 16 bits, so its B operand is 16-bit too).
template <int D, bool kFp8>
struct AttnSmem {
  static constexpr uint32_t kEsz = kFp8 ? 1 : 2;             // bytes per Q/K element
  static constexpr uint32_t kBox = 128 * 128;                // 128 rows x 128 bytes
  static constexpr uint32_t kNBox = D * kEsz / 128;          // boxes per 128-row Q/K tile
  static constexpr uint32_t kTile = kBox * kNBox;            // bytes of one loaded Q/K tile
  static constexpr uint32_t kNBoxV = D * 2 / 128;            // boxes per 128-row V tile
  static constexpr uint32_t kVTile = kBox * kNBoxV;          // bytes of one loaded V tile
  static constexpr int kNSK = kFp8 ? CCA_NSK_FP8 : ::cca::kNSK;  // K pipeline stages
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kNQ * kTile;
  static constexpr uint32_t kV = kK + kNSK * kTile;
  static constexpr uint32_t kBar = kV + kNSV * kVTile;
  static constexpr uint32_t kNumBars = 4 + 2 * kNSK + 2 * kNSV + 8 + 1 + 2 + 1;
  static constexpr uint32_t kXchg = kBar + kNumBars * 8 + 16;  // [2][128] fp32: (m, l) of warpgroup 1's rows
  static constexpr uint32_t kBytes = kXchg + 2 * 128 * 4;
  static constexpr uint32_t kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

// ---- work schedule (identical in every role, the combine kernel included)
// Items are (problem, query pair, head), problem-major and head-major inside a
// problem (so CTAs running together share a head's K/V in L2), for the query
// pairs holding each problem's queries.  With G CTAs, CTA c first takes whole
// items in rounds, item k*G + c in even rounds and k*G + G-1-c in odd ones
// (so that rounds of unequal items even out).  When the items left after the
// full rounds would unbalance the CTAs (one of them more than 1/8 of the
// average load), they are split along their KV tiles instead, in one of two
// ways.  Aligned: with r leftover items and s = G / r >= 2, item i is cut into
// s near-equal pieces taken by CTAs i*s .. i*s+s-1, one piece per CTA (each
// piece pays one Q load, one pipeline fill and one partial write).  Ranges,
// when aligned pieces would be much longer than an even share: the leftover
// items' KV tiles are concatenated into one list cut into G near-equal ranges
// [c*tr/G, (c+1)*tr/G), so a CTA may take two pieces.  A piece that covers
// only part of its item is "partial": its (O, m, l) go to workspace slot 2c
// (aligned pieces, and the piece holding a range's first tile) or 2c+1 (the
// one holding its last tile), and the combine kernel merges them.
struct Sched {
  int n_items, qr;  // items; whole rounds
  int rem0;         // first item of the split remainder (n_items if none)
  int s;            // aligned mode: pieces per leftover item (0: ranges)
  int64_t tr;       // KV tiles in the remainder list (0: no split)
};
struct Seg {
  int prob, pair, head, j0, j1, slot;  // slot < 0: whole item, direct output
};

__device__ __forceinline__ int prob_nq(const AttnArgs &a, int p, int n_q0) { return p == 0 ? n_q0 : a.prob[p].n_q; }
__device__ __forceinline__ int prob_pairs(const AttnArgs &a, int p, int n_q0) {
  return (prob_nq(a, p, n_q0) + kNQ * kBM - 1) / (kNQ * kBM);
}

__device__ __forceinline__ Sched make_sched(const AttnArgs &a, int n_q0, int G) {
  Sched s;
  int n = 0;
  int64_t total = 0;
  for (int p = 0; p < a.n_prob; ++p) {
    const int cnt = prob_pairs(a, p, n_q0) * a.H;
    n += cnt;
    total += static_cast<int64_t>(cnt) * a.prob[p].n_kv;
  }
  s.n_items = n;
  const int q = n / G, r = n % G;
  s.qr = q;
  s.rem0 = q * G;
  s.s = 0;
  s.tr = 0;
  if (r > 0) {
    // longest remainder item (problems are listed by non-increasing n_kv)
    int i0 = 0, nkv_first = 0;
    int64_t tr = 0;
    for (int p = 0; p < a.n_prob; ++p) {
      const int cnt = prob_pairs(a, p, n_q0) * a.H, i1 = i0 + cnt;
      const int b0 = i0 > s.rem0 ? i0 : s.rem0;
      if (b0 < i1) {
        if (tr == 0) nkv_first = a.prob[p].n_kv;
        tr += static_cast<int64_t>(i1 - b0) * a.prob[p].n_kv;
      }
      i0 = i1;
    }
    if (static_cast<int64_t>(nkv_first) * 8 * G > total) {
      s.tr = tr;
      const int pieces = G / r;  // aligned pieces per leftover item
      const int64_t even = (tr + G - 1) / G;
      if (pieces >= 2 && (nkv_first + pieces - 1) / pieces <= even + 2) s.s = pieces;
    } else {  // the leftover items are short next to a CTA's load: one more round of whole items
      s.qr = q + 1;
      s.rem0 = n;
    }
  }
  return s;
}

// Item u -> (problem, pair, head).  When a problem's last pair has at most 128
// queries (its second Q tile is empty, e.g. 84 of 256 rows at 1620 queries),
// those single-tile items are listed after the problem's full pairs, so the
// schedule puts the cheap items into its last round or its split remainder.
__device__ __forceinline__ void item_coords(const AttnArgs &a, int n_q0, int u, int &p, int &pair, int &head) {
  for (p = 0; p + 1 < a.n_prob; ++p) {
    const int cnt = prob_pairs(a, p, n_q0) * a.H;
    if (u < cnt) break;
    u -= cnt;
  }
  const int np = max(prob_pairs(a, p, n_q0), 1);
  const int last_rows = prob_nq(a, p, n_q0) - (np - 1) * (kNQ * kBM);
  if (np > 1 && last_rows <= kBM) {
    const int full = (np - 1) * a.H;
    if (u < full) {
      pair = u % (np - 1);
      head = u / (np - 1);
    } else {
      pair = np - 1;
      head = u - full;
    }
    return;
  }
  pair = u % np;
  head = u / np;
}

// Whether the item's second Q tile holds any query (else its MMAs and its
// softmax warpgroup skip the item).
__device__ __forceinline__ bool second_tile(const AttnArgs &a, int n_q0, const Seg &g) {
  return g.pair * (kNQ * kBM) + kBM < prob_nq(a, g.prob, n_q0);
}

// Remainder item holding tile offset t of the remainder list: its index, first
// tile offset and tile count.
__device__ __forceinline__ void rem_locate(const AttnArgs &a, int n_q0, const Sched &s, int64_t t, int &u,
                                           int64_t &ustart, int &ulen) {
  int i0 = 0;
  int64_t acc = 0;
  for (int p = 0; p < a.n_prob; ++p) {
    const int cnt = prob_pairs(a, p, n_q0) * a.H, i1 = i0 + cnt;
    const int b0 = i0 > s.rem0 ? i0 : s.rem0;
    const int nkv = a.prob[p].n_kv;
    if (b0 < i1) {
      const int64_t span = static_cast<int64_t>(i1 - b0) * nkv;
      if (t < acc + span || p == a.n_prob - 1) {
        const int k = static_cast<int>((t - acc) / nkv);
        u = b0 + k;
        ustart = acc + static_cast<int64_t>(k) * nkv;
        ulen = nkv;
        return;
      }
      acc += span;
    }
    i0 = i1;
  }
  u = s.n_items;
  ustart = acc;
  ulen = 1;
}

// The k-th segment of work of CTA c (false when there is none).
__device__ __forceinline__ bool get_seg(const AttnArgs &a, int n_q0, const Sched &s, int G, int c, int k, Seg &g) {
  if (k < s.qr) {
    const int u = k * G + ((k & 1) ? G - 1 - c : c);
    if (u >= s.rem0) return false;  // only in the last round of an unsplit schedule
    int p, pair, head;
    item_coords(a, n_q0, u, p, pair, head);
    g = {p, pair, head, 0, a.prob[p].n_kv, -1};
    return true;
  }
  if (s.tr == 0) return false;
  k -= s.qr;
  if (s.s > 0) {  // aligned: one piece of item rem0 + c / s
    const int u = s.rem0 + c / s.s, j = c % s.s;
    if (k > 0 || u >= s.n_items) return false;
    int p, pair, head;
    item_coords(a, n_q0, u, p, pair, head);
    const int n = a.prob[p].n_kv;
    const int j0 = j * n / s.s, j1 = (j + 1) * n / s.s;
    if (j0 >= j1) return false;
    g = {p, pair, head, j0, j1, 2 * c};
    return true;
  }
  const int64_t lo = static_cast<int64_t>(c) * s.tr / G, hi = static_cast<int64_t>(c + 1) * s.tr / G;
  int64_t t = lo;
  for (int piece = 0; t < hi; ++piece) {
    int u, ulen;
    int64_t ustart;
    rem_locate(a, n_q0, s, t, u, ustart, ulen);
    const int64_t e = hi < ustart + ulen ? hi : ustart + ulen;
    if (piece == k) {
      int p, pair, head;
      item_coords(a, n_q0, u, p, pair, head);
      const bool whole = t == ustart && e == ustart + ulen;
      g = {p, pair, head, static_cast<int>(t - ustart), static_cast<int>(e - ustart),
           whole ? -1 : (t == lo ? 2 * c : 2 * c + 1)};
      return true;
    }
    t = e;
  }
  return false;
}

// Walks the KV tiles of one item in order: tile j -> segment k (its source
// and slot are a.seg[k]), first row and valid rows.  Segments are visited in
// order, so a step costs O(1); the cursor holds three registers.
struct TileCursor {
  int k;     // current segment
  int t1;    // first tile after it
  int vend;  // 128 * (its first tile) + its rows: valid rows of tile j = vend - 128 j
};
__device__ __forceinline__ void cursor_begin(const AttnArgs &a, int p, TileCursor &cu) {
  cu.k = a.prob[p].seg0 - 1;
  cu.t1 = 0;
  cu.vend = 0;
}
__device__ __forceinline__ void cursor_at(const AttnArgs &a, int p, TileCursor &cu, int j, int &row0, int &valid) {
  while (j >= cu.t1) {
    ++cu.k;
    const int t0 = a.seg_t0[cu.k];
    cu.vend = t0 * kBN + a.src_len[a.seg[cu.k] >> 12];
    const AttnProb &P = a.prob[p];
    cu.t1 = cu.k + 1 < P.seg0 + P.n_seg ? static_cast<int>(a.seg_t0[cu.k + 1]) : P.n_kv;
  }
  const int v = cu.vend - j * kBN;
  valid = v < kBN ? v : kBN;
  row0 = a.src_len[a.seg[cu.k] >> 12] - v;
}
__device__ __forceinline__ int cursor_src(const AttnArgs &a, const TileCursor &cu) { return a.seg[cu.k] >> 12; }
__device__ __forceinline__ int cursor_slot(const AttnArgs &a, const TileCursor &cu) { return a.seg[cu.k] & 0xFFF; }

// Dequantisation scale of a K or V segment for one head.
__device__ __forceinline__ float seg_scale(const float *const *tab, int src, int slot, int H, int head) {
  return __ldg(tab[src] + slot * H + head);
}

// kSplit: items with one Q tile and two KV tiles or more are split between the
// softmax warpgroups along their KV tiles.  Built only for calls whose queries
// are contiguous rows: a call with gathered queries fills its Q tiles (a few
// hundred rows over the chunk's KV tiles), and the split branch's code in the
// MMA warp alone costs it time.
template <int D, bool kFp8, bool kSplit>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k0,
                const __grid_constant__ CUtensorMap tm_v0, const __grid_constant__ CUtensorMap tm_k1,
                const __grid_constant__ CUtensorMap tm_v1, const __grid_constant__ CUtensorMap tm_k2,
                const __grid_constant__ CUtensorMap tm_v2, const __grid_constant__ AttnArgs a) {
  using namespace sm100;
  using S = AttnSmem<D, kFp8>;
  constexpr int kNSK = S::kNSK;
  static_assert(!kFp8 || D == 128, "e4m3 path is built for head_dim 128");
  constexpr int kBoxElems = 128 / S::kEsz;  // elements of D per TMA box
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *gbase = smem_raw + (base - raw);
  uint64_t *bars = reinterpret_cast<uint64_t *>(gbase + S::kBar);
  uint64_t *q_full = bars;              // [kNQ]  producer -> MMA
  uint64_t *q_empty = bars + 2;         // [kNQ]  MMA -> producer
  uint64_t *k_full = bars + 4;           // [kNSK]
  uint64_t *k_empty = k_full + kNSK;     // [kNSK]
  uint64_t *v_full = k_empty + kNSK;     // [kNSV] V tile landed
  uint64_t *v_empty = v_full + kNSV;     // [kNSV] V tile consumed (MMA, or the e4m3 expander)
  uint64_t *s_full = v_empty + kNSV;     // [2] MMA -> softmax: S ready
  uint64_t *p_full = s_full + 2;        // [2] softmax -> MMA: P ready (and O rescaled)
  uint64_t *o_full = p_full + 2;        // [2] MMA -> softmax: O final for the item
  uint64_t *o_empty = o_full + 2;       // [2] softmax -> MMA: O read out
  uint64_t *p_half = o_empty + 2;       // [2] softmax -> MMA: first half of P ready (and O rescaled)
  uint64_t *drain = p_half + 2;         // [1] teardown: all MMAs complete
  uint64_t *split_done = drain + 1;     // [1] softmax 1 -> softmax 0: (m, l) of a split item's rows written
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(split_done + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // The combine grid (a programmatic dependent) may be scheduled from now on; it
  // waits for this grid's completion before it reads anything.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int n_q0 = a.n_q_dev ? min(max(*a.n_q_dev, 0), a.prob[0].n_q) : a.prob[0].n_q;
  const Sched sch = make_sched(a, n_q0, gridDim.x);
  auto kmap = [&](int src) { return src == 0 ? &tm_k0 : src == 1 ? &tm_k1 : &tm_k2; };
  auto vmap = [&](int src) { return src == 0 ? &tm_v0 : src == 1 ? &tm_v1 : &tm_v2; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kBM / 32);  // one arrive per softmax warp
      mbar_init(&p_half[i], kBM / 32);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], kBM / 32);
    }
    for (int s = 0; s < kNSK; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kNSV; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);  // released by the MMA
    }
    mbar_init(drain, 1);
    mbar_init(split_done, kBM / 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    if (!a.q_idx) prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k0);
    prefetch_tmap(&tm_v0);
    prefetch_tmap(&tm_k1);
    prefetch_tmap(&tm_v1);
    if (a.src_len[2] > 0) {
      prefetch_tmap(&tm_k2);
      prefetch_tmap(&tm_v2);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long budget = a.wait_budget;

  // ================================================================ producer
  if (warp == 0) {
    if (kUseSetMaxNReg) regs_dec<88>();
    CCA_TRACE_ROLE(0);
    uint32_t g = 0;   // KV tiles handled by this CTA
    uint32_t gk = 0;  // K tile loads armed
    int it = 0;       // items handled by this CTA
    int q_armed = 0;  // Q phases armed (per tile, identical for both)
    bool ok = true;
    for (int kseg = 0; ok; ++kseg) {
      Seg sg;
      if (!get_seg(a, n_q0, sch, gridDim.x, blockIdx.x, kseg, sg)) break;
      const int pair = sg.pair, head = sg.head, j0 = sg.j0, j1 = sg.j1;
      const int q_slot = a.prob[sg.prob].q_slot;
      const int n_q = prob_nq(a, sg.prob, n_q0);
      if (lane == 0) CCA_TRACE_EV(28, it);
      for (int i = 0; i < kNQ && ok; ++i) {
        if (it > 0) ok = __all_sync(0xffffffffu, mbar_wait(&q_empty[i], (it - 1) & 1, abort_flag, budget));
        if (!ok) break;
        const uint32_t dstq = base + S::kQ + i * S::kTile;
        const int row0 = pair * (kNQ * kBM) + i * kBM;
        if (!a.q_idx) {
          if (lane == 0) {
            mbar_arrive_expect_tx(&q_full[i], S::kTile);
            for (uint32_t b = 0; b < S::kNBox; ++b)
              tma_load_4d(&tm_q, &q_full[i], dstq + b * S::kBox, b * kBoxElems, head, row0, q_slot);
          }
        } else {
          // Gather: row r of the tile is query q_idx[row0 + r], fetched by TMA
          // row-gather loads (four rows per instruction, one per 128-byte column
          // box; the map views Q as [q_rows][H*D]) into the layout a tile load
          // produces.  Lane l takes rows 4l .. 4l+3.  Rows past n_q, and indices
          // outside [0, q_rows) (flagged), point one row past the tensor, where
          // the TMA reads zeros.
          int sr[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int qr = row0 + 4 * lane + k;
            int v = qr < n_q ? __ldg(a.q_idx + qr) : a.q_rows;
            if (qr < n_q && (v < 0 || v >= a.q_rows)) {
              if (a.dev_status) *a.dev_status = CCA_DEV_BAD_INDEX;  // out-of-range index: row read as zeros
              v = a.q_rows;
            }
            sr[k] = v;
          }
          if (lane == 0) mbar_arrive_expect_tx(&q_full[i], S::kTile);
          __syncwarp();
          for (uint32_t b = 0; b < S::kNBox; ++b)
            tma_gather4(&tm_q, &q_full[i], dstq + b * S::kBox + lane * 4 * 128, head * D + b * kBoxElems, sr[0], sr[1],
                        sr[2], sr[3]);
        }
      }
      if (!ok) break;
      if (lane == 0) CCA_TRACE_EV(29, it);
      q_armed = it + 1;
      TileCursor cu;
      cursor_begin(a, sg.prob, cu);
      for (int j = j0; j < j1; ++j, ++g) {
        const uint32_t stage = g % kNSK, ph = (g / kNSK) & 1;
        int row0, valid;
        cursor_at(a, sg.prob, cu, j, row0, valid);
        const int src = cursor_src(a, cu), slot = cursor_slot(a, cu);
        if (g >= kNSK) ok = __all_sync(0xffffffffu, mbar_wait(&k_empty[stage], ph ^ 1, abort_flag, budget));
        if (!ok) break;
        ++gk;
        if (lane == 0) {
          const uint32_t dst = base + S::kK + stage * S::kTile;
          CCA_TRACE_EV(30, g);
          mbar_arrive_expect_tx(&k_full[stage], S::kTile);
          for (uint32_t b = 0; b < S::kNBox; ++b)
            tma_load_4d(kmap(src), &k_full[stage], dst + b * S::kBox, b * kBoxElems, head, row0, slot);
        }
      }
      ++it;
    }
    // Drain: wait (bounded) for the most recent armed phase of every barrier the
    // TMA may still complete, so no copy lands in shared memory after exit.
    if (lane == 0) {
      for (uint32_t k = 0; k < kNSK && k < gk; ++k) {
        const uint32_t gg = gk - 1 - k;
        mbar_drain(&k_full[gg % kNSK], (gg / kNSK) & 1, budget);
      }
      if (q_armed > 0)
        for (int i = 0; i < kNQ; ++i) mbar_drain(&q_full[i], (q_armed - 1) & 1, budget);
    }
  }
  // ================================================================ MMA issuer
  else if (warp == 1) {
    if (kUseSetMaxNReg) regs_dec<88>();
    CCA_TRACE_ROLE(1);
    // The whole warp runs this loop converged, so every operand below is
    // warp-uniform; one elected lane issues each batch of tcgen05 instructions.
    // QK: bf16 x bf16 (kind::f16) or e4m3 x e4m3 (kind::f8f6f4), both K-major.
    // PV: P (bf16, or fp16 for the e4m3 path) from TMEM, V MN-major in smem.
    constexpr uint32_t kIdescQK = kFp8 ? idesc_make(0, 0, 0, 0, kBM, kBN) : idesc_make(1, 1, 0, 0, kBM, kBN);
    constexpr uint32_t kIdescPV = kFp8 ? idesc_make(0, 0, 0, 1, kBM, D) : idesc_make(1, 1, 0, 1, kBM, D);
    constexpr int kQKSteps = D * S::kEsz / 32;  // 32 bytes of K per MMA
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    // Descriptors of every operand tile, built once; a K step inside a tile is
    // an add to the (address >> 4) field.
    const uint64_t dQ0 = sdesc_sw128(base + S::kQ, 16, 1024);
    const uint64_t dK0 = sdesc_sw128(base + S::kK, 16, 1024);
    const uint64_t dV0 = sdesc_sw128(base + S::kV, S::kBox, 1024);
    constexpr uint32_t kVStageBytes = S::kVTile;
    uint64_t *pv_full = v_full;
    uint64_t *pv_empty = v_empty;
    // S_i = Q tile qt x K(stage)
    auto issue_qk = [=](int i, uint32_t stage, int qt) {
      const uint64_t qa = dQ0 + ((qt * S::kTile) >> 4), kb = dK0 + ((stage * S::kTile) >> 4);
      const uint32_t d = tm + i * 128u;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kQKSteps; ++kk) {
          const uint32_t off = ((kk >> 2) * S::kBox + (kk & 3) * 32) >> 4;
          if constexpr (kFp8)
            mma_f8_ss(d, qa + off, kb + off, kIdescQK, kk > 0 ? 1u : 0u);
          else
            mma_f16_ss(d, qa + off, kb + off, kIdescQK, kk > 0 ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    // O_i += P_i V over K columns [16 k0, 16 k1) of the tile.
    auto issue_pv = [=](int i, uint32_t stage, bool acc, int k0, int k1) {
      const uint64_t vb = dV0 + ((stage * kVStageBytes) >> 4);
      const uint32_t d = tm + 256u + i * D, pa = tm + i * 128u;
      if (elect_one()) {
#pragma unroll
        for (int kk = k0; kk < k1; ++kk)
          mma_f16_ts(d, pa + kk * 8, vb + ((kk * 16 * 128) >> 4), kIdescPV, (acc || kk > 0) ? 1u : 0u);
      }
      __syncwarp();
    };
    auto commit = [](uint64_t *bar) {
      if (elect_one()) mma_commit(bar);
      __syncwarp();
    };
    auto wait = [=](uint64_t *bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, budget));
    };
    // The softmax releases P in two halves (first 64 key columns, then the
    // rest), so the first half of PV overlaps the second half of its exps.
    auto pv_in_halves = [&](int i, uint32_t stage, bool acc, uint32_t parity) {
      if (!wait(&p_half[i], parity)) return false;
      tc_fence_after();
      issue_pv(i, stage, acc, 0, kBN / 32);
      if (!wait(&p_full[i], parity)) return false;
      tc_fence_after();
      issue_pv(i, stage, acc, kBN / 32, kBN / 16);
      return true;
    };
    uint32_t g = 0;           // KV tiles handled (their K and V stages)
    uint32_t g0 = 0, g1 = 0;  // tiles of softmax warpgroup 0 / 1 (phases of their S and P barriers)
    int it = 0, it1 = 0;      // items with an O of warpgroup 0 / 1 (phases of their O barriers)
    bool ok = true;
    for (int kseg = 0; ok; ++kseg) {
      Seg sg;
      if (!get_seg(a, n_q0, sch, gridDim.x, blockIdx.x, kseg, sg)) break;
      const int j0 = sg.j0, j1 = sg.j1;
      const int n = j1 - j0;
      const bool two = second_tile(a, n_q0, sg);  // else QK1 / PV1 are skipped (softmax 1 sits the item out)
      ok = wait(&q_full[0], it & 1) && wait(&q_full[1], it & 1);
      // K of the segment's first tile; later K tiles are waited for one tile
      // ahead (after QK1), while the softmax still runs, so that PV0(g) and
      // QK0(g+1) go to the tensor core back to back.
      ok = ok && wait(&k_full[g % kNSK], (g / kNSK) & 1);
      if (!ok) break;
      tc_fence_after();
      if (kSplit && !two && n >= 2) {
        // An item whose second Q tile is empty: both warpgroups work on its one
        // Q tile, warpgroup w on the item's tiles jj = w, w + 2, ... with its
        // own S, P, O and running maximum and sum; the softmax of warpgroup 0
        // merges the two halves at the end.  Per tile: QK of this tile, then the
        // PV of the previous tile (the other warpgroup's), so a warpgroup's
        // PV(jj) and QK(jj + 2) reach the tensor core back to back.
        uint32_t pc0 = g0, pc1 = g1;  // tiles each warpgroup has had before
        bool fresh0 = true, fresh1 = true;  // no PV into this item's O_w yet
        auto pv_of = [&](int u, uint32_t gt) -> bool {  // O_u += P_u V(gt)
          const uint32_t vst = gt % kNSV, vph = (gt / kNSV) & 1;
          if (!wait(&pv_full[vst], vph)) return false;
          const int prev = u == 0 ? it : it1;
          const bool fresh = u == 0 ? fresh0 : fresh1;
          const uint32_t pc = u == 0 ? pc0 : pc1;
          if (fresh && prev > 0 && !wait(&o_empty[u], (prev - 1) & 1)) return false;
          if (!pv_in_halves(u, vst, !fresh, pc & 1)) return false;
          commit(&pv_empty[vst]);
          if (u == 0) {
            fresh0 = false;
            ++pc0;
          } else {
            fresh1 = false;
            ++pc1;
          }
          return true;
        };
        for (int jj = 0; jj < n && ok; ++jj, ++g) {
          const int w = jj & 1;
          const uint32_t stage = g % kNSK;
          tc_fence_after();
          issue_qk(w, stage, 0);
          commit(&s_full[w]);
          commit(&k_empty[stage]);
          if (jj == n - 1) {
            commit(&q_empty[0]);
            commit(&q_empty[1]);
          }
          if (jj > 0 && !(ok = pv_of(w ^ 1, g - 1))) break;
          if (jj < n - 1 && !(ok = wait(&k_full[(g + 1) % kNSK], ((g + 1) / kNSK) & 1))) break;
        }
        if (!ok || !(ok = pv_of((n - 1) & 1, g - 1))) break;
        commit(&o_full[0]);
        commit(&o_full[1]);
        g0 = pc0;
        g1 = pc1;
        ++it;
        ++it1;
        continue;
      }
      for (int jj = 0; jj < n && ok; ++jj, ++g, ++g0) {
        const uint32_t stage = g % kNSK;
        const uint32_t vst = g % kNSV, vph = (g / kNSV) & 1;
        if (lane == 0) CCA_TRACE_EV(1, g);
        tc_fence_after();
        issue_qk(0, stage, 0);
        commit(&s_full[0]);
        if (lane == 0) CCA_TRACE_EV(2, g);
        if (two && jj > 0) {  // O1 += P1 V for the previous tile
          const uint32_t pst = (g - 1) % kNSV;
          if (jj == 1 && it1 > 0 && !(ok = wait(&o_empty[1], (it1 - 1) & 1))) break;
          if (!(ok = pv_in_halves(1, pst, jj > 1, (g1 - 1) & 1))) break;
          if (lane == 0) CCA_TRACE_EV(3, g - 1);
          commit(&pv_empty[pst]);
        }
        if (two) {
          issue_qk(1, stage, 1);
          commit(&s_full[1]);
        }
        commit(&k_empty[stage]);
        if (lane == 0) CCA_TRACE_EV(4, g);
        if (jj == n - 1) {
          commit(&q_empty[0]);
          commit(&q_empty[1]);
        } else {
          if (lane == 0) CCA_TRACE_EV(7, g + 1);
          if (!(ok = wait(&k_full[(g + 1) % kNSK], ((g + 1) / kNSK) & 1))) break;
        }
        if (!(ok = wait(&pv_full[vst], vph))) break;
        if (lane == 0) CCA_TRACE_EV(8, g);
        if (jj == 0 && it > 0 && !(ok = wait(&o_empty[0], (it - 1) & 1))) break;
        if (!(ok = pv_in_halves(0, vst, jj > 0, g0 & 1))) break;
        if (!two) commit(&pv_empty[vst]);  // no PV1 will read this V stage
        if (lane == 0) CCA_TRACE_EV(5, g);
        if (lane == 0) CCA_TRACE_EV(6, g);
        if (jj == n - 1) commit(&o_full[0]);
        if (two) ++g1;
      }
      if (!ok) break;
      if (two) {  // O1 += P1 V for the last tile
        const uint32_t pst = (g - 1) % kNSV;
        if (n == 1 && it1 > 0 && !(ok = wait(&o_empty[1], (it1 - 1) & 1))) break;
        if (!(ok = pv_in_halves(1, pst, n > 1, (g1 - 1) & 1))) break;
        commit(&pv_empty[pst]);
        commit(&o_full[1]);
        ++it1;
      }
      ++it;
    }
    // Teardown: every MMA issued above must be complete before TMEM is freed.
    commit(drain);
    if (lane == 0) mbar_drain(drain, 0, budget);
    __syncwarp();
  }
  // ================================================================ V producer
  else if (warp == 2) {
    if (kUseSetMaxNReg) regs_dec<88>();
    // V tiles run on their own warp so a V slot that frees late (after the PV
    // MMAs) never holds back the next K loads.
    uint32_t g = 0, gv = 0;
    bool ok = true;
    for (int kseg = 0; ok; ++kseg) {
      Seg sg;
      if (!get_seg(a, n_q0, sch, gridDim.x, blockIdx.x, kseg, sg)) break;
      TileCursor cu;
      cursor_begin(a, sg.prob, cu);
      for (int j = sg.j0; j < sg.j1; ++j, ++g) {
        const uint32_t stage = g % kNSV, ph = (g / kNSV) & 1;
        int row0, valid;
        cursor_at(a, sg.prob, cu, j, row0, valid);
        const int src = cursor_src(a, cu), slot = cursor_slot(a, cu);
        if (g >= kNSV) ok = __all_sync(0xffffffffu, mbar_wait(&v_empty[stage], ph ^ 1, abort_flag, budget));
        if (!ok) break;
        ++gv;
        if (lane == 0) {
          const uint32_t dst = base + S::kV + stage * S::kVTile;
          mbar_arrive_expect_tx(&v_full[stage], S::kVTile);
          for (uint32_t b = 0; b < S::kNBoxV; ++b)
            tma_load_4d(vmap(src), &v_full[stage], dst + b * S::kBox, b * 64, sg.head, row0, slot);
        }
      }
    }
    if (lane == 0)
      for (uint32_t k = 0; k < kNSV && k < gv; ++k) {
        const uint32_t gg = gv - 1 - k;
        mbar_drain(&v_full[gg % kNSV], (gg / kNSV) & 1, budget);
      }
  }
  // ================================================================ idle
  else if (warp == 3) {
    if (kUseSetMaxNReg) regs_dec<88>();
  }
  // ================================================================ softmax
  else {
    if (kUseSetMaxNReg) regs_inc<208>();
    const int wg = (warp - 4) >> 2;         // Q tile of this warpgroup
    const int r = ((warp & 3) << 5) + lane;  // row inside the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + wg * 128u;
    const uint32_t tO = tmem + lane_off + 256u + wg * D;
    CCA_TRACE_ROLE(2 + wg);
    uint32_t g = 0;  // tiles this warpgroup has had (phases of its S and P barriers)
    int it = 0;      // items this warpgroup has had (phases of its O barriers)
    int it1 = 0;     // warpgroup 0: items in which warpgroup 1 had an O (phases of o_full[1])
    int ns = 0;      // warpgroup 0: split items (phases of split_done)
    bool ok = true;
    for (int kseg = 0; ok; ++kseg) {
      Seg sg;
      if (!get_seg(a, n_q0, sch, gridDim.x, blockIdx.x, kseg, sg)) break;
      // An item whose second Q tile is empty is split between the warpgroups
      // along its KV tiles (warpgroup w: tiles j0 + w, j0 + w + 2, ...) when it
      // has two tiles or more; warpgroup 0 merges the halves at the end.
      const bool two = second_tile(a, n_q0, sg);
      const bool split = kSplit && !two && sg.j1 - sg.j0 >= 2;
      if (wg == 1 && !two && !split) continue;
      const int pair = sg.pair, head = sg.head, j0 = sg.j0, j1 = sg.j1;
      const int jfirst = j0 + (split ? wg : 0), jstep = split ? 2 : 1;
      const AttnProb &P = a.prob[sg.prob];
      const int n_q = prob_nq(a, sg.prob, n_q0);
      // e4m3: scores carry the factor s_q * s_k(chunk); V's factor s_v(chunk) is
      // folded into P relative to the largest s_v of the visible chunks, which
      // the epilogue multiplies back.
      float s_q = 1.f, s_vmax = 1.f;
      if constexpr (kFp8) {
        s_q = __ldg(a.q_scale + P.q_slot * a.H + head);
        s_vmax = 0.f;
        for (int k = P.seg0; k < P.seg0 + P.n_seg; ++k)
          s_vmax = fmaxf(s_vmax, seg_scale(a.v_scale, a.seg[k] >> 12, a.seg[k] & 0xFFF, a.H, head));
        if (!(s_vmax > 0.f)) s_vmax = 1.f;
      }
      float m_ref = -INFINITY, l_sum = 0.f;
      TileCursor cu;
      cursor_begin(a, sg.prob, cu);
      // e4m3: a tile's scale factors are loaded and derived one tile ahead (on a
      // second cursor), off the path from S ready to P released.
      TileCursor cn = cu;
      float sl2_n = a.scale_log2, pf_n = 1.f, lpf_n = 0.f, ipf_n = 1.f;
      auto fp8_factors = [&](int jn) {
        int r0, vv;
        cursor_at(a, sg.prob, cn, jn, r0, vv);
        const int src = cursor_src(a, cn), slot = cursor_slot(a, cn);
        sl2_n = a.scale_log2 * (s_q * seg_scale(a.k_scale, src, slot, a.H, head));
        // Floored at 2^-100 so that a zero V scale (all values of that chunk
        // zero) still gives finite exponentials whose sum is the sum of P: their
        // 16-bit PV operand rounds to zero, which is the chunk's exact share.
        pf_n = fmaxf(seg_scale(a.v_scale, src, slot, a.H, head) / s_vmax, 0x1p-100f);
        lpf_n = __log2f(pf_n);
        ipf_n = 1.f / pf_n;
      };
      if constexpr (kFp8)
        if (jfirst < j1) fp8_factors(jfirst);
      for (int j = jfirst; j < j1; j += jstep, ++g) {
        int row0, valid;
        cursor_at(a, sg.prob, cu, j, row0, valid);
        (void)row0;
        float sl2 = a.scale_log2, lpf = 0.f, ipf = 1.f;
        if constexpr (kFp8) {
          sl2 = sl2_n;
          lpf = lpf_n;
          ipf = ipf_n;
          if (j + jstep < j1) fp8_factors(j + jstep);
        }
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[wg], g & 1, abort_flag, budget));
        if (!ok) break;
        if (lane == 0 && (warp & 3) == 0) CCA_TRACE_EV(10 + 10 * wg, g);
        tc_fence_after();
        // Scores in two 64-column halves: the second half's TMEM load is in flight
        // while the first half is masked and reduced.  Row maximum: 8 independent
        // 3-input max chains, then a short tree.
        float x[128];
        float mx;
        {
          float acc[8];
          uint32_t u0[32], u1[32];
          tmem_ld32(tS + 0, u0);
          tmem_ld32(tS + 32, u1);
          tmem_ld_wait32(u0);
          tmem_ld_wait32(u1);
          uint32_t u2[32], u3[32];
          tmem_ld32(tS + 64, u2);
          tmem_ld32(tS + 96, u3);
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            x[c] = __uint_as_float(u0[c]);
            x[32 + c] = __uint_as_float(u1[c]);
          }
          if (valid < 64) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (c >= valid) x[c] = -INFINITY;
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[k] = x[k];
#pragma unroll
          for (int c = 8; c < 64; c += 16) {
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] = fmax3(acc[k], x[c + k], x[c + 8 + k > 63 ? 63 : c + 8 + k]);
          }
          tmem_ld_wait32(u2);
          tmem_ld_wait32(u3);
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            x[64 + c] = __uint_as_float(u2[c]);
            x[96 + c] = __uint_as_float(u3[c]);
          }
          if (valid < kBN) {
#pragma unroll
            for (int c = 64; c < 128; ++c)
              if (c >= valid) x[c] = -INFINITY;
          }
#pragma unroll
          for (int c = 64; c < 128; c += 16) {
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] = fmax3(acc[k], x[c + k], x[c + 8 + k]);
          }
          mx = fmax3(fmax3(acc[0], acc[1], acc[2]), fmax3(acc[3], acc[4], acc[5]), fmaxf(acc[6], acc[7]));
        }
        if (lane == 0 && (warp & 3) == 0) CCA_TRACE_EV(11 + 10 * wg, g);
        const float m_tile = mx * sl2;
        const bool need = m_tile > m_ref + kRescaleThreshold;
        const float m_new = need ? m_tile : m_ref;
        const float alpha = need ? ex2_approx(m_ref - m_new) : 1.f;
        // p = 2^(x * scale_log2 - m_new), packed f32x2 FMAs, 4 packed partial sums,
        // 16-bit pairs stored to TMEM over the first 64 columns of S, 16 at a time.
        // e4m3: the V-scale ratio pf enters as log2(pf) in the exponent, so the
        // exponential is already P * pf (the 16-bit PV operand); its sum is
        // multiplied by 1 / pf.
        const float m_off = kFp8 ? m_new - lpf : m_new;
        const uint64_t sl2_2 = f2_pack(sl2, sl2), negm_2 = f2_pack(-m_off, -m_off);
        // Rescale this row of O when the reference maximum moved (O of the
        // previous tile is complete: S of this tile was committed after it);
        // done before the first half of P is released to the PV MMAs.
        if (j > jfirst && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tO + c0, o);
            tmem_ld_wait32(o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tO + c0, o);
          }
        }
        uint64_t sums[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          // The first 64 key columns of P (and the O rescale) are in TMEM after
          // two groups: released to the PV MMAs before the third group's
          // exponentials (e4m3) or after them, ahead of its store, so that the
          // store wait finds the first two groups' stores done (bf16).
          if (kFp8 && q4 == 2) {
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_half[wg]);
          }
          uint32_t p16[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int i = q4 * 32 + 2 * c;
            float e0, e1;
            f2_unpack(f2_fma(f2_pack(x[i], x[i + 1]), sl2_2, negm_2), e0, e1);
            if constexpr (kExpMode == 1) {
              const uint32_t h = ex2_f16x2(e0, e1);  // MUFU, two per instruction
              f16x2_to_f32(h, e0, e1);
              sums[c & 3] = f2_add(sums[c & 3], f2_pack(e0, e1));
              if constexpr (kFp8)
                p16[c] = h;
              else
                p16[c] = pack_bf16x2(e0, e1);
            } else {
              if ((kEmuMask >> (c & 7)) & 1) {
                exp2_poly_pair(e0, e1);  // FMA pipe
              } else {
                e0 = ex2_approx(e0);  // MUFU
                e1 = ex2_approx(e1);
              }
              sums[c & 3] = f2_add(sums[c & 3], f2_pack(e0, e1));
              if constexpr (kFp8)
                p16[c] = pack_f16x2(e0, e1);
              else
                p16[c] = pack_bf16x2(e0, e1);
            }
          }
          if (!kFp8 && q4 == 2) {
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_half[wg]);
          }
          tmem_st16(tS + q4 * 16, p16);
        }
        float s_lo, s_hi;
        f2_unpack(f2_add(f2_add(sums[0], sums[1]), f2_add(sums[2], sums[3])), s_lo, s_hi);
        const float tile_sum = kFp8 ? (s_lo + s_hi) * ipf : (s_lo + s_hi);
        l_sum = l_sum * alpha + tile_sum;
        m_ref = m_new;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[wg]);
        if (lane == 0 && (warp & 3) == 0) CCA_TRACE_EV(12 + 10 * wg, g);
      }
      if (!ok) break;
      float *xm1 = reinterpret_cast<float *>(gbase + S::kXchg), *xl1 = xm1 + 128;
      if (split && wg == 1) {
        // hand this half's (m, l) to warpgroup 0, which reads O1 from TMEM and
        // frees it (o_empty[1]) before this warpgroup takes another item
        xm1[r] = m_ref;
        xl1[r] = l_sum;
        __syncwarp();
        if (lane == 0) mbar_arrive(split_done);
        ok = __all_sync(0xffffffffu, mbar_wait(&o_empty[1], it & 1, abort_flag, budget));
        if (!ok) break;
        ++it;
        continue;
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&o_full[wg], it & 1, abort_flag, budget));
      // split: both halves' PVs done and warpgroup 1's (m, l) written
      if (split && ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_full[1], it1 & 1, abort_flag, budget));
      if (split && ok) ok = __all_sync(0xffffffffu, mbar_wait(split_done, ns & 1, abort_flag, budget));
      if (!ok) break;
      tc_fence_after();
      // merge weights of the two halves (1 and 0 when not split)
      float w0 = 1.f, w1 = 0.f;
      if (split) {
        const float m1 = xm1[r], l1 = xl1[r];
        const float mm = fmaxf(m_ref, m1);
        w0 = ex2_approx(m_ref - mm);
        w1 = ex2_approx(m1 - mm);
        l_sum = w0 * l_sum + w1 * l1;
        m_ref = mm;
      }
      if (split) {
        // fold warpgroup 1's half (its O in the columns after O0) into O0, so
        // that the output code below is the same for every item
        const uint32_t tO1 = tmem + lane_off + 256u + D;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32], o1[32];
          tmem_ld32(tO + c0, o);
          tmem_ld32(tO1 + c0, o1);
          tmem_ld_wait32(o);
          tmem_ld_wait32(o1);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            o[c] = __float_as_uint(fmaf(w0, __uint_as_float(o[c]), w1 * __uint_as_float(o1[c])));
          tmem_st32(tO + c0, o);
        }
        tmem_st_wait();
      }
      const int row = pair * (kNQ * kBM) + wg * kBM + r;
      const bool row_ok = row < n_q;
      if (sg.slot < 0) {
        const float inv = s_vmax / l_sum;
        const int orow = a.scatter_out && row_ok ? __ldg(a.q_idx + row) : row;
        const bool wr_ok = row_ok && orow >= 0 && orow < a.out_rows;
        __nv_bfloat16 *dst =
            a.out + ((static_cast<int64_t>(P.out_slot) * a.out_rows + (wr_ok ? orow : 0)) * a.H + head) * D;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tO + c0, o);
          tmem_ld_wait32(o);
          if (wr_ok) {
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + c0);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
              d4[v] = w;
            }
          }
        }
      } else {
        const int64_t prow = static_cast<int64_t>(sg.slot) * (kNQ * kBM) + wg * kBM + r;
        float *dst = a.ws_o + prow * D;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tO + c0, o);
          tmem_ld_wait32(o);
          if (row_ok) {
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + c0);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              d4[v] = make_uint4(__float_as_uint(__uint_as_float(o[4 * v]) * s_vmax),
                                 __float_as_uint(__uint_as_float(o[4 * v + 1]) * s_vmax),
                                 __float_as_uint(__uint_as_float(o[4 * v + 2]) * s_vmax),
                                 __float_as_uint(__uint_as_float(o[4 * v + 3]) * s_vmax));
          }
        }
        if (row_ok) *reinterpret_cast<float2 *>(a.ws_ml + prow * 2) = make_float2(m_ref, l_sum);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&o_empty[wg]);
        if (split) mbar_arrive(&o_empty[1]);  // O1 read as well
      }
      ++it;
      if (two || split) ++it1;
      if (split) ++ns;
    }
  }

  // ================================================================ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag && a.dev_status) atomicExch(a.dev_status, CCA_DEV_TIMEOUT);
}

// Merge of the partial pieces of the split items: one warp per (item, row),
// out[row][head] = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s over the CTAs
// whose KV range meets the item.  The schedule is recomputed exactly as the
// attention kernel (launched with G CTAs) computed it; items that fell whole
// inside one CTA's range were written by that CTA and are skipped.  Lane i
// examines candidate CTA c_first + i; the O rows of up to 4 found pieces are
// then loaded by the whole warp at once (lane = D/32 columns) before they are
// summed, so a row costs about two memory round trips when it has at most 4
// pieces.  (4 rather than 8 at once: 64 instead of 73 registers, so 4 blocks
// per SM instead of 3; the 486-query call's combine is latency-bound.)  Launched as a
// programmatic dependent of the attention kernel: it is resident before the
// attention grid ends and waits (griddepcontrol.wait) for that grid's memory
// before reading.
__device__ __forceinline__ int64_t rem_offset(const AttnArgs &a, int n_q0, const Sched &s, int u) {
  int i0 = 0;
  int64_t acc = 0;
  for (int p = 0; p < a.n_prob; ++p) {
    const int cnt = prob_pairs(a, p, n_q0) * a.H, i1 = i0 + cnt;
    const int b0 = i0 > s.rem0 ? i0 : s.rem0;
    const int e0 = i1 < u ? i1 : u;
    if (b0 < e0) acc += static_cast<int64_t>(e0 - b0) * a.prob[p].n_kv;
    i0 = i1;
  }
  return acc;
}

template <int D>
__global__ void __launch_bounds__(256) attn_combine_kernel(const __grid_constant__ AttnArgs a, int G) {
  constexpr int kV = D / 32;  // columns per lane
  constexpr int kBatch = 4;   // pieces loaded at once
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int n_q0 = a.n_q_dev ? min(max(*a.n_q_dev, 0), a.prob[0].n_q) : a.prob[0].n_q;
  const Sched sch = make_sched(a, n_q0, G);
  if (sch.tr == 0) return;  // nothing split
  const int lane = threadIdx.x & 31;
  const int64_t tr = sch.tr;
  // Range bounds floor(c * tr / G) and ceil(x * G / tr) in 32-bit arithmetic when
  // every product fits (always at the sizes of one chunk), else in 64-bit.
  const bool small = (tr + 1) * (G + 1) < (int64_t(1) << 32);
  auto bound = [&](int64_t c) -> int64_t {
    if (small) return static_cast<uint32_t>(c) * static_cast<uint32_t>(tr) / static_cast<uint32_t>(G);
    return c * tr / G;
  };
  auto ceil_div = [&](int64_t x) -> int64_t {
    if (small)
      return (static_cast<uint32_t>(x) * static_cast<uint32_t>(G) + static_cast<uint32_t>(tr) - 1u) /
             static_cast<uint32_t>(tr);
    return (x * G + tr - 1) / tr;
  };
  const int n_work = (sch.n_items - sch.rem0) * (kNQ * kBM);
  const int w0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int w = w0; w < n_work; w += nw) {
    const int ur = w / (kNQ * kBM), rr = w % (kNQ * kBM);
    const int u = sch.rem0 + ur;
    int p, pair, head;
    item_coords(a, n_q0, u, p, pair, head);
    const int row = pair * (kNQ * kBM) + rr;
    if (row >= prob_nq(a, p, n_q0)) continue;
    // candidate CTAs c_first .. c_last; probe(c) says whether c holds a piece
    // of this item and in which workspace slot
    int c_first, c_last;
    int64_t t0 = 0, t1 = 0;
    const int n_kv = a.prob[p].n_kv;
    if (sch.s > 0) {
      c_first = ur * sch.s;
      c_last = c_first + sch.s - 1;
    } else {
      t0 = rem_offset(a, n_q0, sch, u);  // the item's tiles in the list
      t1 = t0 + n_kv;
      c_first = static_cast<int>(ceil_div(t0 + 1)) - 1;
      c_last = min(G - 1, static_cast<int>(ceil_div(t1)));
      const int64_t lo = bound(c_first), hi = bound(c_first + 1);
      if (lo <= t0 && hi >= t1) continue;  // whole inside one CTA's range: written directly by that CTA
    }
    auto probe = [&](int c, int &slot) {
      if (c > c_last) return false;
      if (sch.s > 0) {
        const int j = c - c_first;
        slot = 2 * c;
        return j * n_kv / sch.s < (j + 1) * n_kv / sch.s;
      }
      const int64_t lo = bound(c), hi = bound(c + 1);
      slot = 2 * c + (lo >= t0 ? 0 : 1);
      return lo < hi && hi > t0 && lo < t1;
    };
    // pass 1: (m, l) of every piece, one lane per candidate
    float mmax = -INFINITY;
    for (int cb = c_first; cb <= c_last; cb += 32) {
      int slot;
      if (probe(cb + lane, slot))
        mmax = fmaxf(mmax, __ldcg(a.ws_ml + (static_cast<int64_t>(slot) * (kNQ * kBM) + rr) * 2));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mmax = fmaxf(mmax, __shfl_xor_sync(0xffffffffu, mmax, o));
    float den = 0.f, acc[kV];
#pragma unroll
    for (int k = 0; k < kV; ++k) acc[k] = 0.f;
    for (int cb = c_first; cb <= c_last; cb += 32) {
      int slot = 0;
      const bool mine = probe(cb + lane, slot);
      float wgt = 0.f;
      if (mine) {
        const float2 ml =
            __ldcg(reinterpret_cast<const float2 *>(a.ws_ml + (static_cast<int64_t>(slot) * (kNQ * kBM) + rr) * 2));
        wgt = exp2f(ml.x - mmax);
        den += wgt * ml.y;
      }
      // pass 2: O rows of the found pieces, kBatch loads in flight per lane
      unsigned todo = __ballot_sync(0xffffffffu, mine);
      while (todo) {
        float ws[kBatch], x[kBatch][kV];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          const int src = todo ? __ffs(todo) - 1 : 0;
          const bool live = todo != 0;
          todo &= todo - 1;
          ws[b] = live ? __shfl_sync(0xffffffffu, wgt, src) : 0.f;
          const int sl = __shfl_sync(0xffffffffu, slot, src);
          const float *o = a.ws_o + (static_cast<int64_t>(sl) * (kNQ * kBM) + rr) * D + lane * kV;
          if (live) {
            if constexpr (kV == 4) {
              const float4 v = __ldcg(reinterpret_cast<const float4 *>(o));
              x[b][0] = v.x, x[b][1] = v.y, x[b][2] = v.z, x[b][3] = v.w;
            } else {
              const float2 v = __ldcg(reinterpret_cast<const float2 *>(o));
              x[b][0] = v.x, x[b][1] = v.y;
            }
          } else {
#pragma unroll
            for (int k = 0; k < kV; ++k) x[b][k] = 0.f;
          }
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b)
#pragma unroll
          for (int k = 0; k < kV; ++k) acc[k] += ws[b] * x[b][k];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float inv = 1.f / den;
    const int orow = a.scatter_out ? __ldg(a.q_idx + row) : row;  // fused scatter-back
    if (orow < 0 || orow >= a.out_rows) continue;                 // bad index (flagged by the gather)
    __nv_bfloat16 *dst =
        a.out + ((static_cast<int64_t>(a.prob[p].out_slot) * a.out_rows + orow) * a.H + head) * D + lane * kV;
    if constexpr (kV == 4) {
      *reinterpret_cast<uint2 *>(dst) = make_uint2(sm100::pack_bf16x2(acc[0] * inv, acc[1] * inv),
                                                   sm100::pack_bf16x2(acc[2] * inv, acc[3] * inv));
    } else {
      *reinterpret_cast<uint32_t *>(dst) = sm100::pack_bf16x2(acc[0] * inv, acc[1] * inv);
    }
  }
}

// ------------------------------------------------------------------ host side
static PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [slots][rows][H][D] bf16/e4m3 tensor as a rank-4 map; box = 128 bytes of D x
// 1 head x 128 rows x 1 slot, 128-byte swizzle, zero fill past the rows of a
// slot.  Encoded maps are kept in a small per-thread cache keyed by everything
// they depend on, so a stream loop that reuses its buffers encodes each once.
static cca_status make_tmap(CUtensorMap *tm, const void *ptr, CUtensorMapDataType dt, int esize, int D, int H,
                            int rows, int slots) {
  struct Entry {
    const void *ptr;
    int dt, D, H, rows, slots;
    CUtensorMap map;
  };
  constexpr int kCache = 32;
  thread_local Entry cache[kCache];
  thread_local int n_cached = 0, next = 0;
  for (int i = 0; i < n_cached; ++i) {
    const Entry &e = cache[i];
    if (e.ptr == ptr && e.dt == static_cast<int>(dt) && e.D == D && e.H == H && e.rows == rows &&
        e.slots == slots) {
      *tm = e.map;
      return CCA_OK;
    }
  }
  auto enc = tmap_encoder();
  if (!enc) return fail(CCA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(slots)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * esize, static_cast<cuuint64_t>(H) * D * esize,
                           static_cast<cuuint64_t>(rows) * H * D * esize};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / esize), 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(tm, dt, 4, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CCA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  Entry &e = n_cached < kCache ? cache[n_cached++] : cache[next++ % kCache];
  e = {ptr, static_cast<int>(dt), D, H, rows, slots, *tm};
  return CCA_OK;
}

// [rows][H][D] tensor viewed as [rows][H*D] for TMA row gathers: box = 128
// bytes x one row (the gather4 form), 128-byte swizzle, zeros past the rows.
static cca_status make_gather_map(CUtensorMap *tm, const void *ptr, CUtensorMapDataType dt, int esize, int D, int H,
                                  int rows) {
  auto enc = tmap_encoder();
  if (!enc) return fail(CCA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(H) * D, static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(H) * D * esize};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esize), 1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CCA_ERR_CUDA, "cuTensorMapEncodeTiled (gather) failed (%d)", static_cast<int>(r));
  return CCA_OK;
}

static int env_int(const char *name, int dflt) {
  const char *s = std::getenv(name);
  return s && *s ? std::atoi(s) : dflt;
}

// One kernel launch: the arguments plus the tensors behind the maps.
struct AttnLaunch {
  AttnArgs args;
  const void *q;  // Q tensor [q_slots][q_rows][H][D] (dense path)
  int q_rows_map, q_slots;
  const void *k[kMaxSrc], *v[kMaxSrc];
  int src_slots[kMaxSrc];
  int D;
  bool fp8;
  int64_t work;  // upper bound on (item, KV tile) pairs, for the grid size
};

// Persistent grid: one CTA per SM (CCA_ATTN_CTAS overrides), never more CTAs
// than (item, KV tile) pairs of work.
static int attn_grid(int64_t work) {
  int g = env_int("CCA_ATTN_CTAS", 0);
  if (g <= 0) g = num_sms();
  if (work < g) g = static_cast<int>(work > 0 ? work : 1);
  return g;
}

// Partial-piece slots: 2 per CTA, 256 rows each, O (D fp32) plus (m, l).
static size_t workspace_bytes_for_grid(int grid, int D) {
  const size_t rows = static_cast<size_t>(2) * grid * (kNQ * kBM);
  return rows * (static_cast<size_t>(D) + 2) * sizeof(float) + 256;
}

// Workspace that suffices for every attention launch with this head_dim on
// the current device (the grid never exceeds CCA_ATTN_CTAS or the SM count).
static size_t workspace_bytes_any(int D) {
  int g = env_int("CCA_ATTN_CTAS", 0);
  if (g <= 0) g = num_sms();
  return workspace_bytes_for_grid(g, D);
}

// Host copy of the device schedule's decision (make_sched with every
// problem's n_q): 0 = no item split, 1 = ranges, 2 = aligned pieces; *n_split
// = the items that are split.
static int host_split_mode(const AttnArgs &a, int G, int *n_split) {
  *n_split = 0;
  int n = 0;
  int64_t total = 0;
  for (int p = 0; p < a.n_prob; ++p) {
    const int cnt = (a.prob[p].n_q + kNQ * kBM - 1) / (kNQ * kBM) * a.H;
    n += cnt;
    total += static_cast<int64_t>(cnt) * a.prob[p].n_kv;
  }
  const int q = n / G, r = n % G;
  if (r == 0) return 0;
  int i0 = 0, nkv_first = 0;
  int64_t tr = 0;
  for (int p = 0; p < a.n_prob; ++p) {
    const int cnt = (a.prob[p].n_q + kNQ * kBM - 1) / (kNQ * kBM) * a.H, i1 = i0 + cnt;
    const int b0 = i0 > q * G ? i0 : q * G;
    if (b0 < i1) {
      if (tr == 0) nkv_first = a.prob[p].n_kv;
      tr += static_cast<int64_t>(i1 - b0) * a.prob[p].n_kv;
    }
    i0 = i1;
  }
  if (static_cast<int64_t>(nkv_first) * 8 * G <= total) return 0;
  *n_split = r;
  const int pieces = G / r;
  const int64_t even = (tr + G - 1) / G;
  return pieces >= 2 && (nkv_first + pieces - 1) / pieces <= even + 2 ? 2 : 1;
}

static std::mutex g_attr_mu;

template <int D, bool kFp8>
static cca_status launch_attn(AttnLaunch &L, void *workspace, size_t workspace_bytes, cudaStream_t st) {
  using S = AttnSmem<D, kFp8>;
  AttnArgs &args = L.args;
  const int H = args.H;
  const CUtensorMapDataType dt = kFp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  // V is 16-bit in both modes: bf16, or the e4m3 values widened to fp16
  const CUtensorMapDataType dt_v = kFp8 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int es = kFp8 ? 1 : 2;
  const int grid = attn_grid(L.work);
  const size_t need = workspace_bytes_for_grid(grid, D);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(CCA_ERR_INVALID_ARG, "attention: workspace of %zu bytes (16-byte aligned) required", need);
  args.ws_o = static_cast<float *>(workspace);
  args.ws_ml = args.ws_o + static_cast<size_t>(2) * grid * (kNQ * kBM) * D;
  CUtensorMap tq, tk[kMaxSrc], tv[kMaxSrc];
  std::memset(&tq, 0, sizeof(tq));
  if (!args.q_idx)
    CCA_TRY(make_tmap(&tq, L.q, dt, es, D, H, L.q_rows_map, L.q_slots));
  else
    CCA_TRY(make_gather_map(&tq, args.q, dt, es, D, H, args.q_rows));
  for (int s = 0; s < kMaxSrc; ++s) {
    // An unused source reuses source 1's tensor (never read: no segment names it).
    const bool used = args.src_len[s] > 0;
    const void *kp = used ? L.k[s] : L.k[1], *vp = used ? L.v[s] : L.v[1];
    const int rows = used ? args.src_len[s] : args.src_len[1], slots = used ? L.src_slots[s] : L.src_slots[1];
    CCA_TRY(make_tmap(&tk[s], kp, dt, es, D, H, rows, slots));
    CCA_TRY(make_tmap(&tv[s], vp, dt_v, 2, D, H, rows, slots));
  }
  {
    // The shared-memory opt-in is per device and kernel: set it once per device.
    static bool done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_attr_mu);
    if (dev < 0 || dev >= 64 || !done[dev]) {
      for (auto fn : {attn_kernel<D, kFp8, true>, attn_kernel<D, kFp8, false>}) {
        const cudaError_t e =
            cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(S::kAlloc));
        if (e != cudaSuccess) return fail(CCA_ERR_CUDA, "attention: %s", cudaGetErrorString(e));
      }
      if (dev >= 0 && dev < 64) done[dev] = true;
    }
  }
  if (args.q_idx)
    attn_kernel<D, kFp8, false><<<grid, kThreads, S::kAlloc, st>>>(tq, tk[0], tv[0], tk[1], tv[1], tk[2], tv[2], args);
  else
    attn_kernel<D, kFp8, true><<<grid, kThreads, S::kAlloc, st>>>(tq, tk[0], tv[0], tk[1], tv[1], tk[2], tv[2], args);
  CCA_TRY(launched("attn_kernel"));
  // The combine kernel runs unless the host knows the schedule splits no item.
  int n_split = 0;
  const int mode = host_split_mode(args, grid, &n_split);
  if (args.n_q_dev != nullptr || mode != 0) {
    // one warp per row of a split item: every item may be split when the query
    // count is read on the device, else the host knows how many are
    const int64_t warps = static_cast<int64_t>(args.n_q_dev != nullptr ? grid : n_split) * (kNQ * kBM);
    int64_t blocks = (warps + 7) / 8;
    const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t le = cudaLaunchKernelEx(&cfg, attn_combine_kernel<D>, args, grid);
    if (le != cudaSuccess) {
      cudaGetLastError();
      return fail(CCA_ERR_CUDA, "attention: combine launch failed: %s", cudaGetErrorString(le));
    }
    CCA_TRY(launched("attn_combine_kernel"));
  }
  return CCA_OK;
}

static cca_status run_launch(AttnLaunch &L, void *workspace, size_t workspace_bytes, cudaStream_t st) {
  if (L.fp8) return launch_attn<128, true>(L, workspace, workspace_bytes, st);
  if (L.D == 128) return launch_attn<128, false>(L, workspace, workspace_bytes, st);
  return launch_attn<64, false>(L, workspace, workspace_bytes, st);
}

// Builder of the problem / segment tables of one launch.
struct LaunchBuilder {
  AttnLaunch &L;
  int n_seg = 0;
  explicit LaunchBuilder(AttnLaunch &l) : L(l) {}
  bool fits(int extra_segs) const { return L.args.n_prob < kMaxProb && n_seg + extra_segs <= kMaxSegs; }
  // Start a problem; segments follow with add_seg.
  void begin(int n_q, int q_slot, int out_slot) {
    AttnProb &P = L.args.prob[L.args.n_prob];
    P.n_q = n_q;
    P.q_slot = static_cast<int16_t>(q_slot);
    P.out_slot = static_cast<int16_t>(out_slot);
    P.seg0 = static_cast<int16_t>(n_seg);
    P.n_seg = 0;
    P.n_kv = 0;
  }
  void add_seg(int src, int slot) {
    AttnProb &P = L.args.prob[L.args.n_prob];
    L.args.seg[n_seg] = static_cast<uint16_t>((src << 12) | slot);
    L.args.seg_t0[n_seg] = static_cast<uint16_t>(P.n_kv);
    P.n_kv += (L.args.src_len[src] + kBN - 1) / kBN;
    ++P.n_seg;
    ++n_seg;
  }
  void end() {
    const AttnProb &P = L.args.prob[L.args.n_prob];
    L.work += static_cast<int64_t>((P.n_q + kNQ * kBM - 1) / (kNQ * kBM)) * L.args.H * P.n_kv;
    ++L.args.n_prob;
  }
};

static float scale_log2_of(float softmax_scale, int D) {
  const double scale = softmax_scale > 0.f ? static_cast<double>(softmax_scale) : 1.0 / std::sqrt(static_cast<double>(D));
  return static_cast<float>(scale * 1.4426950408889634);  // scale * log2(e)
}

static long long wait_budget() { return static_cast<long long>(env_int("CCA_WAIT_BUDGET_MCYCLES", 4000)) * 1000000LL; }

}  // namespace cca

using namespace cca;

static cca_status chunk_attn_impl(const cca_kv_ring *ring, const void *q, const void *k_cur, const void *v_cur,
                                  const float *q_scale, const float *kcur_scale, const float *vcur_scale,
                                  const int32_t *q_idx, const int32_t *n_q_dev, int32_t n_q_max,
                                  float softmax_scale, void *out, int scatter_out, void *workspace,
                                  size_t workspace_bytes, cca_stream_t stream);

extern "C" {

#ifdef CCA_TRACE
// Trace builds only: copy the 4 x 16K trace records to host and clear them.
int cca_debug_trace_read(unsigned long long *host, int max_n) {
  const int n = max_n < (4 << 14) ? max_n : (4 << 14);
  cudaDeviceSynchronize();
  cudaMemcpyFromSymbol(host, g_trace, n * sizeof(unsigned long long));
  static unsigned long long zeros[4 << 14];
  cudaMemcpyToSymbol(g_trace, zeros, sizeof(zeros));
  return n;
}
#endif

cca_status cca_chunk_attn_workspace_size(const cca_kv_ring *ring, int32_t n_q_max, size_t *bytes) {
  if (!ring || !bytes || n_q_max < 0 || n_q_max > ring->d.chunk_len)
    return fail(CCA_ERR_INVALID_ARG, "cca_chunk_attn_workspace_size: bad argument");
  *bytes = n_q_max == 0 ? 0 : workspace_bytes_any(ring->d.head_dim);
  return CCA_OK;
}

cca_status cca_attn_workspace_size(int32_t head_dim, size_t *bytes) {
  if (!bytes || (head_dim != 64 && head_dim != 128))
    return fail(CCA_ERR_INVALID_ARG, "cca_attn_workspace_size: head_dim must be 64 or 128");
  *bytes = workspace_bytes_any(head_dim);
  return CCA_OK;
}

cca_status cca_chunk_attn(const cca_kv_ring *ring, const void *q, const void *k_cur, const void *v_cur,
                          const float *q_scale, const float *kcur_scale, const float *vcur_scale,
                          const int32_t *q_idx, const int32_t *n_q_dev, int32_t n_q_max, float softmax_scale,
                          void *out, void *workspace, size_t workspace_bytes, cca_stream_t stream) {
  return chunk_attn_impl(ring, q, k_cur, v_cur, q_scale, kcur_scale, vcur_scale, q_idx, n_q_dev, n_q_max,
                         softmax_scale, out, 0, workspace, workspace_bytes, stream);
}

cca_status cca_chunk_attn_scatter(const cca_kv_ring *ring, const void *q, const void *k_cur, const void *v_cur,
                                  const float *q_scale, const float *kcur_scale, const float *vcur_scale,
                                  const int32_t *q_idx, const int32_t *n_q_dev, int32_t n_q_max,
                                  float softmax_scale, void *o_cache, void *workspace, size_t workspace_bytes,
                                  cca_stream_t stream) {
  if (n_q_max > 0 && !q_idx)
    return fail(CCA_ERR_INVALID_ARG, "cca_chunk_attn_scatter: q_idx is required (it also names the output rows)");
  return chunk_attn_impl(ring, q, k_cur, v_cur, q_scale, kcur_scale, vcur_scale, q_idx, n_q_dev, n_q_max,
                         softmax_scale, o_cache, 1, workspace, workspace_bytes, stream);
}

}  // extern "C"

// Common checks of the e4m3 scale pointers (all non-NULL, 4-byte aligned) or
// their absence for BF16.
static cca_status check_scales(const char *what, cca_dtype dt, std::initializer_list<const float *> sc) {
  if (dt == CCA_E4M3) {
    for (const float *p : sc) {
      if (!p) return fail(CCA_ERR_INVALID_ARG, "%s: E4M3 needs every per-head scale", what);
      if (reinterpret_cast<uintptr_t>(p) & 3) return fail(CCA_ERR_INVALID_ARG, "%s: scales must be 4-byte aligned", what);
    }
  } else {
    for (const float *p : sc)
      if (p) return fail(CCA_ERR_INVALID_ARG, "%s: BF16 takes no scales", what);
  }
  return CCA_OK;
}

// The ring's cached chunks visible from its current chunk, as segments of source 0.
static void add_ring_segments(const cca_kv_ring *ring, LaunchBuilder &b) {
  int32_t slots[kMaxWindow + 1];
  const int n = ring_visible(ring, slots, nullptr);
  for (int c = 0; c < n; ++c) b.add_seg(0, slots[c]);
}

static void init_launch(AttnLaunch &L, int H, int D, cca_dtype dt, float softmax_scale, int32_t *dev_status) {
  std::memset(&L, 0, sizeof(L));
  L.args.H = H;
  L.D = D;
  L.fp8 = dt == CCA_E4M3;
  L.args.scale_log2 = scale_log2_of(softmax_scale, D);
  L.args.wait_budget = wait_budget();
  L.args.dev_status = dev_status;
}

static cca_status chunk_attn_impl(const cca_kv_ring *ring, const void *q, const void *k_cur, const void *v_cur,
                                  const float *q_scale, const float *kcur_scale, const float *vcur_scale,
                                  const int32_t *q_idx, const int32_t *n_q_dev, int32_t n_q_max,
                                  float softmax_scale, void *out, int scatter_out, void *workspace,
                                  size_t workspace_bytes, cca_stream_t stream) {
  if (!ring) return fail(CCA_ERR_INVALID_ARG, "cca_chunk_attn: NULL ring");
  const cca_kv_ring_desc &d = ring->d;
  if (n_q_max < 0 || n_q_max > d.chunk_len)
    return fail(CCA_ERR_INVALID_ARG, "cca_chunk_attn: need 0 <= n_q_max <= chunk_len (%d)", d.chunk_len);
  if (n_q_max == 0) return CCA_OK;
  if (!q || !k_cur || !v_cur || !out)
    return fail(CCA_ERR_INVALID_ARG, "cca_chunk_attn: q, k_cur, v_cur and out must be non-NULL");
  if (!aligned16(q) || !aligned16(k_cur) || !aligned16(v_cur) || !aligned16(out))
    return fail(CCA_ERR_INVALID_ARG, "cca_chunk_attn: q, k_cur, v_cur and out must be 16-byte aligned");
  CCA_TRY(check_scales("cca_chunk_attn", d.dtype, {q_scale, kcur_scale, vcur_scale}));
  if (d.dtype == CCA_E4M3 && d.head_dim != 128)
    return fail(CCA_ERR_UNSUPPORTED, "cca_chunk_attn: E4M3 attention is built for head_dim 128");
  if ((q_idx && (reinterpret_cast<uintptr_t>(q_idx) & 3)) || (n_q_dev && (reinterpret_cast<uintptr_t>(n_q_dev) & 3)))
    return fail(CCA_ERR_INVALID_ARG, "cca_chunk_attn: q_idx / n_q_dev must be 4-byte aligned");
  AttnLaunch L;
  init_launch(L, d.n_heads, d.head_dim, d.dtype, softmax_scale, d.dev_status);
  AttnArgs &a = L.args;
  a.q = q;
  a.q_idx = q_idx;
  a.n_q_dev = n_q_dev;
  a.out = static_cast<__nv_bfloat16 *>(out);
  a.scatter_out = scatter_out;
  a.q_scale = q_scale;
  a.k_scale[0] = d.k_scale;
  a.v_scale[0] = d.v_scale;
  a.k_scale[1] = kcur_scale;
  a.v_scale[1] = vcur_scale;
  a.out_rows = scatter_out ? d.chunk_len : n_q_max;
  a.q_rows = d.chunk_len;
  a.src_len[0] = d.chunk_len;
  a.src_len[1] = d.chunk_len;
  L.q = q;
  L.q_rows_map = n_q_max;
  L.q_slots = 1;
  L.k[0] = d.k_slots;
  L.v[0] = d.v_slots;
  L.src_slots[0] = 1 + d.window;
  L.k[1] = k_cur;
  L.v[1] = v_cur;
  L.src_slots[1] = 1;
  LaunchBuilder b(L);
  b.begin(n_q_max, 0, 0);
  add_ring_segments(ring, b);
  b.add_seg(1, 0);
  b.end();
  return run_launch(L, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" {

cca_status cca_chunk_attn_groups(const cca_kv_ring *ring, const void *q, const void *k_cur, const void *v_cur,
                                 int32_t n_cur, const void *k_ref, const void *v_ref, int32_t n_ref,
                                 const float *q_scale, const float *kcur_scale, const float *vcur_scale,
                                 const float *kref_scale, const float *vref_scale, float softmax_scale, void *out,
                                 void *workspace, size_t workspace_bytes, cca_stream_t stream) {
  const char *what = "cca_chunk_attn_groups";
  if (!ring) return fail(CCA_ERR_INVALID_ARG, "%s: NULL ring", what);
  const cca_kv_ring_desc &d = ring->d;
  if (n_cur < 0 || n_cur > (1 << 24) || n_ref < 0 || n_ref > (1 << 24))
    return fail(CCA_ERR_INVALID_ARG, "%s: need 0 <= n_cur, n_ref <= 2^24", what);
  if (n_cur == 0) return CCA_OK;
  if (!q || !k_cur || !v_cur || !out || (n_ref > 0 && (!k_ref || !v_ref)))
    return fail(CCA_ERR_INVALID_ARG, "%s: q, k_cur, v_cur, out (and k_ref, v_ref when n_ref > 0) must be non-NULL",
                what);
  if (!aligned16(q) || !aligned16(k_cur) || !aligned16(v_cur) || !aligned16(out) ||
      (n_ref > 0 && (!aligned16(k_ref) || !aligned16(v_ref))))
    return fail(CCA_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", what);
  if (d.dtype == CCA_E4M3 && d.head_dim != 128)
    return fail(CCA_ERR_UNSUPPORTED, "%s: E4M3 attention is built for head_dim 128", what);
  CCA_TRY(check_scales(what, d.dtype, {q_scale, kcur_scale, vcur_scale}));
  if (n_ref > 0) CCA_TRY(check_scales(what, d.dtype, {kref_scale, vref_scale}));
  AttnLaunch L;
  init_launch(L, d.n_heads, d.head_dim, d.dtype, softmax_scale, d.dev_status);
  AttnArgs &a = L.args;
  a.q = q;
  a.out = static_cast<__nv_bfloat16 *>(out);
  a.q_scale = q_scale;
  a.k_scale[0] = d.k_scale;
  a.v_scale[0] = d.v_scale;
  a.k_scale[1] = kcur_scale;
  a.v_scale[1] = vcur_scale;
  a.k_scale[2] = kref_scale;
  a.v_scale[2] = vref_scale;
  a.out_rows = n_cur;
  a.q_rows = n_cur;
  a.src_len[0] = d.chunk_len;
  a.src_len[1] = n_cur;
  a.src_len[2] = n_ref;
  L.q = q;
  L.q_rows_map = n_cur;
  L.q_slots = 1;
  L.k[0] = d.k_slots;
  L.v[0] = d.v_slots;
  L.src_slots[0] = 1 + d.window;
  L.k[1] = k_cur;
  L.v[1] = v_cur;
  L.src_slots[1] = 1;
  L.k[2] = k_ref;
  L.v[2] = v_ref;
  L.src_slots[2] = 1;
  LaunchBuilder b(L);
  b.begin(n_cur, 0, 0);
  if (n_ref > 0) b.add_seg(2, 0);
  add_ring_segments(ring, b);
  b.add_seg(1, 0);
  b.end();
  return run_launch(L, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

cca_status cca_block_attn(const cca_block_desc *bd, const void *q, const float *q_scale, float softmax_scale,
                          void *out, void *workspace, size_t workspace_bytes, cca_stream_t stream) {
  const char *what = "cca_block_attn";
  if (!bd) return fail(CCA_ERR_INVALID_ARG, "%s: NULL descriptor", what);
  const cca_block_desc &d = *bd;
  const int T = d.n_chunks, Lc = d.chunk_len, W = d.window;
  if (d.n_heads < 1 || (d.head_dim != 64 && d.head_dim != 128) || Lc < 1 || T < 0 || T > 4095 || W < 0 ||
      d.ref_len < 0 || d.ref_len > (1 << 24) || (d.dtype != CCA_BF16 && d.dtype != CCA_E4M3) ||
      static_cast<int64_t>(Lc) * d.n_heads * d.head_dim > (int64_t(1) << 33))
    return fail(CCA_ERR_INVALID_ARG, "%s: bad dims (H >= 1, D in {64,128}, L >= 1, 0 <= T <= 4095, W >= 0)", what);
  if (d.dtype == CCA_E4M3 && d.head_dim != 128)
    return fail(CCA_ERR_UNSUPPORTED, "%s: E4M3 attention is built for head_dim 128", what);
  if (T == 0) return CCA_OK;
  if (!q || !out || !d.k_cur || !d.v_cur || !d.k_hist || !d.v_hist || (d.ref_len > 0 && (!d.k_ref || !d.v_ref)))
    return fail(CCA_ERR_INVALID_ARG, "%s: NULL tensor", what);
  const void *const tens[6] = {q, out, d.k_cur, d.v_cur, d.k_hist, d.v_hist};
  for (const void *p : tens)
    if (!aligned16(p)) return fail(CCA_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", what);
  if (d.ref_len > 0 && (!aligned16(d.k_ref) || !aligned16(d.v_ref)))
    return fail(CCA_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", what);
  CCA_TRY(check_scales(what, d.dtype, {q_scale, d.kcur_scale, d.vcur_scale, d.khist_scale, d.vhist_scale}));
  if (d.ref_len > 0) CCA_TRY(check_scales(what, d.dtype, {d.kref_scale, d.vref_scale}));
  AttnLaunch base;
  init_launch(base, d.n_heads, d.head_dim, d.dtype, softmax_scale, d.dev_status);
  AttnArgs &a = base.args;
  a.q = q;
  a.out = static_cast<__nv_bfloat16 *>(out);
  a.q_scale = q_scale;
  a.k_scale[0] = d.khist_scale;
  a.v_scale[0] = d.vhist_scale;
  a.k_scale[1] = d.kcur_scale;
  a.v_scale[1] = d.vcur_scale;
  a.k_scale[2] = d.kref_scale;
  a.v_scale[2] = d.vref_scale;
  a.out_rows = Lc;
  a.q_rows = Lc;
  a.src_len[0] = Lc;
  a.src_len[1] = Lc;
  a.src_len[2] = d.ref_len;
  base.q = q;
  base.q_rows_map = Lc;
  base.q_slots = T;
  base.k[0] = d.k_hist;
  base.v[0] = d.v_hist;
  base.src_slots[0] = T;
  base.k[1] = d.k_cur;
  base.v[1] = d.v_cur;
  base.src_slots[1] = T;
  base.k[2] = d.k_ref;
  base.v[2] = d.v_ref;
  base.src_slots[2] = 1;
  // Chunk c sees R, history chunks {0} U {max(1, c-W) .. c-1} and its own
  // current chunk.  Chunks are listed longest visible list first (the schedule
  // wants problems by non-increasing KV length) and cut into launches that fit
  // the argument tables.
  auto n_hist = [&](int c) { return c == 0 ? 0 : 1 + (c - 1 - (c - W > 1 ? c - W : 1) + 1); };
  std::vector<int> order(T);
  for (int c = 0; c < T; ++c) order[c] = c;
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return n_hist(x) > n_hist(y); });
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  for (int i = 0; i < T;) {
    AttnLaunch L = base;
    LaunchBuilder b(L);
    for (; i < T; ++i) {
      const int c = order[i];
      const int need = n_hist(c) + 1 + (d.ref_len > 0 ? 1 : 0);
      if (need > kMaxSegs) return fail(CCA_ERR_UNSUPPORTED, "%s: %d visible segments exceed %d", what, need, kMaxSegs);
      if (!b.fits(need)) break;
      b.begin(Lc, c, c);
      if (d.ref_len > 0) b.add_seg(2, 0);
      if (c > 0) {
        b.add_seg(0, 0);
        for (int h = (c - W > 1 ? c - W : 1); h < c; ++h) b.add_seg(0, h);
      }
      b.add_seg(1, c);
      b.end();
    }
    CCA_TRY(run_launch(L, workspace, workspace_bytes, st));
  }
  return CCA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ allocation-free variant
// Some callers cannot hand this library a scratch buffer: a real-time stream
// loop that must not call the device allocator once it is running (an
// allocation can synchronise the device and stall the stream), or a host
// application that owns every device allocation itself and exposes no
// allocator to plug-ins.  cca_chunk_attn_noalloc serves them from one scratch
// array that lives in this library's device image.
namespace cca {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB per GPU that loads the library
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device.  In host code
// the array's name is only a stand-in, never a device address, so it goes
// through cudaGetSymbolAddress, which allocates nothing.  It is looked up on
// every call rather than cached: after a device reset the library's device
// code is loaded again and the array may sit elsewhere.
static cca_status noalloc_scratch(void **out) {
  void *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || !p)
    return fail(CCA_ERR_CUDA, "cca_chunk_attn_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
  *out = p;
  return CCA_OK;
}

}  // namespace cca

extern "C" {

cca_status cca_chunk_attn_noalloc(const cca_kv_ring *ring, const void *q, const void *k_cur, const void *v_cur,
                                  const float *q_scale, const float *kcur_scale, const float *vcur_scale,
                                  const int32_t *q_idx, const int32_t *n_q_dev, int32_t n_q_max,
                                  float softmax_scale, void *out, cca_stream_t stream) {
  if (!ring) return fail(CCA_ERR_INVALID_ARG, "cca_chunk_attn_noalloc: NULL ring");
  if (n_q_max < 0 || n_q_max > ring->d.chunk_len)
    return fail(CCA_ERR_INVALID_ARG, "cca_chunk_attn_noalloc: need 0 <= n_q_max <= chunk_len (%d)",
                ring->d.chunk_len);
  const size_t need = n_q_max == 0 ? 0 : workspace_bytes_any(ring->d.head_dim);
  if (need > kNoAllocScratchBytes)
    return fail(CCA_ERR_INVALID_ARG,
                "cca_chunk_attn_noalloc: this call needs %zu bytes of scratch, more than the %zu-byte built-in "
                "array; use cca_chunk_attn with a caller-provided workspace",
                need, kNoAllocScratchBytes);
  void *scratch = nullptr;
  CCA_TRY(noalloc_scratch(&scratch));
  return cca_chunk_attn(ring, q, k_cur, v_cur, q_scale, kcur_scale, vcur_scale, q_idx, n_q_dev, n_q_max,
                        softmax_scale, out, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
