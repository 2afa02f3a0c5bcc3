// AR-oriented mask cache: per-token L2 mask, stream compaction, scatter-back.
//
// ["LiveEdit 실시간 Diffusion 기반 스트리밍 비디오 편집", sections 방법론 and
// 기술 상세]: the mask of chunk k is 1 at a token exactly when the L2 norm of
// (edited - source) latents of chunk k-1 at that token exceeds tau; tau is chosen
// dynamically to prune about 70 % of the tokens; active tokens are recomputed and
// inactive tokens reuse the cached self-attention output.
//
// The comparison is done on squares (d^2 > tau^2, both non-negative), in fp32.
// The dynamic threshold is an exact order statistic of the fp32 d^2 values,
// found by a 4 x 8-bit radix select on their bit patterns (for non-negative
// floats the unsigned order of the bits is the numeric order).
#include <cmath>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace cca {

constexpr int kMaskThreads = 256;
constexpr int kSelectThreads = 1024;
constexpr int kMaxSelectTokens = 32768;

// Squared distance of position u over the channels of every latent frame of
// the chunk (frames fstride elements apart; one frame for a one-frame chunk).
__device__ __forceinline__ float token_dist2(const float *__restrict__ src, const float *__restrict__ edit,
                                             int64_t u, int n_ch, int n_frames, int64_t fstride) {
  float acc = 0.f;
  for (int f = 0; f < n_frames; ++f) {
    const float4 *s = reinterpret_cast<const float4 *>(src + f * fstride + u * n_ch);
    const float4 *e = reinterpret_cast<const float4 *>(edit + f * fstride + u * n_ch);
    for (int c = 0; c < n_ch / 4; ++c) {
      const float4 a = __ldg(s + c), b = __ldg(e + c);
      const float d0 = b.x - a.x, d1 = b.y - a.y, d2 = b.z - a.z, d3 = b.w - a.w;
      acc = fmaf(d0, d0, acc);
      acc = fmaf(d1, d1, acc);
      acc = fmaf(d2, d2, acc);
      acc = fmaf(d3, d3, acc);
    }
  }
  return acc;
}

// Fixed threshold: one thread per token, grid-stride.
// With n_frames > 1 the decision of position u is written for every frame:
// mask[f * n_tok + u].
__global__ void __launch_bounds__(kMaskThreads) mask_fixed_kernel(const float *__restrict__ src,
                                                                  const float *__restrict__ edit, int n_tok,
                                                                  int n_ch, float tau2, uint8_t *__restrict__ mask,
                                                                  float *__restrict__ dist2, float *tau_out,
                                                                  int n_frames) {
  const int stride = gridDim.x * blockDim.x;
  const int64_t fstride = static_cast<int64_t>(n_tok) * n_ch;
  for (int u = blockIdx.x * blockDim.x + threadIdx.x; u < n_tok; u += stride) {
    const float d2 = token_dist2(src, edit, u, n_ch, n_frames, fstride);
    const uint8_t m = d2 > tau2 ? 1 : 0;
    for (int f = 0; f < n_frames; ++f) mask[static_cast<int64_t>(f) * n_tok + u] = m;
    if (dist2) dist2[u] = d2;
  }
  if (tau_out && blockIdx.x == 0 && threadIdx.x == 0) *tau_out = sqrtf(tau2);
}

// Dynamic threshold, one CTA: d^2 of every token into shared memory, radix
// select of the k-th smallest (k >= 1), then mask = d^2 > that value.
__global__ void __launch_bounds__(kSelectThreads) mask_select_kernel(const float *__restrict__ src,
                                                                     const float *__restrict__ edit, int n_tok,
                                                                     int n_ch, int k, uint8_t *__restrict__ mask,
                                                                     float *__restrict__ dist2, float *tau_out,
                                                                     int n_frames) {
  const int64_t fstride = static_cast<int64_t>(n_tok) * n_ch;
  extern __shared__ unsigned s_bits[];  // n_tok entries
  __shared__ unsigned hist[256];
  __shared__ unsigned s_prefix, s_rank;
  for (int u = threadIdx.x; u < n_tok; u += blockDim.x) {
    const float d2 = token_dist2(src, edit, u, n_ch, n_frames, fstride);
    s_bits[u] = __float_as_uint(d2);
    if (dist2) dist2[u] = d2;
  }
  if (threadIdx.x == 0) {
    s_prefix = 0u;
    s_rank = static_cast<unsigned>(k);  // 1-based rank still to find inside the prefix bucket
  }
  __syncthreads();
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const unsigned hi_mask = pass == 0 ? 0u : (0xffffffffu << (shift + 8));
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    const unsigned prefix = s_prefix;
    for (int u = threadIdx.x; u < n_tok; u += blockDim.x) {
      const unsigned b = s_bits[u];
      if ((b & hi_mask) == prefix) atomicAdd(&hist[(b >> shift) & 0xffu], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {  // warp 0: lane l owns bins 8l..8l+7; first bin whose running sum reaches rank
      const int lane = threadIdx.x;
      unsigned h[8], own = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) own += (h[j] = hist[8 * lane + j]);
      unsigned incl = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned rank = s_rank;
      const unsigned hit = __ballot_sync(0xffffffffu, incl >= rank);  // nonzero: rank <= count in prefix
      const int owner = __ffs(hit) - 1;
      if (lane == owner) {
        unsigned cum = incl - own;
        int j = 0;
        for (; j < 7; ++j) {
          if (cum + h[j] >= rank) break;
          cum += h[j];
        }
        s_rank = rank - cum;
        s_prefix = prefix | (static_cast<unsigned>(8 * lane + j) << shift);
      }
    }
    __syncthreads();
  }
  const float tau2 = __uint_as_float(s_prefix);
  for (int u = threadIdx.x; u < n_tok; u += blockDim.x) {
    const uint8_t m = __uint_as_float(s_bits[u]) > tau2 ? 1 : 0;
    for (int f = 0; f < n_frames; ++f) mask[static_cast<int64_t>(f) * n_tok + u] = m;
  }
  if (tau_out && threadIdx.x == 0) *tau_out = sqrtf(tau2);
}

// 0x01 in every byte of w that is nonzero, 0x00 elsewhere (the ORs fold each
// byte's bits into its bit 0; what crosses into the next byte lands above bit 0
// and is masked off).
__device__ __forceinline__ uint32_t nonzero_bytes(uint32_t w) {
  w |= w >> 4;
  w |= w >> 2;
  w |= w >> 1;
  return w & 0x01010101u;
}
// Bytes b0..b3 in {0, 1} -> bits b0 | b1 << 1 | b2 << 2 | b3 << 3: the product
// with 0x01020408 puts b_j at bit 24 + j; every other partial product lies
// below bit 20, so nothing carries into bits 24..27.
__device__ __forceinline__ uint32_t gather4(uint32_t ones) { return (ones * 0x01020408u) >> 24; }

// Ordered stream compaction in one CTA: tiles of blockDim.x * 16 mask bytes,
// block-wide exclusive scan of per-thread counts, running offset across tiles.
constexpr int kCompactThreads = 1024;
constexpr int kCompactSingleMax = 16384;  // single-CTA path (one tile) up to here
constexpr int kCompactMaxTokens = 1 << 30;
__global__ void __launch_bounds__(kCompactThreads) compact_kernel(const uint8_t *__restrict__ mask, int n_tok,
                                                                  int32_t *__restrict__ idx,
                                                                  int32_t *__restrict__ n_active) {
  __shared__ int warp_sum[kCompactThreads / 32];
  __shared__ int s_base;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) s_base = 0;
  __syncthreads();
  const int tile = blockDim.x * 16;
  for (int t0 = 0; t0 < n_tok; t0 += tile) {
    const int u0 = t0 + threadIdx.x * 16;
    uint32_t bits = 0;  // bit j: token u0 + j is active
    if (u0 + 16 <= n_tok) {
      const uint4 v = *reinterpret_cast<const uint4 *>(mask + u0);
      bits = gather4(nonzero_bytes(v.x)) | gather4(nonzero_bytes(v.y)) << 4 | gather4(nonzero_bytes(v.z)) << 8 |
             gather4(nonzero_bytes(v.w)) << 12;
    } else {
      for (int j = 0; j < 16 && u0 + j < n_tok; ++j) bits |= (mask[u0 + j] != 0 ? 1u : 0u) << j;
    }
    const int cnt = __popc(bits);
    int incl = cnt;  // inclusive warp scan
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int nw = blockDim.x >> 5;
      int x = lane < nw ? warp_sum[lane] : 0;
      int xi = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, xi, o);
        if (lane >= o) xi += y;
      }
      if (lane < nw) warp_sum[lane] = xi - x;  // exclusive warp offsets
    }
    __syncthreads();
    int pos = s_base + warp_sum[warp] + incl - cnt;
    while (bits) {
      idx[pos++] = u0 + __ffs(bits) - 1;
      bits &= bits - 1;
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) s_base = pos;
    __syncthreads();
  }
  if (threadIdx.x == 0) *n_active = s_base;
}

// ---- multi-CTA ordered compaction for large token counts: one cooperative
// launch of G co-resident CTAs, CTA c owning the contiguous run of 8192-token
// sub-tiles [c S / G, (c+1) S / G).
//  1. count: the CTA streams its run once and keeps each sub-tile's count in
//     shared memory; it publishes its total in status[c] (flag in bits 62-63).
//  2. offset: it sums the totals of CTAs 0 .. c-1, waiting (bounded) for any
//     not yet published.  Every CTA publishes before it waits and all G are
//     resident (cooperative launch), so the waits end.
//  3. write: it streams its run again, last sub-tile first, so that the part
//     still in L2 from pass 1 is read first, and writes each sub-tile's
//     indices, staged in shared memory so that the global stores are
//     contiguous.
// The mask reaches shared memory by bulk copies (one 8 KB copy per sub-tile)
// through a kSegStages-deep ring that thread 0 keeps full across both passes,
// so a CTA has up to 32 KB of loads in flight while it computes.  Unlike a
// decoupled look-back there is no chain of inclusive prefixes: with ~900 tiles
// in flight that chain made every tile wait for the slowest load among its
// predecessors.  On an expired wait the count becomes -1.
constexpr int kSegThreads = 256;
constexpr int kSubTok = kSegThreads * 32;  // 8192 tokens per sub-tile: 32 per thread
constexpr int kSegStages = 4;
constexpr int kBitsSub = 16;  // sub-tiles whose activity bits a CTA can keep (1 KB each)
// dynamic shared memory: the mask ring, then 16 KB that hold either the run's
// activity bits (runs of <= kBitsSub sub-tiles) or the index staging
constexpr int kSegDynSmem = kSegStages * kSubTok + kBitsSub * kSegThreads * 4;
static_assert(kBitsSub * kSegThreads * 4 == kSubTok * 2, "the bits area doubles as the uint16 index staging");
constexpr int kMaxSubPerCta = 1024;
constexpr int kMaxSegCtas = 4096;
constexpr long long kSegBudget = 2000000000LL;  // clock64 cycles per wait, about 1 s

__device__ __forceinline__ unsigned long long ld_status(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_status(unsigned long long *p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__global__ void seg_init_kernel(unsigned long long *status, int32_t *n_active, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) status[i] = 0ull;
  if (blockIdx.x == 0 && threadIdx.x == 0) *n_active = 0x7fffffff;  // lowered by atomicMin
}

// Per-byte nonzero flags of the 32 mask bytes at offset a of sub-tile t0: from
// the staged copy where it holds them, else (ragged end) from global memory.
__device__ __forceinline__ void seg_words(const uint8_t *stage, const uint8_t *__restrict__ mask, int64_t t0, int a,
                                          int staged, int64_t n_tok, uint32_t (&w)[8]) {
#pragma unroll
  for (int v = 0; v < 2; ++v) {
    const int o = a + 16 * v;
    if (o + 16 <= staged) {
      const uint4 x = *reinterpret_cast<const uint4 *>(stage + o);
      w[4 * v] = x.x, w[4 * v + 1] = x.y, w[4 * v + 2] = x.z, w[4 * v + 3] = x.w;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t acc = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int64_t u = t0 + o + 4 * j + b;
          if (u < n_tok && mask[u]) acc |= 1u << (8 * b);
        }
        w[4 * v + j] = acc;
      }
    }
  }
  // Masks written by cca_token_mask_l2 hold only 0 and 1; fold other nonzero
  // bytes to 1 only when the warp has met one.
  uint32_t big = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) big |= w[i] & 0xfefefefeu;
  if (__any_sync(0xffffffffu, big != 0)) {
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = nonzero_bytes(w[i]);
  }
}

#ifndef CCA_SEG_MINB
#define CCA_SEG_MINB 4
#endif
__global__ void __launch_bounds__(kSegThreads, CCA_SEG_MINB) compact_seg_kernel(const uint8_t *__restrict__ mask,
                                                                               int n_tok, int32_t *__restrict__ idx,
                                                                               int32_t *n_active,
                                                                               unsigned long long *status,
                                                                               int n_sub) {
  extern __shared__ __align__(128) uint8_t seg_dyn[];
  uint8_t(*ring)[kSubTok] = reinterpret_cast<uint8_t(*)[kSubTok]>(seg_dyn);  // kSegStages x kSubTok bytes
  uint8_t *ext = seg_dyn + kSegStages * kSubTok;                            // 16 KB
  __shared__ uint64_t full[kSegStages];
  __shared__ int s_cnt[kMaxSubPerCta];  // counts per sub-tile, then exclusive offsets within the run
  __shared__ int warp_sum[2][kSegThreads / 32];      // pass 3, by sub-tile parity
  __shared__ int s_wcnt[kBitsSub][kSegThreads / 32];  // kept bits: active tokens per (sub-tile, warp)
  __shared__ unsigned long long s_part[kSegThreads / 32];
  __shared__ int s_total, s_fail;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = blockIdx.x, G = gridDim.x;
  const int sub0 = static_cast<int>(static_cast<int64_t>(n_sub) * c / G);
  const int sub1 = static_cast<int>(static_cast<int64_t>(n_sub) * (c + 1) / G);
  const int n_mine = sub1 - sub0, n_items = 2 * n_mine;
  // A short run keeps each thread's 32 activity bits per sub-tile from pass 1
  // (in ext) and each warp's count per sub-tile, so pass 3 neither re-reads nor
  // re-decodes the mask, needs no block barrier per sub-tile, and stages its
  // indices as int32 in the then idle ring; a long run re-reads the mask in
  // pass 3 and stages 16-bit offsets in ext.
  const bool keep_bits = n_mine <= kBitsSub;
  uint32_t *s_bits = reinterpret_cast<uint32_t *>(ext);  // [sub-tile][thread]
  uint16_t *s_idx = reinterpret_cast<uint16_t *>(ext);
  const int n_loads = keep_bits ? n_mine : n_items;  // items whose mask bytes come through the ring
  // item k: pass 1 reads sub-tile sub0 + k, pass 3 reads sub1 - 1 - (k - n_mine)
  auto item_sub = [&](int k) { return k < n_mine ? sub0 + k : sub1 - 1 - (k - n_mine); };
  auto item_len = [&](int k) {
    const int64_t t0 = static_cast<int64_t>(item_sub(k)) * kSubTok;
    return static_cast<int>(n_tok - t0 < kSubTok ? n_tok - t0 : kSubTok);
  };
  int issued = 0;
  auto issue = [&]() {  // thread 0: next item into its stage
    const int k = issued++;
    const int st = k % kSegStages;
    const uint32_t bytes = static_cast<uint32_t>(item_len(k)) & ~15u;  // the ragged <16 bytes are read directly
    sm100::mbar_arrive_expect_tx(&full[st], bytes);
    if (bytes) sm100::bulk_load(smem_u32(ring[st]), mask + static_cast<int64_t>(item_sub(k)) * kSubTok, bytes, &full[st]);
  };
  for (int i = threadIdx.x; i < n_mine; i += kSegThreads) s_cnt[i] = 0;
  if (threadIdx.x == 0) {
    s_fail = 0;
    for (int st = 0; st < kSegStages; ++st) sm100::mbar_init(&full[st], 1);
    sm100::fence_mbar_init();
    while (issued < n_loads && issued < kSegStages) issue();
  }
  __syncthreads();
  const int a = 32 * threadIdx.x;  // this thread's 32 tokens within a sub-tile
  int k = 0;
  // 1. counts
  for (; k < n_mine; ++k) {
    const int st = k % kSegStages;
    sm100::mbar_wait(&full[st], static_cast<uint32_t>((k / kSegStages) & 1), &s_fail, kSegBudget);
    const int64_t t0 = static_cast<int64_t>(sub0 + k) * kSubTok;
    uint32_t w[8];
    seg_words(ring[st], mask, t0, a, item_len(k) & ~15, n_tok, w);
    int cnt = 0;  // bytes are 0 / 1 here: a byte dot product counts them
    if (keep_bits) {
      uint32_t bits = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) bits |= gather4(w[i]) << (4 * i);
      s_bits[k * kSegThreads + threadIdx.x] = bits;
      cnt = __popc(bits);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) cnt = static_cast<int>(__dp4a(w[i], 0x01010101u, static_cast<unsigned>(cnt)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) {
      atomicAdd(&s_cnt[k], cnt);
      if (keep_bits) s_wcnt[k][warp] = cnt;
    }
    __syncthreads();  // stage st consumed by every thread; s_fail is uniform until the next wait
    if (s_fail) break;
    if (threadIdx.x == 0 && issued < n_loads) issue();
  }
  if (warp == 0) {  // exclusive scan of the run's counts, 32 at a time
    int carry = 0;
    for (int i0 = 0; i0 < n_mine; i0 += 32) {
      const int x = i0 + lane < n_mine ? s_cnt[i0 + lane] : 0;
      int xi = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, xi, o);
        if (lane >= o) xi += y;
      }
      if (i0 + lane < n_mine) s_cnt[i0 + lane] = carry + xi - x;
      carry += __shfl_sync(0xffffffffu, xi, 31);
    }
    if (lane == 0) {
      s_total = carry;
      st_status(&status[c], (1ull << 62) | static_cast<unsigned>(carry));
    }
  }
  // 2. offset of this run: totals of all earlier runs
  unsigned long long v = 0;
  for (int q = threadIdx.x; q < c; q += kSegThreads) {
    unsigned long long sw = ld_status(&status[q]);
    if ((sw >> 62) == 0) {
      const long long c0 = clock64();
      unsigned ns = 32;
      while (((sw = ld_status(&status[q])) >> 62) == 0) {
        if (clock64() - c0 > kSegBudget || s_fail) {
          s_fail = 1;
          break;
        }
        __nanosleep(ns);
        if (ns < 256) ns *= 2;
      }
    }
    v += sw & 0xffffffffull;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) s_part[warp] = v;
  __syncthreads();
  unsigned long long excl = 0;
#pragma unroll
  for (int w = 0; w < kSegThreads / 32; ++w) excl += s_part[w];
  // 3. indices, last sub-tile first
  if (s_fail) k = n_items;  // uniform: read after the barrier above
  if (keep_bits) {
    // Warps run independently: a warp's offset within a sub-tile is the sum of
    // the earlier warps' counts from pass 1.  It stages its indices (int32) in
    // its 4 KB of the ring at the store address's position modulo 16 bytes, so
    // that the run leaves as 16-byte stores with at most 3 scalar ones per end.
    int *mine = reinterpret_cast<int *>(seg_dyn) + warp * 1024;
    for (; k < n_items; ++k) {
      const int s = item_sub(k), kk = s - sub0;
      uint32_t bits = s_bits[kk * kSegThreads + threadIdx.x];
      const int cnt = __popc(bits);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int wcnt = __shfl_sync(0xffffffffu, incl, 31);
      int wofs = 0;
#pragma unroll
      for (int w = 0; w < kSegThreads / 32; ++w) wofs += w < warp ? s_wcnt[kk][w] : 0;
      int32_t *dst = idx + excl + s_cnt[kk] + wofs;
      // dst's position in its 16-byte group; when the run would not fit behind
      // that offset ((almost) every token of the warp active) it goes out as
      // scalar stores from offset 0
      const int mis = static_cast<int>((reinterpret_cast<uintptr_t>(dst) >> 2) & 3u);
      const bool vec = mis + wcnt <= 1024;
      const int off = vec ? mis : 0;
      int pos = off + incl - cnt;
      const int tb = static_cast<int>(static_cast<int64_t>(s) * kSubTok) + a - 1;
      while (bits) {  // set bits only, lowest first
        mine[pos++] = tb + __ffs(bits);
        bits &= bits - 1;
      }
      __syncwarp();
      const int pend = off + wcnt;
      const int qa = (off + 3) >> 2, qb = pend >> 2;  // whole 16-byte groups [qa, qb) of the staging
      if (vec && qa < qb) {
        for (int q = qa + lane; q < qb; q += 32)
          __stcs(reinterpret_cast<int4 *>(dst + (4 * q - off)), *reinterpret_cast<const int4 *>(mine + 4 * q));
        const int nh = 4 * qa - off, nt = pend - 4 * qb;  // 0..3 each
        if (lane < nh)
          __stcs(dst + lane, mine[off + lane]);
        else if (lane >= 4 && lane < 4 + nt)
          __stcs(dst + (4 * qb - off) + (lane - 4), mine[4 * qb + lane - 4]);
      } else {
        for (int i = lane; i < wcnt; i += 32) __stcs(dst + i, mine[off + i]);
      }
      __syncwarp();  // the next sub-tile's staging overwrites what this warp read
    }
  }
  for (; k < n_items; ++k) {
    const int s = item_sub(k);
    const int64_t t0 = static_cast<int64_t>(s) * kSubTok;
    uint32_t bits = 0;
    if (keep_bits) {
      bits = s_bits[(s - sub0) * kSegThreads + threadIdx.x];
    } else {
      const int st = k % kSegStages;
      sm100::mbar_wait(&full[st], static_cast<uint32_t>((k / kSegStages) & 1), &s_fail, kSegBudget);
      uint32_t w[8];
      seg_words(ring[st], mask, t0, a, item_len(k) & ~15, n_tok, w);
#pragma unroll
      for (int i = 0; i < 8; ++i) bits |= gather4(w[i]) << (4 * i);
    }
    const int cnt = __popc(bits);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    // The warps' counts by sub-tile parity: a warp writes this buffer again two
    // sub-tiles later, past a barrier that every other warp reaches only after
    // reading it here.
    int *ws = warp_sum[k & 1];
    if (lane == 31) ws[warp] = incl;
    __syncthreads();  // stage st consumed by every thread; the warps' counts published
    if (s_fail) break;
    if (threadIdx.x == 0 && issued < n_loads) issue();
    int wofs = 0;
#pragma unroll
    for (int w = 0; w < kSegThreads / 32; ++w) wofs += w < warp ? ws[w] : 0;
    // Each warp stages its own indices and stores them as one contiguous run.
    uint16_t *mine = s_idx + warp * 1024;
    int pos = incl - cnt;
    while (bits) {  // set bits only, lowest first
      mine[pos++] = static_cast<uint16_t>(a + __ffs(bits) - 1);
      bits &= bits - 1;
    }
    __syncwarp();
    const int wcnt = __shfl_sync(0xffffffffu, incl, 31);
    int32_t *dst = idx + excl + s_cnt[s - sub0] + wofs;
    for (int i = lane; i < wcnt; i += 32) __stcs(dst + i, static_cast<int32_t>(t0 + mine[i]));
    __syncwarp();  // the next sub-tile's staging overwrites what this loop read
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (s_fail) {
      // let the copies still in flight land before the CTA's shared memory goes away
      for (int j = k; j < issued; ++j)
        sm100::mbar_drain(&full[j % kSegStages], static_cast<uint32_t>((j / kSegStages) & 1), kSegBudget);
      atomicMin(n_active, -1);
    } else if (c == G - 1) {
      atomicMin(n_active, static_cast<int>(excl) + s_total);
    }
  }
}

// One warp per active row: o_cache[idx[i]] <- o_compact[i].  Rows go to warps
// block-interleaved (row i to block i mod grid) so that a short active list
// still spreads over every SM, and each lane issues up to kScatterU 16-byte
// loads before its stores, so a row of a few KB (24 heads x 128 x bf16 = 384
// vectors) is one round trip rather than one per vector.
constexpr int kScatterU = 12;
__global__ void __launch_bounds__(256) scatter_kernel(const uint4 *__restrict__ src, const int32_t *__restrict__ idx,
                                                      const int32_t *__restrict__ n_active, int n_max,
                                                      int vec_per_row, uint4 *__restrict__ dst) {
  const int n = min(*n_active, n_max);
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  for (int i = blockIdx.x + gridDim.x * (threadIdx.x >> 5); i < n; i += warps) {
    const int64_t r = idx[i];
    const uint4 *s = src + static_cast<int64_t>(i) * vec_per_row;
    uint4 *d = dst + r * vec_per_row;
    for (int c0 = lane; c0 < vec_per_row; c0 += 32 * kScatterU) {
      uint4 v[kScatterU];
#pragma unroll
      for (int u = 0; u < kScatterU; ++u)
        if (c0 + 32 * u < vec_per_row) v[u] = __ldcs(s + c0 + 32 * u);
#pragma unroll
      for (int u = 0; u < kScatterU; ++u)
        if (c0 + 32 * u < vec_per_row) d[c0 + 32 * u] = v[u];
    }
  }
}

}  // namespace cca

using namespace cca;

static cca_status token_mask_impl(const float *src, const float *edit, int32_t n_frames, int32_t n_tok,
                                  int32_t n_ch, float tau, float prune_quantile, uint8_t *mask, float *dist2_out,
                                  float *tau_out, cca_stream_t stream) {
  if (n_frames < 1 || n_frames > 64 || static_cast<int64_t>(n_frames) * n_tok > (int64_t(1) << 31) - 1)
    return fail(CCA_ERR_INVALID_ARG, "cca_token_mask_l2: need 1 <= n_frames <= 64 and n_frames * n_pos < 2^31");
  if (n_tok < 0 || n_ch < 4 || n_ch > 256 || (n_ch & 3))
    return fail(CCA_ERR_INVALID_ARG, "cca_token_mask_l2: need n_tok >= 0 and n_ch a multiple of 4 in [4, 256]");
  if (n_tok > 0 && (!src || !edit || !mask || !aligned16(src) || !aligned16(edit)))
    return fail(CCA_ERR_INVALID_ARG, "cca_token_mask_l2: src/edit/mask must be non-NULL, src/edit 16-byte aligned");
  if ((dist2_out && (reinterpret_cast<uintptr_t>(dist2_out) & 3)) || (tau_out && (reinterpret_cast<uintptr_t>(tau_out) & 3)))
    return fail(CCA_ERR_INVALID_ARG, "cca_token_mask_l2: dist2_out/tau_out must be 4-byte aligned");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (prune_quantile < 0.f) {
    if (!(tau >= 0.f) || !std::isfinite(tau))
      return fail(CCA_ERR_INVALID_ARG, "cca_token_mask_l2: fixed tau must be finite and >= 0");
    if (n_tok == 0) return CCA_OK;
    int blocks = (n_tok + kMaskThreads - 1) / kMaskThreads;
    const int cap = num_sms() * 8;
    if (blocks > cap) blocks = cap;
    mask_fixed_kernel<<<blocks, kMaskThreads, 0, st>>>(src, edit, n_tok, n_ch, tau * tau, mask, dist2_out, tau_out,
                                                       n_frames);
    return launched("mask_fixed_kernel");
  }
  if (!(prune_quantile > 0.f && prune_quantile <= 1.f))
    return fail(CCA_ERR_INVALID_ARG, "cca_token_mask_l2: prune_quantile must be < 0 (fixed tau) or in (0, 1]");
  if (n_tok < 1 || n_tok > kMaxSelectTokens)
    return fail(CCA_ERR_INVALID_ARG, "cca_token_mask_l2: dynamic tau needs 1 <= n_tok <= %d", kMaxSelectTokens);
  // k = ceil(q * N) in binary64, as documented.
  const int k = static_cast<int>(std::ceil(static_cast<double>(prune_quantile) * static_cast<double>(n_tok)));
  const size_t smem = static_cast<size_t>(n_tok) * sizeof(unsigned);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(mask_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kMaxSelectTokens * sizeof(unsigned)));
    if (e != cudaSuccess) return fail(CCA_ERR_CUDA, "cca_token_mask_l2: %s", cudaGetErrorString(e));
  }
  mask_select_kernel<<<1, kSelectThreads, smem, st>>>(src, edit, n_tok, n_ch, k < 1 ? 1 : k, mask, dist2_out,
                                                       tau_out, n_frames);
  return launched("mask_select_kernel");
}

extern "C" {

cca_status cca_token_mask_l2(const float *src, const float *edit, int32_t n_tok, int32_t n_ch, float tau,
                             float prune_quantile, uint8_t *mask, float *dist2_out, float *tau_out,
                             cca_stream_t stream) {
  return token_mask_impl(src, edit, 1, n_tok, n_ch, tau, prune_quantile, mask, dist2_out, tau_out, stream);
}

cca_status cca_token_mask_l2_frames(const float *src, const float *edit, int32_t n_frames, int32_t n_pos,
                                    int32_t n_ch, float tau, float prune_quantile, uint8_t *mask, float *dist2_out,
                                    float *tau_out, cca_stream_t stream) {
  return token_mask_impl(src, edit, n_frames, n_pos, n_ch, tau, prune_quantile, mask, dist2_out, tau_out, stream);
}

static size_t seg_workspace_bytes() { return static_cast<size_t>(kMaxSegCtas) * 8 + 16; }

cca_status cca_compact_workspace_size(int32_t n_tok, size_t *bytes) {
  if (!bytes || n_tok < 0) return fail(CCA_ERR_INVALID_ARG, "cca_compact_workspace_size: bad argument");
  *bytes = n_tok <= kCompactSingleMax ? 0 : seg_workspace_bytes();
  return CCA_OK;
}

// Co-resident CTAs of compact_seg_kernel on the current device (cached per device).
static int seg_max_ctas() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    int per_sm = 0;
    if (cudaFuncSetAttribute(compact_seg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSegDynSmem) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, compact_seg_kernel, kSegThreads, kSegDynSmem) !=
            cudaSuccess)
      return 0;
    cache[dev] = per_sm * num_sms();
  }
  return cache[dev];
}

cca_status cca_compact(const uint8_t *mask, int32_t n_tok, int32_t *idx, int32_t *n_active_dev, void *workspace,
                       size_t workspace_bytes, cca_stream_t stream) {
  if (n_tok < 0 || n_tok > kCompactMaxTokens)
    return fail(CCA_ERR_INVALID_ARG, "cca_compact: need 0 <= n_tok <= %d", kCompactMaxTokens);
  if (!n_active_dev || (n_tok > 0 && (!mask || !idx)))
    return fail(CCA_ERR_INVALID_ARG, "cca_compact: NULL argument");
  if (n_tok > 0 && !aligned16(mask)) return fail(CCA_ERR_INVALID_ARG, "cca_compact: mask must be 16-byte aligned");
  if (n_tok > 0 && (reinterpret_cast<uintptr_t>(idx) & 3u) != 0)
    return fail(CCA_ERR_INVALID_ARG, "cca_compact: idx must be 4-byte aligned");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (n_tok <= kCompactSingleMax) {
    compact_kernel<<<1, kCompactThreads, 0, st>>>(mask, n_tok, idx, n_active_dev);
    return launched("compact_kernel");
  }
  if (!workspace || workspace_bytes < seg_workspace_bytes() || !aligned16(workspace))
    return fail(CCA_ERR_INVALID_ARG, "cca_compact: %d tokens need a 16-byte aligned workspace of %zu bytes", n_tok,
                seg_workspace_bytes());
  const int n_sub = (n_tok + kSubTok - 1) / kSubTok;
  int G = seg_max_ctas();
  if (G <= 0) return fail(CCA_ERR_CUDA, "cca_compact: occupancy query failed");
  if (G > kMaxSegCtas) G = kMaxSegCtas;
  // CCA_COMPACT_CTAS caps the grid (tests use it to give each CTA long runs)
  if (const char *e = std::getenv("CCA_COMPACT_CTAS")) {
    const int cap = std::atoi(e);
    if (cap > 0 && cap < G) G = cap;
  }
  if (G > n_sub) G = n_sub;
  if ((n_sub + G - 1) / G > kMaxSubPerCta)
    return fail(CCA_ERR_INVALID_ARG, "cca_compact: %d tokens exceed %d per CTA", n_tok, kMaxSubPerCta * kSubTok);
  unsigned long long *status = static_cast<unsigned long long *>(workspace);
  seg_init_kernel<<<(G + 255) / 256, 256, 0, st>>>(status, n_active_dev, G);
  CCA_TRY(launched("seg_init_kernel"));
  void *args[] = {const_cast<uint8_t **>(&mask), &n_tok, &idx, &n_active_dev, &status, const_cast<int *>(&n_sub)};
  const cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(compact_seg_kernel), dim3(G),
                                                    dim3(kSegThreads), args, kSegDynSmem, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(CCA_ERR_CUDA, "cca_compact: cooperative launch failed: %s", cudaGetErrorString(e));
  }
  return launched("compact_seg_kernel");
}

cca_status cca_scatter(const void *o_compact, const int32_t *idx, const int32_t *n_active_dev, int32_t n_max,
                       int32_t row_bytes, void *o_cache, cca_stream_t stream) {
  if (n_max < 0 || row_bytes <= 0 || (row_bytes & 15))
    return fail(CCA_ERR_INVALID_ARG, "cca_scatter: need n_max >= 0 and row_bytes a positive multiple of 16");
  if (n_max == 0) return CCA_OK;
  if (!o_compact || !idx || !n_active_dev || !o_cache || !aligned16(o_compact) || !aligned16(o_cache))
    return fail(CCA_ERR_INVALID_ARG, "cca_scatter: NULL or misaligned argument");
  const int vec = row_bytes / 16;
  int blocks = (n_max + 7) / 8;
  const int cap = num_sms() * 8;
  if (blocks > cap) blocks = cap;
  scatter_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4 *>(o_compact), idx, n_active_dev, n_max, vec, static_cast<uint4 *>(o_cache));
  return launched("scatter_kernel");
}

}  // extern "C"
