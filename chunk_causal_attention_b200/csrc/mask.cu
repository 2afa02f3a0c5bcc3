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

#include "common.cuh"

namespace cca {

constexpr int kMaskThreads = 256;
constexpr int kSelectThreads = 1024;
constexpr int kMaxSelectTokens = 32768;

__device__ __forceinline__ float token_dist2(const float *__restrict__ src, const float *__restrict__ edit,
                                             int64_t u, int n_ch) {
  const float4 *s = reinterpret_cast<const float4 *>(src + u * n_ch);
  const float4 *e = reinterpret_cast<const float4 *>(edit + u * n_ch);
  float acc = 0.f;
  for (int c = 0; c < n_ch / 4; ++c) {
    const float4 a = __ldg(s + c), b = __ldg(e + c);
    const float d0 = b.x - a.x, d1 = b.y - a.y, d2 = b.z - a.z, d3 = b.w - a.w;
    acc = fmaf(d0, d0, acc);
    acc = fmaf(d1, d1, acc);
    acc = fmaf(d2, d2, acc);
    acc = fmaf(d3, d3, acc);
  }
  return acc;
}

// Fixed threshold: one thread per token, grid-stride.
__global__ void __launch_bounds__(kMaskThreads) mask_fixed_kernel(const float *__restrict__ src,
                                                                  const float *__restrict__ edit, int n_tok,
                                                                  int n_ch, float tau2, uint8_t *__restrict__ mask,
                                                                  float *__restrict__ dist2, float *tau_out) {
  const int stride = gridDim.x * blockDim.x;
  for (int u = blockIdx.x * blockDim.x + threadIdx.x; u < n_tok; u += stride) {
    const float d2 = token_dist2(src, edit, u, n_ch);
    mask[u] = d2 > tau2 ? 1 : 0;
    if (dist2) dist2[u] = d2;
  }
  if (tau_out && blockIdx.x == 0 && threadIdx.x == 0) *tau_out = sqrtf(tau2);
}

// Dynamic threshold, one CTA: d^2 of every token into shared memory, radix
// select of the k-th smallest (k >= 1), then mask = d^2 > that value.
__global__ void __launch_bounds__(kSelectThreads) mask_select_kernel(const float *__restrict__ src,
                                                                     const float *__restrict__ edit, int n_tok,
                                                                     int n_ch, int k, uint8_t *__restrict__ mask,
                                                                     float *__restrict__ dist2, float *tau_out) {
  extern __shared__ unsigned s_bits[];  // n_tok entries
  __shared__ unsigned hist[256];
  __shared__ unsigned s_prefix, s_rank;
  for (int u = threadIdx.x; u < n_tok; u += blockDim.x) {
    const float d2 = token_dist2(src, edit, u, n_ch);
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
    if (threadIdx.x == 0) {  // 256-bin scan by one thread: negligible next to the loads
      unsigned rank = s_rank, cum = 0u;
      int bin = 0;
      for (; bin < 256; ++bin) {
        if (cum + hist[bin] >= rank) break;
        cum += hist[bin];
      }
      s_rank = rank - cum;
      s_prefix = prefix | (static_cast<unsigned>(bin) << shift);
    }
    __syncthreads();
  }
  const float tau2 = __uint_as_float(s_prefix);
  for (int u = threadIdx.x; u < n_tok; u += blockDim.x) mask[u] = __uint_as_float(s_bits[u]) > tau2 ? 1 : 0;
  if (tau_out && threadIdx.x == 0) *tau_out = sqrtf(tau2);
}

// Ordered stream compaction in one CTA: tiles of blockDim.x * 16 mask bytes,
// block-wide exclusive scan of per-thread counts, running offset across tiles.
constexpr int kCompactThreads = 1024;
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
    uint8_t m[16];
    if (u0 + 16 <= n_tok) {
      const uint4 v = *reinterpret_cast<const uint4 *>(mask + u0);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 16; ++j) m[j] = static_cast<uint8_t>((w[j >> 2] >> (8 * (j & 3))) & 0xffu);
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) m[j] = (u0 + j < n_tok) ? mask[u0 + j] : 0;
    }
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) cnt += m[j] != 0;
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
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (m[j]) idx[pos++] = u0 + j;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) s_base = pos;
    __syncthreads();
  }
  if (threadIdx.x == 0) *n_active = s_base;
}

// One warp per active row: o_cache[idx[i]] <- o_compact[i].
__global__ void __launch_bounds__(256) scatter_kernel(const uint4 *__restrict__ src, const int32_t *__restrict__ idx,
                                                      const int32_t *__restrict__ n_active, int n_max,
                                                      int vec_per_row, uint4 *__restrict__ dst) {
  const int n = min(*n_active, n_max);
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < n; i += warps) {
    const int64_t r = idx[i];
    const uint4 *s = src + static_cast<int64_t>(i) * vec_per_row;
    uint4 *d = dst + r * vec_per_row;
    for (int c = lane; c < vec_per_row; c += 32) d[c] = __ldcs(s + c);
  }
}

}  // namespace cca

using namespace cca;

extern "C" {

cca_status cca_token_mask_l2(const float *src, const float *edit, int32_t n_tok, int32_t n_ch, float tau,
                             float prune_quantile, uint8_t *mask, float *dist2_out, float *tau_out,
                             cca_stream_t stream) {
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
    mask_fixed_kernel<<<blocks, kMaskThreads, 0, st>>>(src, edit, n_tok, n_ch, tau * tau, mask, dist2_out, tau_out);
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
                                                       tau_out);
  return launched("mask_select_kernel");
}

cca_status cca_compact(const uint8_t *mask, int32_t n_tok, int32_t *idx, int32_t *n_active_dev,
                       cca_stream_t stream) {
  if (n_tok < 0 || n_tok > (1 << 20)) return fail(CCA_ERR_INVALID_ARG, "cca_compact: need 0 <= n_tok <= 2^20");
  if (!n_active_dev || (n_tok > 0 && (!mask || !idx)))
    return fail(CCA_ERR_INVALID_ARG, "cca_compact: NULL argument");
  if (n_tok > 0 && !aligned16(mask)) return fail(CCA_ERR_INVALID_ARG, "cca_compact: mask must be 16-byte aligned");
  compact_kernel<<<1, kCompactThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(mask, n_tok, idx, n_active_dev);
  return launched("compact_kernel");
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
