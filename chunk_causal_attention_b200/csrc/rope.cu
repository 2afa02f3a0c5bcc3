// Fused 3D + 1D rotary position encoding of the current chunk's Q and K
// (sm_100a).  The rotation and its reading of the pages are described in
// rope.cuh; the clean-KV append applies the same rotation to K as it stores it
// (ring.cu).
//
// HBM-bound: per element one read (bf16 or fp32) and one bf16 write.  Both
// tensors go through one launch; the angles of a token are computed once and
// shared by all of its heads.
#include <cuda_bf16.h>

#include <cmath>

#include "common.cuh"
#include "rope.cuh"

namespace cca {

__device__ __forceinline__ uint4 pack8_bf16(const float (&x)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(x[2 * j], x[2 * j + 1]);
    w[j] = *reinterpret_cast<const uint32_t *>(&p);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// A block takes kRopeTok tokens at a time (810 blocks at 1620 tokens, so that
// several blocks' loads are in flight on every SM): it first fills a shared
// table of (cos, sin) for their D/2 planes -- one sincosf per token and plane,
// shared by all heads (an accurate sincosf costs on the order of a hundred
// instructions, so computing it per element made the rotation compute-bound)
// -- then streams the 16-byte vectors of those tokens of both tensors as one
// index range, kRopeU raw loads in flight per thread before any is converted,
// rotated (or only copied) and stored as bf16.  x1 == nullptr: one tensor.
constexpr int kRopeTok = 2;
constexpr int kRopeU = 8;
constexpr int kRopeThreads = 256;

template <bool kF32, int D>
__global__ void __launch_bounds__(kRopeThreads) rope_rows_kernel(const void *__restrict__ x0,
                                                                 const void *__restrict__ x1, uint4 *__restrict__ y0,
                                                                 uint4 *__restrict__ y1, int rot0, int rot1,
                                                                 RopeArgs r, int H, int n_tok) {
  constexpr int P = D / 2;
  constexpr int kVpd = D / 8;  // vectors per head row
  __shared__ float2 cs[kRopeTok][P];
  const int vpt = H * kVpd;  // vectors per token
  for (int t0 = blockIdx.x * kRopeTok; t0 < n_tok; t0 += gridDim.x * kRopeTok) {
    const int nt = min(kRopeTok, n_tok - t0);
    __syncthreads();  // the previous tokens' table is no longer read
    const int nv = nt * vpt;
    const int n_all = x1 ? 2 * nv : nv;
    const int64_t v0 = static_cast<int64_t>(t0) * vpt;
    // The first batch of loads is issued before the table is computed, so the
    // sincosf work overlaps their latency; every thread runs the first batch.
    int b = threadIdx.x;
    bool first = true;
    do {
      uint4 raw[kRopeU][kF32 ? 2 : 1];
#pragma unroll
      for (int u = 0; u < kRopeU; ++u) {
        const int c = b + u * kRopeThreads;
        if (c < n_all) {
          const bool second = c >= nv;
          const void *x = second ? x1 : x0;
          const int64_t e = v0 + (second ? c - nv : c);
          if constexpr (kF32) {
            raw[u][0] = __ldcs(reinterpret_cast<const uint4 *>(x) + 2 * e);
            raw[u][1] = __ldcs(reinterpret_cast<const uint4 *>(x) + 2 * e + 1);
          } else {
            raw[u][0] = __ldcs(reinterpret_cast<const uint4 *>(x) + e);
          }
        }
      }
      if (first) {
        first = false;
        if (rot0 | rot1) {
          for (int e = threadIdx.x; e < nt * P; e += kRopeThreads) {
            const int tt = e / P, i = e - tt * P;
            const int4 p = __ldg(reinterpret_cast<const int4 *>(r.pos) + t0 + tt);
            const float th = fmaf(static_cast<float>(p.w), __ldg(r.freq + 3 * P + i),
                                  fmaf(static_cast<float>(p.z), __ldg(r.freq + 2 * P + i),
                                       fmaf(static_cast<float>(p.y), __ldg(r.freq + P + i),
                                            static_cast<float>(p.x) * __ldg(r.freq + i))));
            float sn, cn;
            sincosf(th, &sn, &cn);
            cs[tt][i] = make_float2(cn, sn);
          }
        }
        __syncthreads();
      }
#pragma unroll
      for (int u = 0; u < kRopeU; ++u) {
        const int c = b + u * kRopeThreads;
        if (c >= n_all) continue;
        const bool second = c >= nv;
        const int i = second ? c - nv : c;
        uint4 *y = second ? y1 : y0;
        const bool rot = (second ? rot1 : rot0) != 0;
        {
          float v[8];
          if constexpr (kF32) {
            const uint32_t w[8] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w,
                                   raw[u][1].x, raw[u][1].y, raw[u][1].z, raw[u][1].w};
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(w[j]);
          } else {
            const uint32_t w[4] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              v[2 * j] = __uint_as_float(w[j] << 16);
              v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
            }
          }
          if (rot) {
            int tt = 0;
#pragma unroll
            for (int k = 1; k < kRopeTok; ++k) tt += i >= k * vpt;
            const int pl = (i % kVpd) * 4;  // first of the vector's 4 planes
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 cw = cs[tt][pl + j];
              const float a = v[2 * j], bb = v[2 * j + 1];
              v[2 * j] = fmaf(a, cw.x, -bb * cw.y);
              v[2 * j + 1] = fmaf(a, cw.y, bb * cw.x);
            }
          }
          y[v0 + i] = pack8_bf16(v);
        }
      }
      b += kRopeU * kRopeThreads;
    } while (b < n_all);
  }
}

// Launcher shared with the clean-KV append (ring.cu).
cca_status launch_rope_rows(const void *x0, const void *x1, void *y0, void *y1, bool rot0, bool rot1, bool f32,
                            RopeArgs r, int n_tok, int H, int D, cudaStream_t st) {
  if (n_tok == 0) return CCA_OK;
  if (2 * static_cast<int64_t>(kRopeTok) * H * D / 8 >= (int64_t(1) << 31))
    return fail(CCA_ERR_INVALID_ARG, "rotary encoding: H * D too large");
  if (!x0) {  // only the second tensor given: run it as the first
    x0 = x1, y0 = y1, rot0 = rot1;
    x1 = nullptr, y1 = nullptr;
  }
  int blocks = (n_tok + kRopeTok - 1) / kRopeTok;
  const int cap = num_sms() * 8;
  if (blocks > cap) blocks = cap;
  uint4 *a = static_cast<uint4 *>(y0), *b = static_cast<uint4 *>(y1);
  const int r0 = rot0, r1 = rot1;
  if (f32) {
    if (D == 128) rope_rows_kernel<true, 128><<<blocks, kRopeThreads, 0, st>>>(x0, x1, a, b, r0, r1, r, H, n_tok);
    else rope_rows_kernel<true, 64><<<blocks, kRopeThreads, 0, st>>>(x0, x1, a, b, r0, r1, r, H, n_tok);
  } else {
    if (D == 128) rope_rows_kernel<false, 128><<<blocks, kRopeThreads, 0, st>>>(x0, x1, a, b, r0, r1, r, H, n_tok);
    else rope_rows_kernel<false, 64><<<blocks, kRopeThreads, 0, st>>>(x0, x1, a, b, r0, r1, r, H, n_tok);
  }
  return launched("rope_rows_kernel");
}

}  // namespace cca

using namespace cca;

extern "C" {

cca_status cca_mrope_freqs(int32_t head_dim, int32_t sec_t, int32_t sec_h, int32_t sec_w, float base,
                           float *freq) {
  if (!freq || (head_dim != 64 && head_dim != 128) || sec_t < 0 || sec_h < 0 || sec_w < 0 ||
      sec_t + sec_h + sec_w != head_dim / 2 || !(base > 1.f))
    return fail(CCA_ERR_INVALID_ARG,
                "cca_mrope_freqs: need D in {64,128}, sections >= 0 summing to D/2, base > 1");
  const int P = head_dim / 2;
  const int sec[3] = {sec_t, sec_h, sec_w};
  for (int a = 0; a < 4 * P; ++a) freq[a] = 0.f;
  int i0 = 0;
  for (int a = 0; a < 3; ++a) {  // coordinate a turns the pairs of its section, geometric frequencies
    for (int j = 0; j < sec[a]; ++j)
      freq[a * P + i0 + j] = static_cast<float>(std::pow(static_cast<double>(base), -static_cast<double>(j) / sec[a]));
    i0 += sec[a];
  }
  for (int i = 0; i < P; ++i)  // the 1D source rotation turns every pair
    freq[3 * P + i] = static_cast<float>(std::pow(static_cast<double>(base), -2.0 * i / head_dim));
  return CCA_OK;
}

cca_status cca_rope_qk(const void *q, const void *k, cca_dtype src_dtype, int32_t n_tok, int32_t n_heads,
                       int32_t head_dim, const int32_t *pos, const float *freq, void *q_out, void *k_out,
                       cca_stream_t stream) {
  if (n_tok < 0 || n_heads < 1 || (head_dim != 64 && head_dim != 128) ||
      (src_dtype != CCA_BF16 && src_dtype != CCA_F32))
    return fail(CCA_ERR_INVALID_ARG, "cca_rope_qk: need n_tok >= 0, H >= 1, D in {64,128}, BF16 or F32 input");
  if (n_tok == 0 || (!q && !k)) return CCA_OK;
  if (!pos || !freq || (q && !q_out) || (k && !k_out))
    return fail(CCA_ERR_INVALID_ARG, "cca_rope_qk: pos, freq and the outputs of the given inputs are required");
  if ((q && (!aligned16(q) || !aligned16(q_out))) || (k && (!aligned16(k) || !aligned16(k_out))) ||
      !aligned16(pos) || (reinterpret_cast<uintptr_t>(freq) & 3))
    return fail(CCA_ERR_INVALID_ARG, "cca_rope_qk: tensors and pos must be 16-byte aligned, freq 4-byte aligned");
  return launch_rope_rows(q, k, q_out, k_out, q != nullptr, k != nullptr, src_dtype == CCA_F32,
                          RopeArgs{pos, freq}, n_tok, n_heads, head_dim, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
