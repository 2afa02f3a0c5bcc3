// Fused 3D + 1D rotary position encoding of the current chunk's Q and K
// (sm_100a).  The rotation and its reading of the pages are described in
// rope.cuh; the clean-KV append applies the same rotation to K as it stores it
// (ring.cu).
//
// HBM-bound: per element one read (bf16 or fp32) and one bf16 write.  Both
// tensors go through one launch (blockIdx.y picks Q or K); every thread keeps
// kRopeUnroll 16-byte vectors of loads in flight and the grid is one wave.
#include <cuda_bf16.h>

#include <cmath>

#include "common.cuh"
#include "rope.cuh"

namespace cca {

constexpr int kRopeUnroll = 4;

template <bool kF32>
__device__ __forceinline__ void load8f(const void *base, int64_t elem, float (&x)[8]) {
  if constexpr (kF32) {
    const float4 a = __ldcs(reinterpret_cast<const float4 *>(static_cast<const float *>(base) + elem));
    const float4 b = __ldcs(reinterpret_cast<const float4 *>(static_cast<const float *>(base) + elem + 4));
    x[0] = a.x, x[1] = a.y, x[2] = a.z, x[3] = a.w, x[4] = b.x, x[5] = b.y, x[6] = b.z, x[7] = b.w;
  } else {
    const uint4 u = __ldcs(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(base) + elem));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      x[2 * j] = __uint_as_float(w[j] << 16);
      x[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
  }
}

__device__ __forceinline__ uint4 pack8_bf16(const float (&x)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(x[2 * j], x[2 * j + 1]);
    w[j] = *reinterpret_cast<const uint32_t *>(&p);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// y = rope(x) for tensor blockIdx.y (0: q, 1: k), both [n_tok][H][D].
template <bool kF32>
__global__ void __launch_bounds__(256) rope_qk_kernel(const void *__restrict__ q, const void *__restrict__ k,
                                                      uint4 *__restrict__ q_out, uint4 *__restrict__ k_out,
                                                      RopeArgs r, int H, int D, int64_t n_vec) {
  const void *x = blockIdx.y == 0 ? q : k;
  uint4 *y = blockIdx.y == 0 ? q_out : k_out;
  if (!x) return;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int vec_per_tok = H * D / 8;
  for (int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i0 < n_vec;
       i0 += kRopeUnroll * stride) {
    float v[kRopeUnroll][8];
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      const int64_t i = i0 + u * stride;
      if (i < n_vec) load8f<kF32>(x, i * 8, v[u]);
    }
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      const int64_t i = i0 + u * stride;
      if (i < n_vec) {
        const int64_t tok = i / vec_per_tok;
        const int d0 = static_cast<int>((i * 8) % D);
        rope8(r, tok, d0, D, v[u]);
        y[i] = pack8_bf16(v[u]);
      }
    }
  }
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
  const int64_t n_vec = static_cast<int64_t>(n_tok) * n_heads * head_dim / 8;
  int64_t blocks = (n_vec + 256 * kRopeUnroll - 1) / (256 * kRopeUnroll);
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  const dim3 grid(static_cast<unsigned>(blocks), 2);
  const RopeArgs r{pos, freq};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (src_dtype == CCA_F32)
    rope_qk_kernel<true><<<grid, 256, 0, st>>>(q, k, static_cast<uint4 *>(q_out), static_cast<uint4 *>(k_out), r,
                                                n_heads, head_dim, n_vec);
  else
    rope_qk_kernel<false><<<grid, 256, 0, st>>>(q, k, static_cast<uint4 *>(q_out), static_cast<uint4 *>(k_out), r,
                                                 n_heads, head_dim, n_vec);
  return launched("rope_qk_kernel");
}

}  // extern "C"
