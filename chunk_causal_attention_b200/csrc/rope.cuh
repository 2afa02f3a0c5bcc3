// Rotary position encoding with a fused 3D + 1D angle, shared by the Q/K path
// and the clean-KV append.
//
// ["JoyAI-Video-Edit 소개", section 세 부품으로 이루어진 아키텍처: the position
// encoding composes each rotation angle from a 3D spatio-temporal RoPE and a 1D
// source RoPE, so that source and generated tokens of one sequence are told
// apart.]  The formula is not on the pages; the reading used: every token has
// integer coordinates (t, h, w, s) -- time, height, width and a source index --
// and pair i of a head, the elements (2i, 2i+1), turns by
//     theta_i = t F[0][i] + h F[1][i] + w F[2][i] + s F[3][i],
// i.e. the 3D rotation and the 1D source rotation in the same plane, whose
// angles add.  F is a caller-supplied [4][D/2] table (cca_mrope_freqs builds
// the sectioned default).
#pragma once

#include <cstdint>

#include "common.cuh"

namespace cca {

struct RopeArgs {
  const int32_t *pos;  // [n_tok][4] (t, h, w, s); NULL: no rotation
  const float *freq;   // [4][D/2]
};

// Rotates the 8 elements x[0..7] = elements d0 .. d0+7 (d0 a multiple of 8) of
// token tok: pairs d0/2 .. d0/2 + 3.
__device__ __forceinline__ void rope8(const RopeArgs &r, int64_t tok, int d0, int D, float (&x)[8]) {
  const int4 p = __ldg(reinterpret_cast<const int4 *>(r.pos) + tok);
  const float pt = static_cast<float>(p.x), ph = static_cast<float>(p.y), pw = static_cast<float>(p.z),
              ps = static_cast<float>(p.w);
  const int P = D / 2;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int i = d0 / 2 + j;
    const float th = fmaf(ps, __ldg(r.freq + 3 * P + i),
                          fmaf(pw, __ldg(r.freq + 2 * P + i), fmaf(ph, __ldg(r.freq + P + i), pt * __ldg(r.freq + i))));
    float sn, cs;
    sincosf(th, &sn, &cs);
    const float a = x[2 * j], b = x[2 * j + 1];
    x[2 * j] = fmaf(a, cs, -b * sn);
    x[2 * j + 1] = fmaf(a, sn, b * cs);
  }
}

// Rotate (rot0 / rot1) or copy two [n_tok][H][D] tensors (bf16 or fp32 input)
// into bf16 outputs in one launch; x1 may be NULL.  Defined in rope.cu.
cca_status launch_rope_rows(const void *x0, const void *x1, void *y0, void *y1, bool rot0, bool rot1, bool f32,
                            RopeArgs r, int n_tok, int H, int D, cudaStream_t st);

}  // namespace cca
