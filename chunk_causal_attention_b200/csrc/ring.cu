// Bounded KV cache: ring handle, slot arithmetic, clean-KV append (+ e4m3
// quantisation), and the stand-alone e4m3 quantiser.
//
// The cache keeps the first chunk forever (global sink) plus the W most recent
// chunks, evicting the oldest non-sink chunk ["JoyAI-Video-Edit 소개", section
// 30 FPS를 만드는 실시간 배포 파이프라인; "論文解説: JoyAI-Video-Edit", §5 loop].
// Layout choice of this library: slot 0 = chunk 0, chunk t >= 1 -> slot
// 1 + (t-1) mod W, so an append overwrites exactly the evicted chunk and no data
// ever moves.
#include <cuda_fp8.h>
#include <cuda_bf16.h>

#include <cmath>
#include <mutex>
#include <new>
#include <vector>

#include "common.cuh"
#include "ring.cuh"
#include "rope.cuh"
#include "sm100.cuh"

namespace cca {

std::string &last_error() {
  static thread_local std::string s;
  return s;
}
int64_t &launch_counter() {
  static thread_local int64_t n = 0;
  return n;
}

int num_sms() {
  static std::mutex mu;
  static std::vector<int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  if (dev >= static_cast<int>(cache.size())) cache.resize(dev + 1, 0);
  if (cache[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

int ring_slot_of(const cca_kv_ring *r, int64_t chunk) {
  if (chunk == 0) return 0;
  return 1 + static_cast<int>((chunk - 1) % r->d.window);
}

int ring_visible(const cca_kv_ring *r, int32_t *slots, int64_t *chunk_ids) {
  // Cached chunks visible from the current chunk t = n_appended, logical order.
  const int64_t t = r->n_appended;
  int n = 0;
  if (t == 0) return 0;
  if (slots) slots[n] = 0;
  if (chunk_ids) chunk_ids[n] = 0;
  ++n;
  const int64_t lo = t - r->d.window > 1 ? t - r->d.window : 1;
  for (int64_t c = lo; c < t; ++c) {
    if (slots) slots[n] = ring_slot_of(r, c);
    if (chunk_ids) chunk_ids[n] = c;
    ++n;
  }
  return n;
}

size_t dtype_bytes(cca_dtype t) { return t == CCA_E4M3 ? 1 : (t == CCA_BF16 ? 2 : 4); }

// ------------------------------------------------------------------ kernels
// bf16 (or fp32 -> bf16 RNE) copy of K and V into one ring slot; 16-byte
// vectors, blockIdx.y selects K (0) or V (1).  Each thread keeps 4 independent
// loads in flight before its stores (streaming loads: the source is read once).
__device__ __forceinline__ uint4 to_bf16x8(float4 a, float4 b) {
  __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y), p1 = __floats2bfloat162_rn(a.z, a.w);
  __nv_bfloat162 p2 = __floats2bfloat162_rn(b.x, b.y), p3 = __floats2bfloat162_rn(b.z, b.w);
  uint4 o;
  o.x = *reinterpret_cast<uint32_t *>(&p0);
  o.y = *reinterpret_cast<uint32_t *>(&p1);
  o.z = *reinterpret_cast<uint32_t *>(&p2);
  o.w = *reinterpret_cast<uint32_t *>(&p3);
  return o;
}

// Each thread keeps kAppendUnroll 16-byte outputs' worth of loads in flight and
// the grid is at most one wave (4 blocks of 256 per SM at 64 registers), so a
// 720p chunk (2 x 9.95 MB, 486 blocks) is copied in a single round of loads.
constexpr int kAppendUnroll = 10;
constexpr int64_t kMaxChunkElems = int64_t(1) << 33;  // keeps 16-byte vector indices below 2^30
constexpr int kAppendUnrollF32 = 4;  // fp32 sources: two 16-byte loads per output

template <bool kF32>
__global__ void __launch_bounds__(256, 4) append_bf16_kernel(const void *__restrict__ k_src,
                                                             const void *__restrict__ v_src,
                                                             uint4 *__restrict__ k_dst,
                                                             uint4 *__restrict__ v_dst, int n_vec) {
  constexpr int kU = kF32 ? kAppendUnrollF32 : kAppendUnroll;
  const void *src = blockIdx.y == 0 ? k_src : v_src;
  uint4 *dst = blockIdx.y == 0 ? k_dst : v_dst;
  const int stride = gridDim.x * blockDim.x;  // n_vec < 2^31 is checked on the host
  for (int i0 = blockIdx.x * blockDim.x + threadIdx.x; i0 < n_vec; i0 += kU * stride) {
    uint4 v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const unsigned i = static_cast<unsigned>(i0) + static_cast<unsigned>(u * stride);
      if (i < static_cast<unsigned>(n_vec)) {
        if constexpr (!kF32) {
          v[u] = __ldcs(reinterpret_cast<const uint4 *>(src) + i);
        } else {
          v[u] = to_bf16x8(__ldcs(reinterpret_cast<const float4 *>(src) + 2 * static_cast<size_t>(i)),
                           __ldcs(reinterpret_cast<const float4 *>(src) + 2 * static_cast<size_t>(i) + 1));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const unsigned i = static_cast<unsigned>(i0) + static_cast<unsigned>(u * stride);
      if (i < static_cast<unsigned>(n_vec)) dst[i] = v[u];
    }
  }
}

// BF16 -> BF16 append as a TMA bulk copy: one CTA per SM, one thread issuing
// 16 KB global->shared bulk loads (completion on an mbarrier) and shared->global
// bulk stores from a 12-stage ring of shared memory (192 KB).  A 720p chunk is
// 2 x 9.95 MB = 1215 pieces, about 8 per CTA, so every load is in flight at
// once.  A stage is refilled once the store that read it has finished reading
// (bulk_group accounting, kBulkLag stores may still be reading).  Waits are
// bounded: on expiry the ring's status word gets CCA_DEV_TIMEOUT, the CTA waits
// (bounded) for the loads it issued and for its stores, and returns.
constexpr int kBulkPiece = 16384;
__host__ __device__ inline int64_t cca_min64(int64_t a, int64_t b) { return a < b ? a : b; }
constexpr int kBulkStages = 12;
constexpr int kBulkLag = 4;
constexpr long long kBulkBudget = 2000000000LL;  // clock64 cycles, about 1 s

__global__ void __launch_bounds__(32, 1) append_bulk_kernel(const uint8_t *__restrict__ k_src,
                                                           const uint8_t *__restrict__ v_src, uint8_t *k_dst,
                                                           uint8_t *v_dst, int64_t bytes, int32_t *dev_status) {
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ uint64_t bar[kBulkStages];
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  const int64_t per_tensor = (bytes + kBulkPiece - 1) / kBulkPiece;
  const int64_t n_pieces = 2 * per_tensor;
  const int64_t n_mine = (n_pieces - blockIdx.x + gridDim.x - 1) / gridDim.x;  // pieces c, c + G, ...
  for (int s = 0; s < kBulkStages; ++s) sm100::mbar_init(&bar[s], 1);
  abort_flag = 0;
  sm100::fence_mbar_init();
  const uint32_t base = smem_u32(stage_mem);
  auto piece = [&](int64_t i, const uint8_t *&src, uint8_t *&dst, uint32_t &len) {
    const int64_t j = blockIdx.x + i * gridDim.x;
    const bool v = j >= per_tensor;
    const int64_t off = (v ? j - per_tensor : j) * kBulkPiece;
    src = (v ? v_src : k_src) + off;
    dst = (v ? v_dst : k_dst) + off;
    len = static_cast<uint32_t>(cca_min64(kBulkPiece, bytes - off));
  };
  auto issue_load = [&](int64_t i) {
    const uint8_t *src;
    uint8_t *dst;
    uint32_t len;
    piece(i, src, dst, len);
    const int s = static_cast<int>(i % kBulkStages);
    sm100::mbar_arrive_expect_tx(&bar[s], len);
    sm100::bulk_load(base + s * kBulkPiece, src, len, &bar[s]);
  };
  int64_t issued = 0, done = 0;
  for (; issued < n_mine && issued < kBulkStages; ++issued) issue_load(issued);
  bool ok = true;
  for (int64_t i = 0; i < n_mine; ++i) {
    const int s = static_cast<int>(i % kBulkStages);
    if (!sm100::mbar_wait(&bar[s], static_cast<uint32_t>((i / kBulkStages) & 1), &abort_flag, kBulkBudget)) {
      ok = false;
      break;
    }
    done = i + 1;
    const uint8_t *src;
    uint8_t *dst;
    uint32_t len;
    piece(i, src, dst, len);
    sm100::bulk_store(dst, base + s * kBulkPiece, len);
    sm100::bulk_commit();
    const int64_t r = i + 1 - kBulkLag;  // its store has finished reading after the wait below
    if (r >= 0 && r + kBulkStages < n_mine) {
      asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(kBulkLag - 1) : "memory");
      issue_load(issued++);
    }
  }
  if (!ok) {
    for (int64_t i = done; i < issued; ++i)
      sm100::mbar_drain(&bar[i % kBulkStages], static_cast<uint32_t>((i / kBulkStages) & 1), kBulkBudget);
    if (dev_status) *dev_status = CCA_DEV_TIMEOUT;
  }
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Single-launch per-head quantisation: a cluster of kQC CTAs per (tensor,
// head), each over an eighth of the tokens.  Pass 1: the CTA's absmax (warp
// shuffles, then shared memory); the cluster's maximum is read from the other
// CTAs' shared memory after a hardware cluster barrier.  Pass 2: the CTA
// quantises its rows with s = absmax / 448 (1 for an all-zero head) and codes
// e4m3_rn_satfinite(x / s), both IEEE fp32 divisions.  Rank 0 writes the scale.  A second
// cluster barrier keeps every CTA's shared memory alive until the others have
// read it.  Two kernels share this structure:
//   quant_cpa_kernel: every thread copies its vectors into shared memory with
//     cp.async, all in flight at once, so the tensor is read from HBM once
//     (up to 64 KB of rows per CTA: 2048 tokens of a 128-wide bf16 head);
//   quant_cluster_kernel: larger heads are streamed twice from global memory
//     (pass 2 mostly from L2), kQU loads in flight per thread.
constexpr int kQC = 8;          // CTAs per (tensor, head): a portable cluster
constexpr int kQThreads = 256;

// 8 elements (16 bytes of bf16, or 2 x 16 bytes of fp32) -> fp32, optionally rotated.
template <bool kF32>
__device__ __forceinline__ void q_unpack(const uint4 *w, float (&v)[8]) {
  if constexpr (kF32) {
    const uint32_t u[8] = {w[0].x, w[0].y, w[0].z, w[0].w, w[1].x, w[1].y, w[1].z, w[1].w};
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(u[j]);
  } else {
    const uint32_t u[4] = {w[0].x, w[0].y, w[0].z, w[0].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = __uint_as_float(u[j] << 16);
      v[2 * j + 1] = __uint_as_float(u[j] & 0xffff0000u);
    }
  }
}

// Codes of 8 elements at element offset e of y: e4m3 bytes, or (wide) their values as fp16.
__device__ __forceinline__ void q_store8(void *y, int64_t e, const float (&v)[8], float s, bool wide) {
  uint32_t w[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(v[4 * j], s), __fdiv_rn(v[4 * j + 1], s)), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(v[4 * j + 2], s), __fdiv_rn(v[4 * j + 3], s)), __NV_SATFINITE, __NV_E4M3);
    w[j] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
  }
  if (!wide) {
    *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(y) + e) = make_uint2(w[0], w[1]);
  } else {
    uint32_t hw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half2_raw p2 = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>((w[j >> 1] >> (16 * (j & 1))) & 0xffffu), __NV_E4M3);
      hw[j] = static_cast<uint32_t>(p2.x) | (static_cast<uint32_t>(p2.y) << 16);
    }
    *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(y) + e) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  }
}

// The cluster-wide absmax: CTA maximum m (every thread's partial), then the
// maximum over the cluster's CTAs through distributed shared memory.  Ends
// with the second cluster barrier, after which the shared words may be reused.
__device__ __forceinline__ float q_cluster_max(float m, float *red, float *cta_max) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kQThreads / 32; ++w) m = fmaxf(m, red[w]);
    *cta_max = m;
  }
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  float a = 0.f;
  for (int r = 0; r < kQC; ++r) {
    uint32_t local = smem_u32(cta_max), remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(r));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    a = fmaxf(a, v);
  }
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  return a;
}

struct QuantArgs {  // up to three tensors of one shape, blockIdx.z selects one
  const void *x[3];
  void *y[3];
  float *scale[3];
  int wide[3];
  RopeArgs rope0;  // rotation of tensor 0 before quantising (pos == nullptr: none)
  int n_tok, H, n_tensors;
};

// 16-byte word(s) of the 8 elements of vector i (row t0 + i / vpr, column i % vpr) of head h.
template <bool kF32, int D>
__device__ __forceinline__ void q_fetch(const void *x, int H, int h, int t0, int i, uint4 *w) {
  constexpr int vpr = D / 8;
  const int64_t e = (static_cast<int64_t>(t0 + i / vpr) * H + h) * D + (i % vpr) * 8;
  if constexpr (kF32) {
    w[0] = __ldg(reinterpret_cast<const uint4 *>(static_cast<const float *>(x) + e));
    w[1] = __ldg(reinterpret_cast<const uint4 *>(static_cast<const float *>(x) + e) + 1);
  } else {
    w[0] = __ldg(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(x) + e));
  }
}

// Shared-memory form: every thread copies its vectors into shared memory
// with cp.async (all in flight at once, no registers held), then both passes
// read shared memory.
template <bool kF32, int D>
__global__ void __cluster_dims__(kQC, 1, 1) __launch_bounds__(kQThreads)
    quant_cpa_kernel(const __grid_constant__ QuantArgs q) {
  extern __shared__ __align__(16) uint4 rows16[];
  __shared__ float red[kQThreads / 32];
  __shared__ float cta_max;
  const int tensor = blockIdx.z, h = blockIdx.y, rank = blockIdx.x;
  const bool rot = tensor == 0 && q.rope0.pos != nullptr;
  constexpr int kW = kF32 ? 2 : 1;
  constexpr int vpr = D / 8;
  const int t0 = static_cast<int>(static_cast<int64_t>(q.n_tok) * rank / kQC);
  const int t1 = static_cast<int>(static_cast<int64_t>(q.n_tok) * (rank + 1) / kQC);
  const int n_vec = (t1 - t0) * vpr;
  const uint4 *x = static_cast<const uint4 *>(q.x[tensor]);
  for (int i = threadIdx.x; i < n_vec; i += kQThreads) {
    const int64_t e = ((static_cast<int64_t>(t0 + i / vpr) * q.H + h) * D + (i % vpr) * 8) / (8 / kW);
#pragma unroll
    for (int k = 0; k < kW; ++k)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(rows16 + i * kW + k)),
                   "l"(x + e + k)
                   : "memory");
  }
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  float m = 0.f;
  for (int i = threadIdx.x; i < n_vec; i += kQThreads) {  // a thread reads back only what it copied
    float v[8];
    q_unpack<kF32>(rows16 + i * kW, v);
    if (rot) rope8(q.rope0, t0 + i / vpr, (i % vpr) * 8, D, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
  }
  const float a = q_cluster_max(m, red, &cta_max);
  const float s = a > 0.f ? __fdiv_rn(a, 448.f) : 1.f;
  if (rank == 0 && threadIdx.x == 0) q.scale[tensor][h] = s;
  const bool wide = q.wide[tensor] != 0;
  for (int i = threadIdx.x; i < n_vec; i += kQThreads) {
    float v[8];
    q_unpack<kF32>(rows16 + i * kW, v);
    const int l = t0 + i / vpr, c = i % vpr;
    if (rot) rope8(q.rope0, l, c * 8, D, v);
    q_store8(q.y[tensor], (static_cast<int64_t>(l) * q.H + h) * D + c * 8, v, s, wide);
  }
}

template <bool kF32, int D>
__global__ void __cluster_dims__(kQC, 1, 1) __launch_bounds__(kQThreads)
    quant_cluster_kernel(const __grid_constant__ QuantArgs q) {
  __shared__ float red[kQThreads / 32];
  __shared__ float cta_max;
  const int tensor = blockIdx.z, h = blockIdx.y, rank = blockIdx.x;
  const void *x = q.x[tensor];
  const bool rot = tensor == 0 && q.rope0.pos != nullptr;
  constexpr int vpr = D / 8;
  const int t0 = static_cast<int>(static_cast<int64_t>(q.n_tok) * rank / kQC);
  const int t1 = static_cast<int>(static_cast<int64_t>(q.n_tok) * (rank + 1) / kQC);
  const int n_vec = (t1 - t0) * vpr;
  // kQU raw 16-byte loads in flight per thread before any is used
  constexpr int kQU = 4;
  constexpr int kW = kF32 ? 2 : 1;
  float m = 0.f;
  for (int b = threadIdx.x; b < n_vec; b += kQU * kQThreads) {
    uint4 w[kQU][kW];
#pragma unroll
    for (int u = 0; u < kQU; ++u)
      if (b + u * kQThreads < n_vec) q_fetch<kF32, D>(x, q.H, h, t0, b + u * kQThreads, w[u]);
#pragma unroll
    for (int u = 0; u < kQU; ++u) {
      const int i = b + u * kQThreads;
      if (i >= n_vec) continue;
      float v[8];
      q_unpack<kF32>(w[u], v);
      if (rot) rope8(q.rope0, t0 + i / vpr, (i % vpr) * 8, D, v);
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
    }
  }
  const float a = q_cluster_max(m, red, &cta_max);
  const float s = a > 0.f ? __fdiv_rn(a, 448.f) : 1.f;
  if (rank == 0 && threadIdx.x == 0) q.scale[tensor][h] = s;
  const bool wide = q.wide[tensor] != 0;
  for (int b = threadIdx.x; b < n_vec; b += kQU * kQThreads) {
    uint4 wr[kQU][kW];
#pragma unroll
    for (int u = 0; u < kQU; ++u)
      if (b + u * kQThreads < n_vec) q_fetch<kF32, D>(x, q.H, h, t0, b + u * kQThreads, wr[u]);
#pragma unroll
    for (int u = 0; u < kQU; ++u) {
      const int i = b + u * kQThreads;
      if (i >= n_vec) continue;
      float v[8];
      q_unpack<kF32>(wr[u], v);
      const int l = t0 + i / vpr, c = i % vpr;
      if (rot) rope8(q.rope0, l, c * 8, D, v);
      q_store8(q.y[tensor], (static_cast<int64_t>(l) * q.H + h) * D + c * 8, v, s, wide);
    }
  }
}

static cca_status bulk_copy_pair(const uint8_t *k_src, const uint8_t *v_src, uint8_t *k_dst, uint8_t *v_dst,
                                 int64_t bytes, int32_t *dev_status, cudaStream_t st) {
  // The shared-memory limit is a per-device function attribute: set it once per device.
  static std::mutex mu;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t attr_err = cudaGetDevice(&dev);
  if (attr_err == cudaSuccess && (dev < 0 || dev >= 64)) return fail(CCA_ERR_UNSUPPORTED, "append: device %d", dev);
  if (attr_err == cudaSuccess) {
    std::lock_guard<std::mutex> lock(mu);
    if (!attr_set[dev]) {
      attr_err = cudaFuncSetAttribute(append_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kBulkStages * kBulkPiece);
      attr_set[dev] = attr_err == cudaSuccess;
    }
  }
  if (attr_err != cudaSuccess) return fail(CCA_ERR_CUDA, "append: %s", cudaGetErrorString(attr_err));
  const int64_t n_pieces = 2 * ((bytes + kBulkPiece - 1) / kBulkPiece);
  const int grid = static_cast<int>(cca_min64(num_sms(), n_pieces));
  append_bulk_kernel<<<grid, 32, kBulkStages * kBulkPiece, st>>>(k_src, v_src, k_dst, v_dst, bytes, dev_status);
  return launched("append_bulk_kernel");
}

// Quantise one or two [n_tok][H][D] tensors; scale arrays are [H] each.
constexpr int kQStageMax = 64 * 1024;  // shared memory per CTA of the staged form: at least 3 CTAs per SM

template <bool kF32, int D>
static cca_status quant_launch(const QuantArgs &q, cudaStream_t st) {
  const dim3 grid(kQC, q.H, q.n_tensors);
  const int64_t per_cta = (static_cast<int64_t>(q.n_tok) + kQC - 1) / kQC * (D / 8);  // vectors
  const int64_t stage = per_cta * 16 * (kF32 ? 2 : 1);
  if (stage <= kQStageMax) {
    static std::mutex mu;
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err == cudaSuccess && (dev < 0 || dev >= 64)) return fail(CCA_ERR_UNSUPPORTED, "quantise: device %d", dev);
    if (err == cudaSuccess) {
      std::lock_guard<std::mutex> lock(mu);
      if (!attr_set[dev]) {
        err = cudaFuncSetAttribute(quant_cpa_kernel<kF32, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   kQStageMax);
        attr_set[dev] = err == cudaSuccess;
      }
    }
    if (err != cudaSuccess) return fail(CCA_ERR_CUDA, "quantise: %s", cudaGetErrorString(err));
    quant_cpa_kernel<kF32, D><<<grid, kQThreads, static_cast<size_t>(stage), st>>>(q);
    return launched("quant_cpa_kernel");
  }
  quant_cluster_kernel<kF32, D><<<grid, kQThreads, 0, st>>>(q);
  return launched("quant_cluster_kernel");
}

static cca_status quantize_args(const QuantArgs &q, cca_dtype src, int D, cudaStream_t st) {
  if (src == CCA_F32) return D == 128 ? quant_launch<true, 128>(q, st) : quant_launch<true, 64>(q, st);
  return D == 128 ? quant_launch<false, 128>(q, st) : quant_launch<false, 64>(q, st);
}

static cca_status quantize_pair(const void *x0, const void *x1, cca_dtype src, int n_tok, int H, int D,
                                void *y0, void *y1, float *s0, float *s1, cudaStream_t st,
                                RopeArgs r0 = RopeArgs{nullptr, nullptr}, int wide0 = 0, int wide1 = 0) {
  const QuantArgs q{{x0, x1, nullptr}, {y0, y1, nullptr}, {s0, s1, nullptr}, {wide0, wide1, 0}, r0, n_tok, H,
                    x1 ? 2 : 1};
  return quantize_args(q, src, D, st);
}

}  // namespace cca

using namespace cca;

extern "C" {

cca_status cca_kv_ring_create(const cca_kv_ring_desc *desc, cca_kv_ring **out) {
  if (!desc || !out) return fail(CCA_ERR_INVALID_ARG, "cca_kv_ring_create: NULL argument");
  const cca_kv_ring_desc &d = *desc;
  if (d.n_heads < 1 || d.chunk_len < 1 || d.window < 0 || d.window > kMaxWindow)
    return fail(CCA_ERR_INVALID_ARG, "cca_kv_ring_create: need H >= 1, L >= 1, 0 <= W <= %d", kMaxWindow);
  if (d.head_dim != 64 && d.head_dim != 128)
    return fail(CCA_ERR_INVALID_ARG, "cca_kv_ring_create: head_dim must be 64 or 128 (got %d)", d.head_dim);
  if (static_cast<int64_t>(d.chunk_len) * d.n_heads * d.head_dim > kMaxChunkElems)
    return fail(CCA_ERR_INVALID_ARG, "cca_kv_ring_create: L * H * D must be <= 2^33");
  if (d.dtype != CCA_BF16 && d.dtype != CCA_E4M3)
    return fail(CCA_ERR_INVALID_ARG, "cca_kv_ring_create: dtype must be CCA_BF16 or CCA_E4M3");
  if (!d.k_slots || !d.v_slots || !aligned16(d.k_slots) || !aligned16(d.v_slots))
    return fail(CCA_ERR_INVALID_ARG, "cca_kv_ring_create: k_slots/v_slots must be non-NULL and 16-byte aligned");
  if (d.dtype == CCA_E4M3 && (!d.k_scale || !d.v_scale))
    return fail(CCA_ERR_INVALID_ARG, "cca_kv_ring_create: E4M3 ring needs k_scale and v_scale");
  if (d.dtype == CCA_BF16 && (d.k_scale || d.v_scale))
    return fail(CCA_ERR_INVALID_ARG, "cca_kv_ring_create: BF16 ring takes no scales");
  cca_kv_ring *r = new (std::nothrow) cca_kv_ring;
  if (!r) return fail(CCA_ERR_INVALID_ARG, "cca_kv_ring_create: out of host memory");
  r->d = d;
  r->n_appended = 0;
  *out = r;
  return CCA_OK;
}

cca_status cca_kv_ring_destroy(cca_kv_ring *ring) {
  delete ring;
  return CCA_OK;
}

cca_status cca_kv_ring_reset(cca_kv_ring *ring) {
  if (!ring) return fail(CCA_ERR_INVALID_ARG, "cca_kv_ring_reset: NULL ring");
  ring->n_appended = 0;
  return CCA_OK;
}

cca_status cca_kv_ring_query(const cca_kv_ring *ring, int64_t *n_appended, int32_t *slots,
                             int64_t *chunk_ids, int32_t *n_cached) {
  if (!ring) return fail(CCA_ERR_INVALID_ARG, "cca_kv_ring_query: NULL ring");
  if (n_appended) *n_appended = ring->n_appended;
  const int n = ring_visible(ring, slots, chunk_ids);
  if (n_cached) *n_cached = n;
  return CCA_OK;
}

cca_status cca_kv_ring_restore(cca_kv_ring *ring, int64_t n_appended) {
  if (!ring || n_appended < 0) return fail(CCA_ERR_INVALID_ARG, "cca_kv_ring_restore: bad argument");
  ring->n_appended = n_appended;
  return CCA_OK;
}

}  // extern "C"

static cca_status kv_append_impl(cca_kv_ring *ring, const void *k_new, const void *v_new, cca_dtype src_dtype,
                                 RopeArgs rk, cca_stream_t stream) {
  if (!ring || !k_new || !v_new) return fail(CCA_ERR_INVALID_ARG, "cca_kv_append: NULL argument");
  if (!aligned16(k_new) || !aligned16(v_new))
    return fail(CCA_ERR_INVALID_ARG, "cca_kv_append: k_new/v_new must be 16-byte aligned");
  if (src_dtype != CCA_BF16 && src_dtype != CCA_F32)
    return fail(CCA_ERR_INVALID_ARG, "cca_kv_append: src_dtype must be CCA_BF16 or CCA_F32");
  const cca_kv_ring_desc &d = ring->d;
  const int64_t t = ring->n_appended;
  if (t > 0 && d.window == 0) {  // nothing but the sink is ever cached
    ring->n_appended = t + 1;
    return CCA_OK;
  }
  const int slot = ring_slot_of(ring, t);
  const int64_t n_elem = static_cast<int64_t>(d.chunk_len) * d.n_heads * d.head_dim;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (d.dtype == CCA_BF16) {
    uint4 *kd = reinterpret_cast<uint4 *>(static_cast<char *>(d.k_slots) + slot * n_elem * 2);
    uint4 *vd = reinterpret_cast<uint4 *>(static_cast<char *>(d.v_slots) + slot * n_elem * 2);
    const int64_t n_vec = n_elem / 8;
    const int64_t per_block = (src_dtype == CCA_F32 ? kAppendUnrollF32 : kAppendUnroll) * 256;
    int64_t blocks = (n_vec + per_block - 1) / per_block;
    const int64_t cap = static_cast<int64_t>(num_sms()) * 2;  // x2 tensors: 4 blocks of 256 per SM
    if (blocks > cap) blocks = cap;
    dim3 grid(static_cast<unsigned>(blocks), 2);
    if (rk.pos) {  // K rotated on the way into the ring, V copied
      CCA_TRY(launch_rope_rows(k_new, v_new, kd, vd, true, false, src_dtype == CCA_F32, rk, d.chunk_len, d.n_heads,
                               d.head_dim, st));
    } else if (src_dtype == CCA_F32) {
      append_bf16_kernel<true><<<grid, 256, 0, st>>>(k_new, v_new, kd, vd, static_cast<int>(n_vec));
      CCA_TRY(launched("append_bf16_kernel"));
    } else {
      CCA_TRY(bulk_copy_pair(static_cast<const uint8_t *>(k_new), static_cast<const uint8_t *>(v_new),
                             reinterpret_cast<uint8_t *>(kd), reinterpret_cast<uint8_t *>(vd), n_elem * 2,
                             d.dev_status, st));
    }
  } else {
    uint8_t *kd = static_cast<uint8_t *>(d.k_slots) + slot * n_elem;
    uint16_t *vd = static_cast<uint16_t *>(d.v_slots) + slot * n_elem;  // e4m3 values widened to fp16
    CCA_TRY(quantize_pair(k_new, v_new, src_dtype, d.chunk_len, d.n_heads, d.head_dim, kd, vd,
                          d.k_scale + slot * d.n_heads, d.v_scale + slot * d.n_heads, st, rk, 0, 1));
  }
  ring->n_appended = t + 1;
  return CCA_OK;
}

extern "C" {

cca_status cca_kv_append(cca_kv_ring *ring, const void *k_new, const void *v_new, cca_dtype src_dtype,
                         cca_stream_t stream) {
  return kv_append_impl(ring, k_new, v_new, src_dtype, RopeArgs{nullptr, nullptr}, stream);
}

cca_status cca_kv_append_rope(cca_kv_ring *ring, const void *k_new, const void *v_new, cca_dtype src_dtype,
                              const int32_t *pos, const float *freq, cca_stream_t stream) {
  if (!pos || !freq || !aligned16(pos) || (reinterpret_cast<uintptr_t>(freq) & 3))
    return fail(CCA_ERR_INVALID_ARG, "cca_kv_append_rope: pos (16-byte aligned) and freq (4-byte aligned) required");
  return kv_append_impl(ring, k_new, v_new, src_dtype, RopeArgs{pos, freq}, stream);
}

cca_status cca_quant_e4m3(const void *x, cca_dtype src_dtype, int32_t n_tok, int32_t n_heads, int32_t head_dim,
                          uint8_t *x8, float *scale, cca_stream_t stream) {
  if (!scale || (n_tok > 0 && (!x || !x8)))
    return fail(CCA_ERR_INVALID_ARG, "cca_quant_e4m3: NULL argument");
  if (n_tok < 0 || n_heads < 1 || (head_dim != 64 && head_dim != 128))
    return fail(CCA_ERR_INVALID_ARG, "cca_quant_e4m3: need n_tok >= 0, H >= 1, D in {64,128}");
  if (src_dtype != CCA_BF16 && src_dtype != CCA_F32)
    return fail(CCA_ERR_INVALID_ARG, "cca_quant_e4m3: src_dtype must be CCA_BF16 or CCA_F32");
  if (n_tok > 0 && (!aligned16(x) || !aligned16(x8)))
    return fail(CCA_ERR_INVALID_ARG, "cca_quant_e4m3: x/x8 must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(scale) & 3u) != 0)
    return fail(CCA_ERR_INVALID_ARG, "cca_quant_e4m3: scale must be 4-byte aligned");
  return quantize_pair(x, nullptr, src_dtype, n_tok, n_heads, head_dim, x8, nullptr, scale, nullptr,
                       reinterpret_cast<cudaStream_t>(stream));
}

cca_status cca_quant_e4m3_f16(const void *x, cca_dtype src_dtype, int32_t n_tok, int32_t n_heads, int32_t head_dim,
                              void *x16, float *scale, cca_stream_t stream) {
  if (!scale || (n_tok > 0 && (!x || !x16)))
    return fail(CCA_ERR_INVALID_ARG, "cca_quant_e4m3_f16: NULL argument");
  if (n_tok < 0 || n_heads < 1 || (head_dim != 64 && head_dim != 128))
    return fail(CCA_ERR_INVALID_ARG, "cca_quant_e4m3_f16: need n_tok >= 0, H >= 1, D in {64,128}");
  if (src_dtype != CCA_BF16 && src_dtype != CCA_F32)
    return fail(CCA_ERR_INVALID_ARG, "cca_quant_e4m3_f16: src_dtype must be CCA_BF16 or CCA_F32");
  if (n_tok > 0 && (!aligned16(x) || !aligned16(x16)))
    return fail(CCA_ERR_INVALID_ARG, "cca_quant_e4m3_f16: x/x16 must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(scale) & 3u) != 0)
    return fail(CCA_ERR_INVALID_ARG, "cca_quant_e4m3_f16: scale must be 4-byte aligned");
  return quantize_pair(x, nullptr, src_dtype, n_tok, n_heads, head_dim, x16, nullptr, scale, nullptr,
                       reinterpret_cast<cudaStream_t>(stream), RopeArgs{nullptr, nullptr}, 1, 0);
}

cca_status cca_quant_e4m3_qkv(const void *q, const void *k, const void *v, cca_dtype src_dtype, int32_t n_tok,
                              int32_t n_heads, int32_t head_dim, uint8_t *q8, uint8_t *k8, void *v16, float *q_scale,
                              float *k_scale, float *v_scale, cca_stream_t stream) {
  if (!q_scale || !k_scale || !v_scale || (n_tok > 0 && (!q || !k || !v || !q8 || !k8 || !v16)))
    return fail(CCA_ERR_INVALID_ARG, "cca_quant_e4m3_qkv: NULL argument");
  if (n_tok < 0 || n_heads < 1 || (head_dim != 64 && head_dim != 128))
    return fail(CCA_ERR_INVALID_ARG, "cca_quant_e4m3_qkv: need n_tok >= 0, H >= 1, D in {64,128}");
  if (src_dtype != CCA_BF16 && src_dtype != CCA_F32)
    return fail(CCA_ERR_INVALID_ARG, "cca_quant_e4m3_qkv: src_dtype must be CCA_BF16 or CCA_F32");
  if (n_tok > 0 && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q8) || !aligned16(k8) ||
                    !aligned16(v16)))
    return fail(CCA_ERR_INVALID_ARG, "cca_quant_e4m3_qkv: tensors must be 16-byte aligned");
  if (((reinterpret_cast<uintptr_t>(q_scale) | reinterpret_cast<uintptr_t>(k_scale) |
        reinterpret_cast<uintptr_t>(v_scale)) & 3u) != 0)
    return fail(CCA_ERR_INVALID_ARG, "cca_quant_e4m3_qkv: scales must be 4-byte aligned");
  const QuantArgs a{{q, k, v}, {q8, k8, v16}, {q_scale, k_scale, v_scale}, {0, 0, 1}, RopeArgs{nullptr, nullptr},
                    n_tok, n_heads, 3};
  return quantize_args(a, src_dtype, head_dim, reinterpret_cast<cudaStream_t>(stream));
}

const char *cca_last_error(void) { return last_error().c_str(); }

int32_t cca_version(void) { return (0 << 16) | 1; }

int64_t cca_take_launch_count(void) {
  const int64_t n = launch_counter();
  launch_counter() = 0;
  return n;
}

}  // extern "C"
