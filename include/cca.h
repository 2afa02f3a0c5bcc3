/*
 * cca.h -- C ABI of libcca.so: chunk-wise causal attention over a bounded KV
 * cache, plus the L2 token-mask cache, for NVIDIA B200 (sm_100a).
 *
 * The operations follow the pages' statement of the problem:
 *
 *  - Chunk-wise causal attention with a global sink and a sliding window
 *    ["JoyAI-Video-Edit 소개", section 청크 단위 자기회귀 적응 (chunk-wise
 *    autoregressive adaptation); "論文解説: JoyAI-Video-Edit", step 1 (§4.1)]:
 *    tokens of a chunk attend to each other bidirectionally; chunk t attends
 *    causally to the first chunk (kept forever as a global sink) and to the W
 *    most recent earlier chunks, so per-chunk cost and memory are constant.
 *  - The bounded clean-KV store ["JoyAI-Video-Edit 소개", section 30 FPS를
 *    만드는 실시간 배포 파이프라인 (deployment pipeline); "論文解説", §5 loop]:
 *    after a chunk is generated its clean K/V are cached for the next chunk;
 *    the store keeps the sink plus the most recent chunks, evicting the oldest
 *    non-sink chunk.
 *  - FP8 quantisation in deployment (same deployment section); the e4m3 format
 *    with per-head absmax scales is this library's reading (not on the pages).
 *  - The AR-oriented mask cache ["LiveEdit 실시간 Diffusion 기반 스트리밍
 *    비디오 편집", sections 방법론 and 기술 상세]: mask_u = [ || z_edit,u -
 *    z_src,u ||_2 > tau ] on the previous chunk's latents, tau set to prune
 *    about 70 % of the tokens; active tokens are recomputed, the others reuse
 *    the cached self-attention output.
 *
 * Conventions shared by every call:
 *  - Pointers named "device" must point to device memory of the current CUDA
 *    device; "host" pointers to host memory.  The library never allocates
 *    device memory: the caller owns every device buffer.  The library owns only
 *    the small host-side ring handle.
 *  - Every call is asynchronous on the given stream (NULL = legacy default
 *    stream) and returns a status synchronously after host-side validation and
 *    kernel launch.  Errors raised on the device are written to the ring's
 *    optional device status word (CCA_DEV_*), never by trapping.
 *  - Every device buffer must be 16-byte aligned unless stated otherwise.
 *  - Tensors are dense and row-major.  [L][H][D] means token-major: element
 *    (l, h, d) is at ((l * H) + h) * D + d.
 *  - E4M3 mode: queries and keys are e4m3 codes (one byte); values are the
 *    e4m3-quantised values widened to fp16 (two bytes, exact: every e4m3
 *    value is an fp16 value), each tensor with fp32 per-head scales.  The
 *    attention keeps P in 16 bits (its e4m3 rounding alone moved outputs by
 *    0.1 on heavy-tailed inputs), so the PV product is 16-bit and reads V
 *    16-bit; widening V once, where it is quantised, spares every CTA a
 *    conversion of every V tile.  QK runs on the e4m3 tensor cores.
 *  - Handles are not thread-safe; distinct handles are independent.
 *  - On any non-CCA_OK status nothing has been launched unless the status is
 *    CCA_ERR_CUDA (a launch failed part-way); cca_last_error() then describes it.
 */
#ifndef CCA_H
#define CCA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ABI-compatible with cudaStream_t / CUstream. */
typedef struct CUstream_st *cca_stream_t;

typedef enum cca_status {
  CCA_OK = 0,
  CCA_ERR_INVALID_ARG = 1,    /* NULL pointer, misalignment, bad size or dtype   */
  CCA_ERR_UNSUPPORTED = 2,    /* valid request this build does not implement      */
  CCA_ERR_STATE = 3,          /* ring misuse (e.g. dtype mismatch with the ring)  */
  CCA_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed             */
  CCA_ERR_DEVICE_TIMEOUT = 5  /* returned by host-side readers of a status word   */
} cca_status;

/* Values written by kernels into the optional device status word. */
#define CCA_DEV_OK 0
#define CCA_DEV_TIMEOUT 1   /* a bounded device-side wait ran out; outputs invalid */
#define CCA_DEV_BAD_INDEX 2 /* a query index was outside [0, L); that row read as 0 */

typedef enum cca_dtype {
  CCA_BF16 = 0, /* bfloat16                                  */
  CCA_E4M3 = 1, /* OCP fp8 e4m3fn, with fp32 per-head scales */
  CCA_F32 = 2   /* float32                                   */
} cca_dtype;

/* ------------------------------------------------------------------------ */
/* Bounded KV cache ("ring")                                                 */
/* ------------------------------------------------------------------------ */

typedef struct cca_kv_ring cca_kv_ring; /* opaque host-side handle */

typedef struct cca_kv_ring_desc {
  int32_t n_heads;    /* H >= 1                                                  */
  int32_t head_dim;   /* D: 64 or 128                                            */
  int32_t chunk_len;  /* L >= 1 tokens per chunk; L * H * D <= 2^33            */
  int32_t window;     /* W >= 0 most recent non-sink chunks kept                 */
  cca_dtype dtype;    /* CCA_BF16 or CCA_E4M3                                    */
  void *k_slots;      /* device, [(1+W)][L][H][D] elements of dtype              */
  void *v_slots;      /* device, same shape; E4M3: fp16 (widened e4m3 values)    */
  float *k_scale;     /* device, [(1+W)][H] fp32 dequantisation scales (E4M3)    */
  float *v_scale;     /* device, [(1+W)][H] (E4M3); both NULL for BF16           */
  int32_t *dev_status;/* device, one int32 (CCA_DEV_*), may be NULL              */
} cca_kv_ring_desc;

/* Create a ring over caller-owned slot buffers (not cleared; nothing is read
 * before it is written).  Slot 0 holds chunk 0 (the sink, never evicted);
 * chunk t >= 1 lives in slot 1 + (t-1) mod W, overwriting chunk t-W.
 * Errors: CCA_ERR_INVALID_ARG (NULL/misaligned pointers, H < 1, D not in
 * {64,128}, L < 1, W < 0, W > 15, scales missing for E4M3). */
cca_status cca_kv_ring_create(const cca_kv_ring_desc *desc, cca_kv_ring **out);

/* Free the host handle (the caller's device buffers are untouched). */
cca_status cca_kv_ring_destroy(cca_kv_ring *ring);

/* Start a new stream: the next append becomes chunk 0 (the new sink). */
cca_status cca_kv_ring_reset(cca_kv_ring *ring);

/* Report the cache state.  n_appended (host, may be NULL) = chunks appended
 * so far = index t of the next (current) chunk.  slots / chunk_ids (host
 * arrays of >= 1+W entries, each may be NULL) receive, in logical order (sink
 * first, then oldest to newest), the ring slot and chunk index of every cached
 * chunk; *n_cached (host, may be NULL) their count.  With the caller's copy of
 * the slot buffers this is a complete snapshot of the stream state. */
cca_status cca_kv_ring_query(const cca_kv_ring *ring, int64_t *n_appended,
                             int32_t *slots, int64_t *chunk_ids,
                             int32_t *n_cached);

/* Restore a snapshot: set the number of appended chunks (the slot buffers must
 * hold the matching contents, e.g. copied back by the caller). */
cca_status cca_kv_ring_restore(cca_kv_ring *ring, int64_t n_appended);

/* Append the clean K/V of the chunk just generated (chunk t = n_appended) and
 * advance t.  k_new / v_new: device [L][H][D] of src_dtype (CCA_BF16 or
 * CCA_F32).  BF16 ring: bf16 copy (F32 input is rounded to nearest even).
 * E4M3 ring: per-head absmax quantisation, scale = absmax/448 (1 if all zero),
 * code = e4m3_rn_satfinite(x / scale) with an IEEE fp32 division; the scales
 * go to k_scale/v_scale[slot][h]; V is stored as the codes' values widened
 * to fp16.  Eviction is the overwrite of the slot.
 * Errors: CCA_ERR_INVALID_ARG, CCA_ERR_CUDA. */
cca_status cca_kv_append(cca_kv_ring *ring, const void *k_new, const void *v_new,
                         cca_dtype src_dtype, cca_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Rotary position encoding (fused 3D + 1D angle)                            */
/* ------------------------------------------------------------------------ */

/* ["JoyAI-Video-Edit 소개", section 세 부품으로 이루어진 아키텍처: positions are
 * encoded by a rotation whose angle fuses a 3D spatio-temporal RoPE with a 1D
 * source RoPE, so source and generated tokens of one sequence differ.]  The
 * formula is not on the pages; this library's reading: each token carries
 * integer coordinates pos = (t, h, w, s) -- latent frame, row, column and a
 * source index -- and pair i (elements 2i, 2i+1 of every head) is rotated by
 *     theta_i = t F[0][i] + h F[1][i] + w F[2][i] + s F[3][i]
 * (x'_{2i} = x_{2i} cos - x_{2i+1} sin, x'_{2i+1} = x_{2i} sin + x_{2i+1} cos):
 * the 3D rotation and the 1D source rotation act in the same plane, so their
 * angles add.  pos: device int32 [n_tok][4], 16-byte aligned.  F ("freq"):
 * device fp32 [4][D/2]. */

/* Default table into host memory freq[4][D/2]: coordinate a in {t, h, w}
 * turns the sec_a pairs of its section (t first, then h, then w; sec_t +
 * sec_h + sec_w = D/2) at frequencies base^(-j / sec_a), j = 0 .. sec_a-1, and
 * 0 elsewhere; the source index turns every pair i at base^(-2i / D).
 * Errors: CCA_ERR_INVALID_ARG. */
cca_status cca_mrope_freqs(int32_t head_dim, int32_t sec_t, int32_t sec_h, int32_t sec_w, float base,
                           float *freq);

/* Rotate the current chunk's queries and keys in one launch: q_out = rope(q),
 * k_out = rope(k), all [n_tok][H][D]; inputs CCA_BF16 or CCA_F32 (fp32
 * rotation, one rounding to the bf16 outputs).  Either q or k may be NULL (its
 * output is then ignored); outputs may alias their inputs for BF16 input.
 * Errors: CCA_ERR_INVALID_ARG, CCA_ERR_CUDA. */
cca_status cca_rope_qk(const void *q, const void *k, cca_dtype src_dtype, int32_t n_tok, int32_t n_heads,
                       int32_t head_dim, const int32_t *pos, const float *freq, void *q_out, void *k_out,
                       cca_stream_t stream);

/* cca_kv_append with the rotation applied to K as it is stored (V is stored
 * as given): the clean chunk's keys enter the cache already encoded.  For an
 * E4M3 ring the rotated keys are what the absmax scale and the codes are taken
 * from.  pos: [L][4] of the chunk being appended.  Errors: as cca_kv_append. */
cca_status cca_kv_append_rope(cca_kv_ring *ring, const void *k_new, const void *v_new, cca_dtype src_dtype,
                              const int32_t *pos, const float *freq, cca_stream_t stream);

/* ------------------------------------------------------------------------ */
/* FP8 quantiser                                                             */
/* ------------------------------------------------------------------------ */

/* Per-head absmax e4m3 quantisation of x (device [n_tok][H][D] of src_dtype,
 * CCA_BF16 or CCA_F32) into x8 (device [n_tok][H][D] uint8 codes) and scale
 * (device [H] fp32), with the same rule as cca_kv_append.  n_tok may be 0
 * (scales become 1).  Errors: CCA_ERR_INVALID_ARG, CCA_ERR_CUDA. */
cca_status cca_quant_e4m3(const void *x, cca_dtype src_dtype, int32_t n_tok,
                          int32_t n_heads, int32_t head_dim, uint8_t *x8,
                          float *scale, cca_stream_t stream);

/* The same quantisation, writing the codes' values widened to fp16 (device
 * [n_tok][H][D], two bytes each) instead of the codes: the form E4M3 attention
 * takes its V-side tensors in.  Errors: as cca_quant_e4m3. */
cca_status cca_quant_e4m3_f16(const void *x, cca_dtype src_dtype, int32_t n_tok, int32_t n_heads,
                              int32_t head_dim, void *x16, float *scale, cca_stream_t stream);

/* The current chunk's three attention inputs in one launch, each with its own
 * per-head scales: q8 = codes of q, k8 = codes of k, v16 = codes of v widened
 * to fp16 -- exactly cca_quant_e4m3(q), cca_quant_e4m3(k) and
 * cca_quant_e4m3_f16(v), the operands of an E4M3 cca_chunk_attn call.  All
 * tensors [n_tok][H][D], 16-byte aligned; scales device [H] fp32.
 * Errors: as cca_quant_e4m3. */
cca_status cca_quant_e4m3_qkv(const void *q, const void *k, const void *v, cca_dtype src_dtype, int32_t n_tok,
                              int32_t n_heads, int32_t head_dim, uint8_t *q8, uint8_t *k8, void *v16,
                              float *q_scale, float *k_scale, float *v_scale, cca_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Chunk attention                                                           */
/* ------------------------------------------------------------------------ */

/* O = softmax(Q K^T * softmax_scale) V for the queries of the current chunk
 * t = n_appended, over the keys/values of every visible chunk: the sink
 * (chunk 0), chunks max(1, t-W) .. t-1 from the ring, and the current chunk
 * itself from k_cur / v_cur (never from the ring: at a denoising step they are
 * computed from the noisy input).  No element mask inside that set.
 *
 *  q, k_cur, v_cur: device [L][H][D] in the ring's dtype (BF16; or E4M3: q and
 *      k_cur e4m3 codes, v_cur fp16-widened e4m3 values as cca_quant_e4m3_f16
 *      writes them, with per-head scales q_scale / kcur_scale / vcur_scale,
 *      device [H] fp32; the scale pointers must be NULL for BF16).  Scales must be finite
 *      and >= 0; a zero scale means all values of that head are zero.
 *  q_idx: NULL (queries are rows 0 .. n_q-1 of q) or device int32 row indices
 *      into q (the compacted active tokens of the mask cache).
 *  n_q_dev: NULL (n_q = n_q_max) or device int32 holding n_q <= n_q_max; read
 *      on the device, so no host synchronisation is needed.
 *  n_q_max: host bound on n_q, 0 <= n_q_max <= L.
 *  softmax_scale: <= 0 selects 1/sqrt(D).
 *  out: device [n_q_max][H][D] bf16; row i holds query i (rows >= n_q are
 *      not written).
 *  workspace / workspace_bytes: device scratch of at least the size reported
 *      by cca_chunk_attn_workspace_size (may be NULL if that size is 0); its
 *      contents need not be initialised and are garbage afterwards.
 * Errors: CCA_ERR_INVALID_ARG (NULL/misaligned pointers, n_q_max out of range,
 *      workspace too small), CCA_ERR_STATE (ring empty while the sink is
 *      needed is impossible: t = 0 attends to itself only), CCA_ERR_CUDA. */
cca_status cca_chunk_attn(const cca_kv_ring *ring, const void *q,
                          const void *k_cur, const void *v_cur,
                          const float *q_scale, const float *kcur_scale,
                          const float *vcur_scale, const int32_t *q_idx,
                          const int32_t *n_q_dev, int32_t n_q_max,
                          float softmax_scale, void *out, void *workspace,
                          size_t workspace_bytes, cca_stream_t stream);

/* Active-query attention with the scatter-back fused into its epilogue
 * ["LiveEdit ...", sections 방법론 and 기술 상세: recompute only where the mask
 * is 1, reuse the cached self-attention output elsewhere]: exactly
 * cca_chunk_attn with q_idx, except that the result for query i is written to
 * row q_idx[i] of o_cache instead of row i of a compact buffer, so no separate
 * cca_scatter pass (and no compact buffer) is needed.  Rows of o_cache that no
 * active query names keep their contents.
 *  q_idx: required, device int32 [n_q_max] (as produced by cca_compact);
 *      an index outside [0, L) sets CCA_DEV_BAD_INDEX and that row is skipped.
 *  o_cache: device bf16 [L][H][D].
 *  Other arguments, workspace and errors: as cca_chunk_attn (same workspace
 *  size). */
cca_status cca_chunk_attn_scatter(const cca_kv_ring *ring, const void *q,
                                  const void *k_cur, const void *v_cur,
                                  const float *q_scale, const float *kcur_scale,
                                  const float *vcur_scale, const int32_t *q_idx,
                                  const int32_t *n_q_dev, int32_t n_q_max,
                                  float softmax_scale, void *o_cache,
                                  void *workspace, size_t workspace_bytes,
                                  cca_stream_t stream);

/* Bytes of device workspace cca_chunk_attn needs for this ring and n_q_max
 * (the split-KV partial results; 0 when no split is used). */
cca_status cca_chunk_attn_workspace_size(const cca_kv_ring *ring, int32_t n_q_max,
                                         size_t *bytes);

/* Allocation-free cca_chunk_attn (no counterpart on the pages: a service for
 * callers that cannot provide device scratch memory, such as a real-time
 * stream loop that must not call the device allocator once running, or a host
 * application that owns every device allocation and gives plug-ins no
 * allocator).  Same arguments and results as cca_chunk_attn without the
 * workspace: the split-KV partial results go to a 64 MiB array compiled into
 * this library, which every GPU that loads the library holds until the
 * process exits.
 *  - No cudaMalloc, cudaFree or other allocating call is made.  Every call
 *    looks the array's device address up with cudaGetSymbolAddress (which
 *    allocates nothing).  The first call on a device also makes the CUDA
 *    runtime load this library's device code there, which places the array
 *    and can stall the stream once: make one warm-up call on each device
 *    before a real-time loop starts, and before any stream capture.
 *  - All calls share the one array and it keeps the last call's contents
 *    (nothing in it needs to start at zero).  Calls that may overlap on the
 *    GPU (different streams, or different host threads) race on it: serialise
 *    them, or use cca_chunk_attn with separate workspaces.
 *  - Errors: as cca_chunk_attn, plus CCA_ERR_INVALID_ARG when the call needs
 *    more scratch than the array holds (the message gives both sizes). */
cca_status cca_chunk_attn_noalloc(const cca_kv_ring *ring, const void *q,
                                  const void *k_cur, const void *v_cur,
                                  const float *q_scale, const float *kcur_scale,
                                  const float *vcur_scale, const int32_t *q_idx,
                                  const int32_t *n_q_dev, int32_t n_q_max,
                                  float softmax_scale, void *out,
                                  cca_stream_t stream);

/* Bytes of device workspace that suffice for every attention call of this
 * library with the given head_dim (64 or 128) on the current device: the
 * split-KV partial results of at most one CTA per SM (or CCA_ATTN_CTAS). */
cca_status cca_attn_workspace_size(int32_t head_dim, size_t *bytes);

/* ------------------------------------------------------------------------ */
/* Token groups of the active chunk, and the packed block-causal forward      */
/* ------------------------------------------------------------------------ */

/* Attention of one denoising step with the token groups of the pages' mask
 * ["JoyAI-Video-Edit 소개", section 세 부품으로 이루어진 아키텍처 (the
 * attention-mask figure: noisy tokens N_t, global tokens H_0, history tokens
 * H_{t-1}, MLLM condition tokens C_t, reference VAE tokens R, source VAE
 * tokens S_t) and section 청크 단위 자기회귀 적응 (the active chunk sees its
 * own source and condition tokens in both directions, the windowed history
 * and the global sink causally; future chunks are masked; only R is open to
 * every query)].
 *
 * The active block of chunk t = n_appended -- its groups N_t, S_t and C_t,
 * concatenated in any order as n_cur rows -- attends with one dense softmax to
 * the reference group R (n_ref rows; none when n_ref = 0), to the ring's
 * cached chunks (the sink and the window, exactly as cca_chunk_attn) and to
 * itself.  No element mask inside that set.  The history chunks of the ring
 * hold the clean tokens of earlier chunks (chunk_len rows each).
 *  q, k_cur, v_cur: device [n_cur][H][D] in the ring's dtype (E4M3: v_cur
 *      fp16-widened values); 0 <= n_cur <= 2^24.
 *  k_ref, v_ref: device [n_ref][H][D] (ring dtype; E4M3: v_ref fp16-widened),
 *      NULL when n_ref = 0.
 *  q_scale, kcur_scale, vcur_scale, kref_scale, vref_scale: E4M3 only,
 *      device [H] fp32 (NULL for BF16; the ref scales also NULL when n_ref = 0).
 *  out: device [n_cur][H][D] bf16.
 *  workspace: as cca_chunk_attn, of at least cca_attn_workspace_size(D) bytes.
 * R's own queries see R only: that is cca_block_attn with one chunk of R and
 * no history.  Errors: CCA_ERR_INVALID_ARG, CCA_ERR_UNSUPPORTED (E4M3 with
 * D = 64), CCA_ERR_CUDA. */
cca_status cca_chunk_attn_groups(const cca_kv_ring *ring, const void *q, const void *k_cur, const void *v_cur,
                                 int32_t n_cur, const void *k_ref, const void *v_ref, int32_t n_ref,
                                 const float *q_scale, const float *kcur_scale, const float *vcur_scale,
                                 const float *kref_scale, const float *vref_scale, float softmax_scale, void *out,
                                 void *workspace, size_t workspace_bytes, cca_stream_t stream);

/* Packed block-causal forward: every chunk of a sequence in one call, as in
 * training with teacher forcing ["JoyAI-Video-Edit 소개", section 청크 단위
 * 자기회귀 적응: the noisy active chunks, their clean history and the other
 * groups are packed into one sequence under the group mask, each target chunk
 * with its own noise level].  Chunk c (0 <= c < T) of the "current" tensors
 * (the noisy chunks) attends to: R (ref_len rows, optional), the history
 * chunks {0} U {max(1, c-W) .. c-1} of the "history" tensors (the clean
 * chunks; chunk 0 is the sink) and current chunk c itself.  With the history
 * tensors equal to the current ones this is plain windowed block-causal
 * attention (W >= T-1: full block-causal), which also gives the clean
 * chunks' own outputs.
 *  k_cur, v_cur, k_hist, v_hist: device [T][L][H][D] (dtype; E4M3: the V
 *      tensors fp16-widened values); the history tensors may alias the current
 *      ones.
 *  k_ref, v_ref: device [ref_len][H][D] or NULL with ref_len = 0.
 *  Scales (E4M3 only, else NULL): kcur/vcur/khist/vhist [T][H], kref/vref [H].
 *  dev_status: device int32 (CCA_DEV_*), may be NULL. */
typedef struct cca_block_desc {
  int32_t n_heads;      /* H >= 1                                   */
  int32_t head_dim;     /* D: 64 or 128 (E4M3: 128)                 */
  int32_t chunk_len;    /* L >= 1 tokens per chunk                  */
  int32_t n_chunks;     /* T, 0 <= T <= 4095                        */
  int32_t window;       /* W >= 0 history chunks besides the sink   */
  cca_dtype dtype;      /* CCA_BF16 or CCA_E4M3                     */
  const void *k_cur, *v_cur, *k_hist, *v_hist, *k_ref, *v_ref;
  int32_t ref_len;
  const float *kcur_scale, *vcur_scale, *khist_scale, *vhist_scale, *kref_scale, *vref_scale;
  int32_t *dev_status;
} cca_block_desc;

/* q: device [T][L][H][D] (dtype); q_scale: E4M3 [T][H] else NULL; out: device
 * [T][L][H][D] bf16.  workspace: at least cca_attn_workspace_size(D) bytes
 * (reused by the launches of the call, which run in order on the stream).
 * Errors: CCA_ERR_INVALID_ARG, CCA_ERR_UNSUPPORTED, CCA_ERR_CUDA. */
cca_status cca_block_attn(const cca_block_desc *desc, const void *q, const float *q_scale, float softmax_scale,
                          void *out, void *workspace, size_t workspace_bytes, cca_stream_t stream);

/* ------------------------------------------------------------------------ */
/* L2 token mask, compaction, scatter (LiveEdit mask cache)                 */
/* ------------------------------------------------------------------------ */

/* mask[u] = (d2[u] > tau2) with d2[u] = sum_c (edit[u][c] - src[u][c])^2 in
 * fp32, i.e. ||edit_u - src_u||_2 > tau.
 *  src, edit: device [n_tok][n_ch] fp32 latents of the previous chunk.
 *  prune_quantile < 0: fixed threshold, tau2 = tau * tau (fp32).
 *  0 < prune_quantile <= 1: dynamic threshold, tau2 = the k-th smallest d2
 *      with k = ceil(prune_quantile * n_tok) computed in binary64, so exactly
 *      n_tok - k tokens are active when distances are distinct (ties at the
 *      threshold stay inactive).  Needs n_tok <= 32768.
 *  mask: device uint8 [n_tok] (0/1).  dist2_out: device fp32 [n_tok] or NULL.
 *  tau_out: device fp32, receives sqrt(tau2), or NULL.
 * n_ch must be a multiple of 4 (<= 256); src/edit 16-byte aligned.
 * Errors: CCA_ERR_INVALID_ARG, CCA_ERR_CUDA. */
cca_status cca_token_mask_l2(const float *src, const float *edit, int32_t n_tok,
                             int32_t n_ch, float tau, float prune_quantile,
                             uint8_t *mask, float *dist2_out, float *tau_out,
                             cca_stream_t stream);

/* The mask over a chunk of several latent frames ["LiveEdit ...", section 기술
 * 상세: inference runs chunks of 3 latent frames; the mask M^k_{u,v} is
 * indexed by spatial position only].  Reading: one decision per position p,
 * from the L2 norm over the channels of every frame of chunk k-1 at p, applied
 * to the tokens of all frames of chunk k at p.
 *  src, edit: device [n_frames][n_pos][n_ch] fp32 (frame-major, 16-byte aligned).
 *  mask: device uint8 [n_frames][n_pos]; mask[f][p] = [d2(p) > tau2] for every f.
 *  dist2_out: device fp32 [n_pos] or NULL; tau_out as cca_token_mask_l2.
 *  Dynamic tau: the k-th smallest d2 over the n_pos positions, k = ceil(q n_pos)
 *  (n_pos <= 32768).  1 <= n_frames <= 64; n_frames = 1 is cca_token_mask_l2.
 *  Compacting the mask (cca_compact over n_frames * n_pos tokens) lists the
 *  active tokens frame by frame, ascending.  Errors: as cca_token_mask_l2. */
cca_status cca_token_mask_l2_frames(const float *src, const float *edit, int32_t n_frames, int32_t n_pos,
                                    int32_t n_ch, float tau, float prune_quantile, uint8_t *mask, float *dist2_out,
                                    float *tau_out, cca_stream_t stream);

/* idx[0 .. n) = ascending positions u with mask[u] != 0; *n_active_dev = n.
 *  mask: device uint8 [n_tok], 16-byte aligned; idx: device int32 [n_tok],
 *  4-byte aligned (entries >= n are not written); n_active_dev: device int32.
 *  0 <= n_tok <= 2^30.  n_tok <= 16384: one CTA, workspace may be NULL.
 *  Larger n_tok: one cooperative launch of co-resident CTAs (count, offset of
 *  each CTA's run from the totals of the runs before it, write), which needs
 *  a 16-byte aligned device workspace of cca_compact_workspace_size bytes
 *  (contents need not be initialised; not shared by concurrent calls).  If
 *  one of its bounded device-side waits runs out, *n_active_dev is set to -1
 *  and idx is not valid.
 * Errors: CCA_ERR_INVALID_ARG, CCA_ERR_CUDA. */
cca_status cca_compact(const uint8_t *mask, int32_t n_tok, int32_t *idx,
                       int32_t *n_active_dev, void *workspace,
                       size_t workspace_bytes, cca_stream_t stream);

/* Bytes of workspace cca_compact needs for n_tok tokens (0 up to 16384). */
cca_status cca_compact_workspace_size(int32_t n_tok, size_t *bytes);

/* o_cache row idx[i] <- o_compact row i for i < *n_active_dev; every other row
 * of o_cache is left untouched (it keeps the output cached at chunk k-1).
 *  o_compact: device [n_max][row_bytes]; o_cache: device [*][row_bytes];
 *  idx, n_active_dev: as produced by cca_compact; n_max: host bound on n.
 *  row_bytes must be a multiple of 16.  Errors: CCA_ERR_INVALID_ARG, CCA_ERR_CUDA. */
cca_status cca_scatter(const void *o_compact, const int32_t *idx,
                       const int32_t *n_active_dev, int32_t n_max,
                       int32_t row_bytes, void *o_cache, cca_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Diagnostics                                                               */
/* ------------------------------------------------------------------------ */

/* Self-test of the device-side bounded wait used by every kernel here: one
 * thread waits on an mbarrier phase that nothing completes (arrive_first = 0)
 * or that it completed itself (arrive_first != 0, a positive control), giving
 * up after budget_cycles SM clock cycles (1 .. 4e9).  *dev_status (device int32)
 * receives CCA_DEV_TIMEOUT or CCA_DEV_OK; the context stays usable either way.
 * No counterpart on the pages: it backs the library's failure reporting. */
cca_status cca_selftest_bounded_wait(int32_t *dev_status, int64_t budget_cycles,
                                     int32_t arrive_first, cca_stream_t stream);

/* Message describing the last error of the calling thread ("" if none). */
const char *cca_last_error(void);

/* Library version, (major << 16) | minor. */
int32_t cca_version(void);

/* Number of kernels the calling thread has launched through this library
 * since the last call (the counter is reset by the call). */
int64_t cca_take_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* CCA_H */
