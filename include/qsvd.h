/*
 * qsvd.h -- C ABI of the joint-QKV latent decode library (NVIDIA B200, sm_100a).
 *
 * The operation.  QSVD compresses the query, key and value projections of an
 * attention layer jointly: [W_Q W_K W_V] (E x 3E) ~= W^d [W^u_q W^u_k W^u_v],
 * with one shared down-projection W^d (E x r) and three up-projections W^u_*
 * (r x E each).  Only the latent C = X W^d (L x r per sequence) is cached;
 * keys and values are rebuilt from it on the fly as C W^u_k and C W^u_v.
 *   - QSVD paper notes (Paper-Notes, NeurIPS 2025), section 关键设计,
 *     "QKV联合SVD分解" (joint SVD, shared latent of size r x L, 4rE weights).
 *   - QSVD paper digest, section Method, Step 1 (C_qkv buffered, K and V
 *     recomputed on the fly) and Step 3 (H1/H2 rotations, beta split,
 *     latent quantisation).
 *   - WSVD paper digest, sections Problem and Method 3.4: a decoder that
 *     re-reads the shared latent once per head moves more bytes than an
 *     uncompressed cache; a fused flash-decoding kernel reconstructs keys
 *     on-chip and applies rotary embedding.
 * This library implements one decode step of that attention: every head
 * reads the latent tile once from HBM (split-KV flash decoding), with the
 * query absorbed into latent space (no rotary embedding) or with per-tile key
 * reconstruction on the tensor cores followed by rotary embedding.
 *
 * Conventions shared by all calls:
 *   - Every tensor pointer is a DEVICE pointer owned by the caller, unless
 *     the argument says "host".  The library never allocates device memory
 *     and keeps no per-model state; scratch lives in a caller-provided
 *     workspace whose size the library reports.
 *   - All work is enqueued asynchronously on `stream` (a cudaStream_t passed
 *     as void*; NULL is the legacy default stream).  No call synchronises.
 *   - Row-major layouts; "B x E" means B rows of E contiguous elements.
 *   - Heads: head h owns columns [h*d_h, (h+1)*d_h) of every E-wide matrix.
 *   - Errors detectable on the host return a status and enqueue nothing.
 *     Violations only visible on the device (a length or position out of
 *     range) are clamped and recorded as bits in a device status word; no
 *     kernel traps.
 *   - Device pointers must be 16-byte aligned, except fp16 group scales
 *     (2-byte) and the float32 c_out of an append (4-byte).  The calls
 *     check the pointers they vectorise or hand to TMA and return
 *     QSVD_ERR_INVALID_ARG for a misaligned one.
 */
#ifndef QSVD_H
#define QSVD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QSVD_ABI_VERSION 3

typedef enum {
  QSVD_OK = 0,
  QSVD_ERR_INVALID_ARG = 1,  /* null pointer, inconsistent or unsupported sizes */
  QSVD_ERR_UNSUPPORTED = 2,  /* valid request that this build has no kernel for */
  QSVD_ERR_WORKSPACE = 3,    /* workspace or packed buffer too small */
  QSVD_ERR_CUDA = 4          /* a CUDA runtime call or kernel launch failed */
} qsvd_status;

typedef enum {
  QSVD_F32 = 0,
  QSVD_F16 = 1,
  QSVD_BF16 = 2,
  QSVD_I8 = 3,   /* latent cache only: int8 codes + fp16 group scales */
  QSVD_I4 = 4    /* latent cache only: packed int4 codes + fp16 group scales */
} qsvd_dtype;

/* Split-KV granularity: sequences are cut into tiles of this many tokens. */
#define QSVD_TILE_TOKENS 128

/* Phases of qsvd_decode_attn (bit mask; 0 means all). */
#define QSVD_PHASE_PROLOGUE 1u  /* query (c_new W^u_q), absorption or rotary */
#define QSVD_PHASE_SPLIT 2u     /* split-KV attention over the latent tiles */
#define QSVD_PHASE_COMBINE 4u   /* merge of the split partials, value up-projection */
#define QSVD_PHASE_ALL 7u
/* The two passes of the split phase in rotary mode on the tensor cores
 * (QSVD_PHASE_SPLIT runs both): keys rebuilt from the latent, rotated and
 * scored into the workspace; then the softmax and the latent accumulation
 * over those scores.  Any other path rejects them with INVALID_ARG. */
#define QSVD_PHASE_SPLIT_SCORES 8u
#define QSVD_PHASE_SPLIT_ACCUM 16u

/* Device status bits (workspace word 0 for decode; `status` for append). */
#define QSVD_STATUS_LEN_CLAMPED 1   /* some lengths[b] < 0 or > max_len (clamped) */
#define QSVD_STATUS_POS_OOB 2       /* some pos[b] outside [0, max_len) (row not written) */
#define QSVD_STATUS_SCALE_SAT 4     /* a group scale exceeded the fp16 range (saturated) */
#define QSVD_STATUS_TIMEOUT 8       /* a pipeline wait in the split kernel timed out (the
                                       output of that call is invalid) */

/* Split-kernel choice (qsvd_dims.kernel). */
#define QSVD_KERNEL_AUTO 0
#define QSVD_KERNEL_SIMT 1      /* CUDA-core split kernel: every dtype and mode */
#define QSVD_KERNEL_TCGEN05 2   /* tensor cores (tcgen05, TMA): one CTA per split where
                                   that kernel applies, else the cluster kernel */
#define QSVD_KERNEL_TCGEN05_CTA 3      /* tensor cores, one CTA per split */
#define QSVD_KERNEL_TCGEN05_CLUSTER 4  /* tensor cores, the latent channels of a tile
                                          spread over a thread-block cluster (absorbed
                                          mode, fp16/bf16 cache, r = 128 k or 256 k with
                                          2 <= k <= 8, H <= 32) */
/* The workspace header records the kernel that ran: SIMT, TCGEN05_CTA or
 * TCGEN05_CLUSTER. */

/* Output projection applied by the combine (qsvd_dims.out_proj).  WSVD
 * digest, Method, fused kernel (§3.4): the value up-projection is merged
 * into the attention layer's output projection W_O so that V is never built.
 *   NONE   out = o (B x E, heads concatenated), o_h = z_h W^u_{v,h}.
 *   CHAIN  out = o W_O: the V-up GEMV, then a GEMV by W_O (E x E).
 *   FOLD   out = sum_h z_h F_h with F_h = W^u_{v,h} W_{O,h} (r x E), the
 *          rows h d_h .. h d_h + d_h - 1 of W_O: one GEMV over the merged
 *          latents, no V-up.  F (H r x E) is formed once by
 *          qsvd_prepare_out_proj.
 * CHAIN and FOLD need 16-bit weights and d_h % 64 == 0. */
#define QSVD_OUT_PROJ_NONE 0
#define QSVD_OUT_PROJ_CHAIN 1
#define QSVD_OUT_PROJ_FOLD 2

typedef struct {
  int E;               /* model width, E = H * d_h */
  int H;               /* heads */
  int d_h;             /* head dim (multiple of 8, at most 256) */
  int r;               /* retained rank (latent width; multiple of 32, 32..8192) */
  int batch;           /* B sequences per call (at most 65535) */
  int max_len;         /* cache rows per sequence (capacity); batch x max_len < 2^31 */
  int group;           /* channels per quantisation group (I8/I4 caches) */
  int rope;            /* 0: no rotary embedding, query absorbed; 1: rotary */
  float rope_base;     /* rotary base (e.g. 10000) */
  float softmax_scale; /* score scale; <= 0 selects 1/sqrt(d_h) */
  qsvd_dtype cache_dtype;   /* F32, F16, BF16, I8 or I4 */
  qsvd_dtype weight_dtype;  /* F32, F16 or BF16: W^d, W^u_*, and append's x */
  qsvd_dtype out_dtype;     /* F32, F16 or BF16 */
  int h2;              /* 1: append applies H2 to the latent before quantising */
  int h2_m;            /* order m of the small factor of H2 = H_{r/m} (x) Q_m */
  int kernel;          /* QSVD_KERNEL_* */
  int out_proj;        /* QSVD_OUT_PROJ_* */
} qsvd_dims;

/*
 * qsvd_prepare_weights -- lay out the factors for the decode kernels.
 * Source: QSVD paper notes, 关键设计 (shared W^d, separate W^u_q/k/v; the
 * rotation identity Y = (X H1^T)(H1 W^d H2^T)(H2 W^u)); QSVD digest, Method,
 * Step 3.
 *   wd            device, E x r, weight_dtype: W^d.
 *   wuq/wuk/wuv   device, r x E each, weight_dtype: W^u_q, W^u_k, W^u_v.
 *   h2_q          HOST, h2_m x h2_m float32 row-major orthogonal matrix Q, or
 *                 NULL.  When given, H2 = H_{r/h2_m} (x) Q (normalised
 *                 Sylvester Hadamard; r/h2_m must be a power of two) is
 *                 folded into the up-projections (W^u_* <- H2 W^u_*) and,
 *                 unless dims->h2 == 1, into W^d (W^d <- W^d H2^T).  With
 *                 dims->h2 == 1, W^d is kept and append rotates each latent.
 *                 The fold runs in float32 and rounds once to weight_dtype.
 *   packed        device buffer receiving the laid-out weights (owned by the
 *                 caller, 256-byte aligned), or NULL to query the size.
 *   packed_bytes  in: capacity of `packed`; out: bytes required.
 * Rotary mode also stores a float32 cos/sin table for positions < max_len,
 * built from float64 angles.  The packed buffer is read-only afterwards and
 * may be shared by concurrent calls with the same dims.
 * Errors: INVALID_ARG (dims, null inputs), WORKSPACE (capacity too small),
 * CUDA (launch failure).
 */
qsvd_status qsvd_prepare_weights(const qsvd_dims* dims, const void* wd,
                                 const void* wuq, const void* wuk,
                                 const void* wuv, const float* h2_q,
                                 void* packed, size_t* packed_bytes,
                                 void* stream);

/*
 * qsvd_append_latent -- project one new token per sequence into the latent
 * and write it into the cache.
 * Source: QSVD digest, Method, Step 1 (C = X W^d is the buffered
 * intermediate) and Step 3 (H2 rotation, latent quantisation); QSVD paper
 * notes, 实验关键数据 (A8/A4 latent precisions).
 *   x       device, B x E, weight_dtype: the new tokens' activations.
 *   pos     device, B int32: row written for sequence b (0 <= pos < max_len).
 *   cache   device, B x max_len rows; row layout by cache_dtype:
 *             F32/F16/BF16: r elements;  I8: r int8 codes;
 *             I4: r/2 bytes, element 2j in the low nibble, 2j+1 in the high
 *             nibble (two's complement).
 *   scales  device, B x max_len x (r/group) float16, 2-byte aligned (I8/I4
 *           only; else NULL).
 *   c_out   device, B x r float32 (4-byte aligned), or NULL: receives
 *           c = x W^d (after H2 when dims->h2 == 1), i.e. the exact input
 *           of the quantiser.
 *   status  device int32 word or NULL; bits QSVD_STATUS_* are OR-ed in.
 *   workspace        device scratch (split-K partials of x W^d), or NULL to
 *                    query the size into *workspace_bytes (in: capacity).
 * Quantiser (I8/I4): per token and group of `group` channels,
 *   scale = fp16_rn(amax / qmax) (IEEE float32 division; saturates at 65504
 *   and sets QSVD_STATUS_SCALE_SAT), code = 0 if scale == 0 else
 *   clamp(rint_half_even(c / scale), -qmax, qmax), qmax = 127 or 7.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
qsvd_status qsvd_append_latent(const qsvd_dims* dims, const void* packed,
                               const void* x, const int32_t* pos, void* cache,
                               void* scales, float* c_out, int32_t* status,
                               void* workspace, size_t* workspace_bytes,
                               void* stream);

/*
 * qsvd_prefill_latent -- the latent rows of many tokens at once (a prompt):
 * c_i = x_i W^d for n_rows rows of x, each rounded to the cache type or
 * quantised exactly as qsvd_append_latent does, stored at cache row
 * dst_rows[i] (= b * max_len + t for token t of sequence b).
 * Source: QSVD paper notes, 关键设计 (only C = X W^d is cached); QSVD digest,
 * Method, Step 3 (quantised latent).  One tensor-core GEMM with the rounding
 * or quantisation fused into its epilogue.
 *   x             device, n_rows x E, weight_dtype, row-major, 16-byte aligned.
 *   n_rows        >= 0 (0: nothing is enqueued).
 *   dst_rows      device, n_rows int32: destination cache row of each x row;
 *                 rows outside [0, B * max_len) are skipped and flagged
 *                 (QSVD_STATUS_POS_OOB).
 *   cache, scales as in qsvd_append_latent.
 *   c_fp32_debug  device, n_rows x r float32 (16-byte aligned), or NULL:
 *                 receives c before rounding, the exact input of the
 *                 quantiser.
 *   status        device int32 word or NULL; bits QSVD_STATUS_* are OR-ed in.
 * Requires 16-bit weights, r % 256 == 0, E % 64 == 0, group == 128 for int
 * caches, and H2 folded into the weights (dims->h2 == 0); else UNSUPPORTED.
 * The tensor cores sum the fp32 products in their own order, so c can differ
 * from qsvd_append_latent's in the last bits; a given c is rounded and
 * quantised identically.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
qsvd_status qsvd_prefill_latent(const qsvd_dims* dims, const void* packed,
                                const void* x, int n_rows, const int32_t* dst_rows,
                                void* cache, void* scales, float* c_fp32_debug,
                                int32_t* status, void* stream);

/*
 * qsvd_beta_exponents -- the split exponents of one beta for
 * qsvd_split_factors: a_j = float(sigma_j^beta), b_j = float(sigma_j^(1 -
 * beta)), the powers taken in float64 (QSVD paper notes, 关键设计: the latent
 * is X U_r Sigma_r^beta; the up-projection carries Sigma_r^(1 - beta)).
 *   sigma  device, r float32 singular values (>= 0); 1 <= r <= 8192.
 *   a, b   device, r float32 each (written).
 * Stream-ordered.  Errors: INVALID_ARG, CUDA.
 */
qsvd_status qsvd_beta_exponents(const float* sigma, int r, double beta, float* a, float* b, void* stream);

/*
 * qsvd_sq_diff_sum -- *out = sum_i (y_i - yq_i)^2 over n float32 pairs,
 * accumulated in float64 on the device: the calibration objective
 * sum_d ||Y_d - Y'_d||^2 of the beta search (QSVD paper notes, 核心创新) over
 * the decode outputs from the float32 and the quantised latent rows.
 *   y, yq  device, n float32 each.
 *   out    device, one float64 (overwritten; the sum of per-block partials,
 *          added in an unspecified order).
 * Stream-ordered.  Errors: INVALID_ARG, CUDA.
 */
qsvd_status qsvd_sq_diff_sum(const float* y, const float* yq, int64_t n, double* out, void* stream);

/*
 * qsvd_prefill_attention -- causal attention over the prompts whose latent
 * rows are in the cache (the attention of a prefill step).  Source: QSVD
 * digest, Method, Step 1 (queries, keys and values are rebuilt from the
 * buffered latent: Q = C W^u_q, K = C W^u_k, V = C W^u_v) and Key
 * Contributions (the prompt is read once, into the latent); rotary embedding
 * as in the decode (WSVD digest, Method §3.4).  For prompt b of length
 * len_b (its latent rows are cache rows b max_len + t, t < len_b) and head h:
 *   o_t = sum_{u <= t} softmax_u(tau q_t . k_u) v_u
 * with q_t, k_u rotated to their own positions when dims->rope is set and
 * tau = dims->softmax_scale (<= 0: 1/sqrt(d_h)).  Q, K and V are rebuilt by
 * the tensor-core latent GEMM in float32 and held as two 16-bit parts each
 * (hi and rounding residual); the attention runs on tcgen05 with float32
 * accumulation.
 *   packed     from qsvd_prepare_weights (its W^u_q, W^u_k, W^u_v and, with
 *              dims->rope, its rotary table).
 *   cache      device, B x max_len x r, cache_dtype (F16 or BF16, equal to
 *              weight_dtype), 16-byte aligned.
 *   lengths    device, B int32 prompt lengths, clamped to [0, max_len].
 *   workspace  device scratch, 16-byte aligned, or NULL to query its size
 *              into *workspace_bytes (in: capacity):
 *              B max_len E (4 + 6 x 2) bytes.
 *   out        device, B x max_len x E, out_dtype, 16-byte aligned: rows
 *              t < len_b are written, other rows are left as they were.
 *   status     device int32 word; QSVD_STATUS_TIMEOUT is OR-ed in if a
 *              pipeline wait expired.
 * Requires d_h == 128, E % 256 == 0, r % 64 == 0; else UNSUPPORTED.
 * Stream-ordered; nothing is allocated.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 */
qsvd_status qsvd_prefill_attention(const qsvd_dims* dims, const void* packed, const void* cache,
                                   const int32_t* lengths, void* workspace, size_t* workspace_bytes,
                                   void* out, int32_t* status, void* stream);

/*
 * qsvd_append_latent_static -- qsvd_append_latent without a workspace.
 * The paper has no counterpart: this is an interface variant for callers
 * that cannot allocate device memory -- a serving engine or plugin host that
 * owns every buffer and passes only the call's tensors, or a deployment with
 * a fixed memory budget that forbids allocation after start-up.
 * Same arguments, results and status bits as qsvd_append_latent, minus the
 * workspace.  The split-K partials of x W^d go to a static device array of
 * 1,048,576 floats (4 MiB) that every GPU loading the library holds until
 * the process exits; requests needing more, i.e. ksplit * batch * r >
 * 1,048,576 with ksplit = ceil(E / 512) for 16-bit weights (ceil(E / 64)
 * for float32), return QSVD_ERR_WORKSPACE and enqueue nothing.  Nothing is
 * allocated.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - Every call shares the array.  It needs no clearing (each call writes
 *     every partial it reads), but calls that overlap on the GPU -- on
 *     different streams, or from several host threads -- race on it and
 *     must be serialised by the caller.
 */
qsvd_status qsvd_append_latent_static(const qsvd_dims* dims, const void* packed,
                                      const void* x, const int32_t* pos, void* cache,
                                      void* scales, float* c_out, int32_t* status,
                                      void* stream);

/*
 * qsvd_split_factors -- the rank-r factors for one split of the singular
 * values between the down- and the up-projection (QSVD paper notes, 关键设计:
 * the latent is X U_r Sigma_r^beta; 核心创新: beta is fitted on calibration
 * data): W^d = U_r diag(a), [W^u_q W^u_k W^u_v] = diag(b) V_r^T, each entry
 * one float32 product rounded once to weight_dtype.  For a split exponent
 * beta the caller passes a_j = sigma_j^beta, b_j = sigma_j^(1 - beta).
 *   u      device, E x r float32 row-major: the first r left singular vectors.
 *   vt     device, r x 3E float32 row-major: the first r right singular
 *          vectors of [W_Q W_K W_V] (columns 0..E-1 belong to W_Q, E..2E-1
 *          to W_K, 2E..3E-1 to W_V).
 *   a, b   device, r float32 each.
 *   wd     device, E x r, weight_dtype (written).
 *   wuq, wuk, wuv  device, r x E each, weight_dtype (written); the inputs
 *          of qsvd_prepare_weights.
 * Stream-ordered; nothing is allocated.
 * Errors: INVALID_ARG (NULL pointer, bad dims), CUDA.
 */
qsvd_status qsvd_split_factors(const qsvd_dims* dims, const float* u, const float* vt,
                               const float* a, const float* b, void* wd, void* wuq, void* wuk,
                               void* wuv, void* stream);

/*
 * qsvd_prepare_out_proj -- add the output projection W_O to a packed buffer
 * that qsvd_prepare_weights filled with the same dims (dims->out_proj CHAIN
 * or FOLD; qsvd_prepare_weights reports the size with room for it).
 * Source: WSVD digest, Method, fused kernel (§3.4).
 *   wo            device, E x E row-major, weight_dtype: y = o W_O, row
 *                 h d_h + i of W_O multiplies channel i of head h.
 *   packed        the buffer of qsvd_prepare_weights (read: W^u_v, already
 *                 rotated by H2 when one was folded in; written: the W_O
 *                 section).  CHAIN copies W_O; FOLD writes
 *                 F[h r + j][n] = sum_i W^u_v[j][h d_h + i] W_O[h d_h + i][n],
 *                 accumulated in float32 over i in order and rounded once
 *                 to weight_dtype.
 *   packed_bytes  in: capacity of packed.
 * Stream-ordered; nothing is allocated.
 * Errors: INVALID_ARG (out_proj NONE, NULL pointers, small buffer),
 * UNSUPPORTED (fp32 weights, d_h % 64 != 0), CUDA.
 */
qsvd_status qsvd_prepare_out_proj(const qsvd_dims* dims, const void* wo, void* packed,
                                  size_t packed_bytes, void* stream);

/*
 * qsvd_decode_attn -- one decode step of multi-head attention over the
 * latent cache, output B x E.
 * Source: QSVD digest, Method, Step 1 (keys/values rebuilt from C_qkv);
 * WSVD digest, Method 3.4 (flash decoding over latent tiles, rotary keys).
 *   qin            device, float32: B x r latent of the current token when
 *                  qin_is_latent != 0 (q = qin W^u_q), else the B x E query.
 *   cache, scales  as in qsvd_append_latent.
 *   lengths        device, B int32: tokens attended by sequence b (rows
 *                  0..len-1; the query sits at position len-1 for rotary).
 *                  len == 0 gives a zero output row.  Values outside
 *                  [0, max_len] are clamped and flagged.
 *   num_splits     number of split CTAs G of the split phase (0: one wave on
 *                  this device), capped at B x ceil(max_len / 128) and at
 *                  2048.  Tiles of 128 tokens are dealt to the G splits in
 *                  equal contiguous runs over all sequences.
 *   workspace      device scratch, or NULL to query the size into
 *                  *workspace_bytes (in: capacity).  Layout (256-byte aligned
 *                  sections): header (int32 status, G, tile, kernel), query
 *                  buffers, then per split-partial slot s = split + b:
 *                  m[s][H], l[s][H] (float32, log2 domain), z[s][H][r].
 *   out            device, B x E, out_dtype: o, or the projected o W_O when
 *                  dims->out_proj is CHAIN or FOLD.
 *   phases         QSVD_PHASE_* mask (0 = all).  Running the phases as
 *                  separate calls in order gives the same result; so does
 *                  running the split as its two rotary passes
 *                  (QSVD_PHASE_SPLIT_SCORES, then QSVD_PHASE_SPLIT_ACCUM).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 */
qsvd_status qsvd_decode_attn(const qsvd_dims* dims, const void* packed,
                             const float* qin, int qin_is_latent,
                             const void* cache, const void* scales,
                             const int32_t* lengths, int num_splits,
                             void* workspace, size_t* workspace_bytes,
                             void* out, unsigned phases, void* stream);

/*
 * qsvd_combine_splits -- merge the split partials held in `workspace`
 * (written by the split phase of qsvd_decode_attn with the same dims,
 * lengths and num_splits) and apply the value up-projection: with M = max_s m_s,
 * w_s = 2^(m_s - M):  z = sum_s w_s z_s / sum_s w_s l_s,  o_h = z_h W^u_{v,h}.
 * Source: WSVD digest, Method 3.4 (flash decoding); QSVD digest, Step 1.
 * With dims->out_proj the output is o W_O (see QSVD_OUT_PROJ_*).
 * Equivalent to qsvd_decode_attn with phases = QSVD_PHASE_COMBINE.
 * The workspace's size is not passed: it must be the one the decode call
 * used, and num_splits must be that call's (the merge takes the split
 * count recorded in the workspace and the partials' offsets from
 * num_splits; with another value it reads other offsets, possibly past
 * the workspace).
 * Errors: INVALID_ARG, CUDA.
 */
qsvd_status qsvd_combine_splits(const qsvd_dims* dims, const void* packed,
                                void* workspace, int num_splits,
                                const int32_t* lengths, void* out, void* stream);

/*
 * qsvd_decode_attn_per_head -- decode-step attention over per-head latents
 * (WSVD digest, Method, per-head SVD §3.1, fused kernel §3.4).  Head h keeps
 * its own key latent C_{Kh} = X A_{Kh} and value latent C_{Vh} = X A_{Vh}
 * (L x r each; dims->r is the per-head rank) with W_{Kh} = A_{Kh} B_{Kh},
 * W_{Vh} = A_{Vh} B_{Vh}.  With tau = dims->softmax_scale (<= 0: 1/sqrt(d_h)):
 *   qt_h = tau B_{Kh} q_h,  s_t = C_{Kh,t} . qt_h,  p = softmax(s),
 *   o_h = (p^T C_{Vh}) B_{Vh}.
 * Computed in float32 on CUDA cores, 256 tokens per split CTA, chunks merged
 * in the log2 domain; 16-bit latents with r = 64, 128 or 256 are read as
 * 16-byte vectors.  With dims->rope (rotary mode; d_h == 128, r = 64 or
 * 128, H <= 59, an F16 or BF16 cache of the weight type): keys are rebuilt per
 * 128-token tile on the tensor cores, K_h = C_{Kh} B_{Kh}, rotated to their
 * positions and dotted with the query rotated to len_b - 1 (base
 * dims->rope_base; the cos/sin table of every position, from float64 angles,
 * is built in the workspace by each call).
 *   bk, bv     device, H x r x d_h each, weight_dtype (F32, F16 or BF16):
 *              B_{Kh} and B_{Vh} stacked by head.  With dims->out_proj ==
 *              QSVD_OUT_PROJ_FOLD (16-bit weights), bv is instead the fold
 *              F = [B_{V1} W_{O,1}; ..; B_{VH} W_{O,H}] (H r x E, from
 *              qsvd_prepare_per_head_fold) and out receives y = o W_O.
 *   q          device, B x E float32, 16-byte aligned: the query (head h
 *              in columns h d_h .. h d_h + d_h - 1).
 *   ck, cv     device, 16-byte aligned, cache_dtype (F32, F16 or BF16), in one of two
 *              layouts (rows 0 .. len_b - 1 of every head are read):
 *              QSVD_PER_HEAD_HEAD_MAJOR   B x H x max_len x r;
 *              QSVD_PER_HEAD_TOKEN_MAJOR  B x max_len x H x r: row t of a
 *              sequence holds every head's latent, so it is exactly the
 *              cache row that qsvd_prefill_latent / qsvd_append_latent write
 *              with W^d = [A_1 .. A_H] (E x H r) and rank H r.
 *   layout     QSVD_PER_HEAD_*.
 *   lengths    device, B int32; clamped to [0, max_len] and flagged
 *              (QSVD_STATUS_LEN_CLAMPED); len 0 gives a zero output row.
 *   workspace  device scratch, 16-byte aligned, or NULL to query the size
 *              into *workspace_bytes (in: capacity).  Its first int32 is the
 *              status word.
 *   out        device, B x E, out_dtype.
 * Stream-ordered; nothing is allocated.
 * Errors: INVALID_ARG (also an unknown layout), UNSUPPORTED (rotary mode
 * outside the shapes above, int caches, online H2, the chained output
 * projection, the fold with float32 weights, max_len beyond ~50 M tokens),
 * WORKSPACE, CUDA.
 */
#define QSVD_PER_HEAD_HEAD_MAJOR 0
#define QSVD_PER_HEAD_TOKEN_MAJOR 1
qsvd_status qsvd_decode_attn_per_head(const qsvd_dims* dims, const void* bk, const void* bv,
                                      const float* q, const void* ck, const void* cv,
                                      const int32_t* lengths, int layout, void* workspace,
                                      size_t* workspace_bytes, void* out, void* stream);

/*
 * qsvd_prepare_per_head_fold -- the per-head value factor folded into the
 * output projection (WSVD digest, Method, fused kernel §3.4):
 *   F[h r + j][n] = sum_i B_{Vh}[j][i] W_O[h d_h + i][n]
 * in float32, rounded once to weight_dtype.  With it the per-head decode
 * (dims->out_proj = QSVD_OUT_PROJ_FOLD) ends in one GEMV of the merged
 * latents (B x H r) by F instead of B_{Vh} then W_O.
 *   bv  device, H x r x d_h, weight_dtype (F16 or BF16).
 *   wo  device, E x E, weight_dtype (row h d_h + i multiplies channel i of
 *       head h).
 *   f   device, H r x E, weight_dtype (written).
 * Stream-ordered.  Errors: INVALID_ARG, UNSUPPORTED (float32 weights), CUDA.
 */
qsvd_status qsvd_prepare_per_head_fold(const qsvd_dims* dims, const void* bv, const void* wo, void* f,
                                       void* stream);

/* Human-readable name of a status code (static string). */
const char* qsvd_status_string(qsvd_status s);

/* Message describing the last failing call on this host thread. */
const char* qsvd_last_error(void);

/* Number of kernels this library has launched in this process. */
uint64_t qsvd_kernel_launches(void);

/* QSVD_ABI_VERSION of the loaded library. */
int qsvd_abi_version(void);

/*
 * qsvd_testing_set_score_wait_ns -- failure injection for tests (the pages
 * have no counterpart).  Every wait inside a kernel gives up after 2 s and
 * records QSVD_STATUS_TIMEOUT.  With ns != 0, the softmax warps of the
 * tensor-core split kernel (absorbed mode) begin their first tile by waiting
 * on a barrier that nothing releases, with a limit of ns nanoseconds: the
 * wait expires on every call, without any fault -- the kernel flags the
 * timeout, the other roles stop, wait (with the normal limit) for their
 * copies and MMAs in flight, free TMEM and return.  Applies to the current
 * device; ns = 0 turns it off.  Synchronous; for tests only.
 * Errors: CUDA.
 */
qsvd_status qsvd_testing_set_score_wait_ns(unsigned long long ns);

#ifdef __cplusplus
}
#endif

#endif /* QSVD_H */
