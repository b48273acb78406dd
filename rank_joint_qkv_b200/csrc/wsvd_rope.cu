// Per-head latents with rotary embedding (WSVD digest, Method §3.4: the
// fused kernel rebuilds each head's keys from its latent tile on chip and
// rotates them before the scores).  Head h: K_h[t] = C_{Kh}[t] B_{Kh}
// (r -> d_h), rotated to position t; the query q_h rotated to len - 1 and
// scaled by tau log2(e); s_t = q'_h . R(t) K_h[t].  Values stay in latent
// space (z_h = p^T C_{Vh}, o_h = z_h B_{Vh}) as in the absorbed mode.
//
// k_wsvd_rope_scores, one CTA per (128 tokens, head, sequence), 128 threads:
// the latent tile (128 x r, K-major) and B_{Kh} (r x d_h, read in place as the
// MN-major B operand) arrive by TMA (128-byte swizzle); one thread issues
// r / 16 tcgen05 MMAs (M = 128 tokens, N = d_h = 128, K = 16) into TMEM; every
// thread then takes its token's key row (TMEM lane = token), rotates the
// pairs (i, i + 64) with the fp64-built cos/sin row of its position and dots
// it with the rotated query.  Both MMA operands are the stored 16-bit values,
// so every product is exact and only the float32 accumulation rounds.  The
// scores ([B][H][max_len]) go to the chunk kernel of split_wsvd.cu, which
// runs the softmax and the value side.
#include <cuda.h>

#include <cstring>

#include "internal.cuh"
#include "tc_common.cuh"
#include "wsvd.cuh"

namespace qsvd {
namespace {

constexpr int kWrT = 128;   // threads (tokens) per scores CTA

// q'[b][h][i] = sl2 R(len_b - 1) q[b][h d + i], pairs (i, i + d/2).  grid (H, B).
__global__ void __launch_bounds__(128)
k_wsvd_rope_query(const float* __restrict__ q, const int32_t* __restrict__ lengths,
                  const float* __restrict__ tab, float* __restrict__ qr, int32_t* __restrict__ status,
                  int32_t* __restrict__ tickets, int n_tickets, int H, int d, int max_len, float sl2) {
  const int h = blockIdx.x, b = blockIdx.y;
  if (h == 0 && b == 0) {
    if (threadIdx.x == 0) *status = 0;   // the combine ORs flags in later
    for (int i = threadIdx.x; i < n_tickets; i += 128) tickets[i] = 0;
  }
  const int n = min(max(lengths[b], 0), max_len);
  const int pos = n > 0 ? n - 1 : 0;
  const int half = d / 2;
  const float* qh = q + (size_t(b) * H + h) * d;
  float* out = qr + (size_t(b) * H + h) * d;
  for (int k = threadIdx.x; k < half; k += 128) {
    const float a = qh[k], c = qh[k + half];
    const float cs = tab[(size_t(pos) * half + k) * 2], sn = tab[(size_t(pos) * half + k) * 2 + 1];
    out[k] = (a * cs - c * sn) * sl2;
    out[k + half] = (c * cs + a * sn) * sl2;
  }
}

// grid (ceil(max_len / 128), H, B), block 128.  R: per-head rank (64, 128 or
// 256); d_h = 128.  TMA maps: latent rows (head-major: 2D {r, rows}; token-
// major: 3D {r, H, B max_len} with a box one head high), B_K as 2D {d_h, H r}.
template <bool BF16, int R>
__global__ void __launch_bounds__(kWrT)
k_wsvd_rope_scores(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_b,
                   const float* __restrict__ qr, const float* __restrict__ tab,
                   const int32_t* __restrict__ lengths, float* __restrict__ scores,
                   int32_t* __restrict__ status, int H, int max_len, int token_major) {
  constexpr int D = 128, NB = R / 64;
  constexpr int CBYTES = 128 * R * 2, BBYTES = R * D * 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + CBYTES + BBYTES);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2);
  __shared__ float qs[D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int len = min(max(lengths[b], 0), max_len);
  const int t0 = blockIdx.x * 128;
  if (t0 >= len) return;   // uniform across the CTA, before any barrier or TMEM use
  const uint32_t s0 = saddr(base);
  const uint32_t full = saddr(&bars[0]), done = saddr(&bars[1]);
  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 128;" ::"r"(
                     saddr(tmem_holder))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    tc_fence_before();
  }
  for (int i = threadIdx.x; i < D; i += kWrT) qs[i] = qr[(size_t(b) * H + h) * D + i];
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  bool ok = true;
  if (threadIdx.x == 0) {
    mbar_expect_tx(full, uint32_t(CBYTES + BBYTES));
#pragma unroll
    for (int kb = 0; kb < NB; ++kb) {
      if (token_major)
        tma_load_3d_hint(s0 + kb * 128 * 128, &tm_c, 64 * kb, h, b * max_len + t0, full, policy_evict_first());
      else
        tma_load_2d(s0 + kb * 128 * 128, &tm_c, 64 * kb, (b * H + h) * max_len + t0, full);
    }
    tma_load_2d(s0 + CBYTES, &tm_b, 0, h * R, full);
    tma_load_2d(s0 + CBYTES + R * 128, &tm_b, 64, h * R, full);
    ok = mbar_wait(full, 0);
    if (ok) {
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(128, D, BF16, false, true);   // B MN-major
#pragma unroll
      for (int kk = 0; kk < R / 16; ++kk) {   // K = 16 latent channels per MMA
        const uint64_t a = sdesc(s0 + uint32_t((kk >> 2) * 128 * 128 + (kk & 3) * 32), 16, 1024);
        const uint64_t bd = sdesc(s0 + CBYTES + uint32_t(kk * 16 * 128), R * 128, 1024);
        tc_mma(tmem, a, bd, id, kk > 0 ? 1u : 0u);
      }
    }
    tc_commit(done);   // also when nothing was issued: the epilogue's wait completes
  }
  __syncwarp();
  const bool got = __syncthreads_and(mbar_wait(done, 0) && ok);
  if (!got) {
    if (threadIdx.x == 0) atomicOr(status, QSVD_STATUS_TIMEOUT);
  } else {
    tc_fence_after();
    const int t = threadIdx.x, p = t0 + t;
    const uint32_t ta = tmem + (uint32_t(32 * warp) << 16);
    const float* trow = tab + size_t(p < max_len ? p : 0) * D;   // (cos, sin) x 64
    float s = 0.f;
#pragma unroll 1
    for (int i0 = 0; i0 < 64; i0 += 16) {
      float klo[16], khi[16];
      tmem_ld16(ta + uint32_t(i0), klo);
      tmem_ld16(ta + uint32_t(64 + i0), khi);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int j = i0 + e;
        const float2 cs = *reinterpret_cast<const float2*>(trow + 2 * j);
        s = fmaf(qs[j], fmaf(klo[e], cs.x, -khi[e] * cs.y), s);
        s = fmaf(qs[64 + j], fmaf(khi[e], cs.x, klo[e] * cs.y), s);
      }
    }
    if (p < len) scores[(size_t(b) * H + h) * max_len + p] = s;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 128;" ::"r"(tmem) : "memory");
  }
}

template <bool BF16, int R>
cudaError_t scores_t(const qsvd_dims& d, const void* bk, const void* ck, const float* qr, const float* tab,
                     const int32_t* lengths, float* scores, int32_t* status, int token_major, cudaStream_t s) {
  TensorMapEncode enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt = BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap tc, tb;
  memset(&tc, 0, sizeof(tc));
  memset(&tb, 0, sizeof(tb));
  const size_t rows = size_t(d.batch) * d.max_len;
  if (token_major) {
    const cuuint64_t dims[3] = {cuuint64_t(R), cuuint64_t(d.H), cuuint64_t(rows)};
    const cuuint64_t strides[2] = {cuuint64_t(R) * 2, cuuint64_t(d.H) * R * 2};
    const cuuint32_t box[3] = {64, 1, 128};
    const cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tc, dt, 3, const_cast<void*>(ck), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    const cuuint64_t dims[2] = {cuuint64_t(R), cuuint64_t(rows * d.H)};
    const cuuint64_t strides[1] = {cuuint64_t(R) * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&tc, dt, 2, const_cast<void*>(ck), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {cuuint64_t(d.d_h), cuuint64_t(d.H) * R};
    const cuuint64_t strides[1] = {cuuint64_t(d.d_h) * 2};
    const cuuint32_t box[2] = {64, cuuint32_t(R)};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&tb, dt, 2, const_cast<void*>(bk), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const int smem = 1024 + 128 * R * 2 + R * 128 * 2 + 64;
  auto kern = k_wsvd_rope_scores<BF16, R>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3((d.max_len + 127) / 128, d.H, d.batch), kWrT, smem, s>>>(tc, tb, qr, tab, lengths, scores, status,
                                                                     d.H, d.max_len, token_major);
  note_launch();
  return check_launch();
}

template <bool BF16>
cudaError_t scores_r(const qsvd_dims& d, const void* bk, const void* ck, const float* qr, const float* tab,
                     const int32_t* lengths, float* scores, int32_t* status, int tm, cudaStream_t s) {
  switch (d.r) {
    case 64: return scores_t<BF16, 64>(d, bk, ck, qr, tab, lengths, scores, status, tm, s);
    case 128: return scores_t<BF16, 128>(d, bk, ck, qr, tab, lengths, scores, status, tm, s);
    case 256: return scores_t<BF16, 256>(d, bk, ck, qr, tab, lengths, scores, status, tm, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool wsvd_rope_supported(const qsvd_dims& d) {
  return d.d_h == 128 && (d.cache_dtype == QSVD_F16 || d.cache_dtype == QSVD_BF16) &&
         d.weight_dtype == d.cache_dtype && (d.r == 64 || d.r == 128 || d.r == 256);
}

cudaError_t launch_wsvd_rope_front(const qsvd_dims& d, const void* bk, const float* q, const void* ck,
                                   const int32_t* lengths, float sl2, void* workspace, const WsvdLayout& W,
                                   int token_major, cudaStream_t s) {
  uint8_t* wb = static_cast<uint8_t*>(workspace);
  float* tab = reinterpret_cast<float*>(wb + W.rope);
  cudaError_t e = launch_rope_table(tab, d.max_len, d.d_h, d.rope_base, s);
  if (e != cudaSuccess) return e;
  int32_t* status = reinterpret_cast<int32_t*>(wb + W.hdr);
  float* qr = reinterpret_cast<float*>(wb + W.qt);
  k_wsvd_rope_query<<<dim3(d.H, d.batch), 128, 0, s>>>(q, lengths, tab, qr, status,
                                                       reinterpret_cast<int32_t*>(wb + W.tickets), W.NT, d.H,
                                                       d.d_h, d.max_len, sl2);
  note_launch();
  if ((e = check_launch()) != cudaSuccess) return e;
  float* scores = reinterpret_cast<float*>(wb + W.scores);
  return d.cache_dtype == QSVD_BF16
             ? scores_r<true>(d, bk, ck, qr, tab, lengths, scores, status, token_major, s)
             : scores_r<false>(d, bk, ck, qr, tab, lengths, scores, status, token_major, s);
}

}  // namespace qsvd
