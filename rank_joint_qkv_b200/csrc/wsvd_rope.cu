// Per-head latents with rotary embedding (WSVD digest, Method §3.4: the
// fused kernel rebuilds each head's keys from its latent tile on chip and
// rotates them before the scores).  Head h: K_h[t] = C_{Kh}[t] B_{Kh}
// (r -> d_h), rotated to position t; the query q_h rotated to len - 1 and
// scaled by tau log2(e); s_t = q'_h . R(t) K_h[t].  Values stay in latent
// space (z_h = p^T C_{Vh}, o_h = z_h B_{Vh}) as in the absorbed mode.
//
// k_wsvd_rope_scores, one CTA per (128 tokens, sequence) walking the heads:
// per head the latent tile (128 x r, K-major) and B_{Kh} (r x d_h, read in
// place as the MN-major B operand) arrive by TMA (128-byte swizzle, two
// stages); one thread issues r / 16 tcgen05 MMAs (M = 128 tokens, N = d_h =
// 128, K = 16) into one of two TMEM buffers; every epilogue thread then takes
// its token's key row (TMEM lane = token), rotates the pairs (i, i + 64) with
// the fp64-built cos/sin row of its position (staged once for all heads) and
// dots it with the rotated query.  Both MMA operands are the stored 16-bit values,
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

// grid (ceil(max_len / 128), B), block kWrThreads.  R: per-head rank (64 or
// 128); d_h = 128.  One CTA walks every head of its 128 positions: warp 4 kWrG's
// first thread loads (TMA: the head's latent tile and B_{Kh}, a ring of
// wr_stages<R>() stages, so that several heads' tiles are in flight) and
// issues the MMAs into one of two TMEM buffers; kWrG groups of four warps
// (TMEM lanes 32 (w % 4) .., one token each) rotate and score, group g over
// its share of the 64 rotation pairs, their partial dots summed through
// shared memory; the positions' cos/sin rows are staged once in shared
// memory for all heads.  TMA maps: latent rows
// (head-major: 2D {r, rows}; token-major: 3D {r, H, B max_len} with a box one
// head high), B_K as 2D {d_h, H r}.
constexpr int kWrTab = 130;   // floats per staged table row (pitch: 2-way bank conflicts at most)
// Load stages: as many as fit beside the staged table (32 KB stages at r 64,
// 64 KB at r 128); a stage's loads wait in flight for about one load latency.
template <int R>
__host__ __device__ constexpr int wr_stages() { return R == 64 ? 4 : 2; }
// Scoring groups of four warps (one token per thread), each over 64 / kWrG
// of the rotation pairs; warp 4 kWrG issues the loads and MMAs.
constexpr int kWrG = 4;
constexpr int kWrThreads = 128 * kWrG + 32;
// Shared memory of one CTA: the dynamic part (1024 bytes of alignment slack,
// the load stages, the cos/sin rows, 128 bytes of barriers, every head's
// rotated query) plus the static partial dots; the sum must not exceed the
// per-block opt-in limit.
constexpr int kWrStaticBytes = (kWrG - 1) * 2 * 128 * 4;
inline int wr_dynamic_smem(int r, int H) {
  const int stages = r == 64 ? wr_stages<64>() : wr_stages<128>();
  return 1024 + stages * (128 * r * 2 + r * 128 * 2) + 128 * kWrTab * 4 + 128 + H * 128 * 4;
}
constexpr int kWrSmemLimit = 232448;   // opt-in shared memory per block on sm_100
template <bool BF16, int R>
__global__ void __launch_bounds__(kWrThreads, 1)
k_wsvd_rope_scores(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_b,
                   const float* __restrict__ qr, const float* __restrict__ tab,
                   const int32_t* __restrict__ lengths, float* __restrict__ scores,
                   int32_t* __restrict__ status, int H, int max_len, int token_major) {
  constexpr int D = 128, NB = R / 64, NST = wr_stages<R>();
  constexpr int CBYTES = 128 * R * 2, BBYTES = R * D * 2, STAGE = CBYTES + BBYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* tabs = reinterpret_cast<float*>(base + NST * STAGE);          // [128][kWrTab]
  uint64_t* bars = reinterpret_cast<uint64_t*>(tabs + 128 * kWrTab);
  uint64_t* full = bars;                // [NST] stage loaded
  uint64_t* empty = bars + NST;         // [NST] stage's MMAs done
  uint64_t* done = bars + 2 * NST;      // [2] TMEM buffer holds a head's keys
  uint64_t* tfree = done + 2;           // [2] TMEM buffer read by the epilogue
  uint64_t* drain = tfree + 2;          // the MMA thread's last commit
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  float* qsm = tabs + 128 * kWrTab + 32;   // [H][128] the rotated queries (after 128 bytes of barriers)
  __shared__ float ps[kWrG - 1][2][128];   // the other groups' partial dots, by TMEM buffer
  constexpr int MW = 4 * kWrG;             // the loading / MMA warp
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int len = min(max(lengths[b], 0), max_len);
  const int t0 = blockIdx.x * 128;
  if (t0 >= len) return;   // uniform across the CTA, before any barrier or TMEM use
  const uint32_t s0 = saddr(base);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(saddr(&full[i]), 1);
      mbar_init(saddr(&empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(saddr(&done[i]), 1);
      mbar_init(saddr(&tfree[i]), 1);
    }
    mbar_init(saddr(drain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == MW) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;" ::"r"(
                     saddr(tmem_holder))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    tc_fence_before();
  } else {
    if (warp < 4) {
      // this token's cos/sin row (64 pairs), staged once for every head
      const int p = t0 + threadIdx.x;
      const float4* src = reinterpret_cast<const float4*>(tab + size_t(p < max_len ? p : 0) * D);
      float* dst = tabs + threadIdx.x * kWrTab;
#pragma unroll 8
      for (int v = 0; v < D / 4; ++v) {
        const float4 x = __ldg(src + v);
        dst[4 * v] = x.x; dst[4 * v + 1] = x.y; dst[4 * v + 2] = x.z; dst[4 * v + 3] = x.w;
      }
    }
    // every head's rotated query of this sequence, read by all scoring threads
    const float* qb = qr + size_t(b) * H * D;
    for (int i = threadIdx.x; i < H * D; i += 128 * kWrG) qsm[i] = __ldg(qb + i);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == MW) {
    if (lane == 0) {
      constexpr uint32_t id = idesc_f16(128, D, BF16, false, true);   // B MN-major
      bool ok = true;
      int issued = 0;
      auto load = [&](int h) -> bool {
        const int st = h % NST;
        if (!mbar_wait(saddr(&empty[st]), (uint32_t(h / NST) & 1u) ^ 1u)) return false;
        const uint32_t dst = s0 + uint32_t(st * STAGE), fb = saddr(&full[st]);
        mbar_expect_tx(fb, uint32_t(STAGE));
#pragma unroll
        for (int kb = 0; kb < NB; ++kb) {
          if (token_major)
            tma_load_3d_hint(dst + kb * 128 * 128, &tm_c, 64 * kb, h, b * max_len + t0, fb, policy_evict_first());
          else
            tma_load_2d(dst + kb * 128 * 128, &tm_c, 64 * kb, (b * H + h) * max_len + t0, fb);
        }
        tma_load_2d(dst + CBYTES, &tm_b, 0, h * R, fb);
        tma_load_2d(dst + CBYTES + R * 128, &tm_b, 64, h * R, fb);
        ++issued;
        return true;
      };
      for (int x = 0; x < NST - 1 && x < H && ok; ++x) ok = load(x);   // NST - 1 heads ahead
      for (int h = 0; h < H && ok; ++h) {
        if (h + NST - 1 < H && !load(h + NST - 1)) { ok = false; break; }
        const int st = h % NST, tb = h & 1;   // load stage, TMEM buffer
        if (!mbar_wait(saddr(&full[st]), uint32_t(h / NST) & 1u)) { ok = false; break; }
        if (h >= 2 && !mbar_wait(saddr(&tfree[tb]), uint32_t((h - 2) >> 1) & 1u)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sb = s0 + uint32_t(st * STAGE);
#pragma unroll
        for (int kk = 0; kk < R / 16; ++kk) {   // K = 16 latent channels per MMA
          const uint64_t a = sdesc(sb + uint32_t((kk >> 2) * 128 * 128 + (kk & 3) * 32), 16, 1024);
          const uint64_t bd = sdesc(sb + CBYTES + uint32_t(kk * 16 * 128), R * 128, 1024);
          tc_mma(tmem + uint32_t(tb * D), a, bd, id, kk > 0 ? 1u : 0u);
        }
        tc_commit(saddr(&done[tb]));
        tc_commit(saddr(&empty[st]));
        if (*abort_flag) ok = false;
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(status, QSVD_STATUS_TIMEOUT);
        // every copy issued has landed before the CTA may leave
        for (int h = issued > NST ? issued - NST : 0; h < issued; ++h)
          mbar_wait(saddr(&full[h % NST]), uint32_t(h / NST) & 1u);
      }
      tc_commit(saddr(drain));   // every MMA issued has completed before TMEM is freed
      mbar_wait(saddr(drain), 0);
    }
    __syncwarp();
  } else {
    const int g = warp >> 2, t = threadIdx.x & 127, p = t0 + t;   // pair half, token
    const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
    const float* trow = tabs + t * kWrTab;
    for (int h = 0; h < H; ++h) {
      const int st = h & 1;
      // every group takes the same decision (one barrier over all their
      // threads), which also covers an abort flagged during the last head
      if (bar_or(*abort_flag || !mbar_wait(saddr(&done[st]), uint32_t(h >> 1) & 1u), 1 + kWrG, 128 * kWrG)) {
        if (threadIdx.x == 0) { *abort_flag = 1; atomicOr(status, QSVD_STATUS_TIMEOUT); }
        break;
      }
      tc_fence_after();
      const float* qh = qsm + h * D;
      const uint32_t ta = tmem + lane_off + uint32_t(st * D);
      float s = 0.f;
#pragma unroll 1
      for (int i0 = (64 / kWrG) * g; i0 < (64 / kWrG) * (g + 1); i0 += 16) {
        float klo[16], khi[16];
        tmem_ld16(ta + uint32_t(i0), klo);
        tmem_ld16(ta + uint32_t(64 + i0), khi);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int j = i0 + e;
          const float c = trow[2 * j], sn = trow[2 * j + 1];
          s = fmaf(qh[j], fmaf(klo[e], c, -khi[e] * sn), s);
          s = fmaf(qh[64 + j], fmaf(khi[e], c, klo[e] * sn), s);
        }
      }
      tc_fence_before();
      if (g > 0) ps[g - 1][st][t] = s;
      bar_sync(1 + kWrG, 128 * kWrG);   // every group's TMEM reads and partial dots are done
      if (threadIdx.x == 0) mbar_arrive(saddr(&tfree[st]));
      if (g == 0 && p < len) {
#pragma unroll
        for (int o = 0; o < kWrG - 1; ++o) s += ps[o][st][t];
        scores[(size_t(b) * H + h) * max_len + p] = s;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == MW) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem) : "memory");
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
  const int smem = wr_dynamic_smem(R, d.H);
  auto kern = k_wsvd_rope_scores<BF16, R>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3((d.max_len + 127) / 128, d.batch), kWrThreads, smem, s>>>(tc, tb, qr, tab, lengths, scores, status,
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
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool wsvd_rope_supported(const qsvd_dims& d) {
  return d.d_h == 128 && (d.cache_dtype == QSVD_F16 || d.cache_dtype == QSVD_BF16) &&
         d.weight_dtype == d.cache_dtype && (d.r == 64 || d.r == 128) &&   // a head's key rank is <= d_h
         // every head's rotated query is staged in shared memory: H <= 59
         wr_dynamic_smem(d.r, d.H) + kWrStaticBytes <= kWrSmemLimit;
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
