// Causal attention over a prompt whose latent rows are cached (prefill
// attention): queries, keys and values are rebuilt from the shared latent,
// Q = C W^u_q, K = C W^u_k, V = C W^u_v (QSVD digest, Method, Step 1: K and V
// are recomputed from the buffered latent; Key Contributions: the input is
// read once, into the latent), every query row attending to the rows at or
// before its own position, with optional rotary embedding of queries and keys
// at their positions (WSVD digest, Method §3.4).
//
// Three steps on the GPU:
//   1. Q, K, V: the latent-row GEMM of the prefill (tcgen05, prefill.cu) with
//      W^u_{q,k,v} as its weight and float32 rows out;
//   2. k_qkv_parts: rotary embedding of Q and K, then every value written as
//      two 16-bit parts, hi = rn(x) and lo = rn(x - hi) (rows past a prompt's
//      length become zeros);
//   3. k_prefill_attn: flash attention on tcgen05 per (128 queries, head,
//      prompt): S = Q_hi K_hi^T + Q_hi K_lo^T + Q_lo K_hi^T into TMEM, online
//      softmax in the log2 domain on CUDA cores (one query row per thread), P
//      as two 16-bit parts, O += P_hi V_hi + P_hi V_lo + P_lo V_hi into TMEM.
//
// The two-part operands are what the 2e-3 bar needs: one 16-bit part per
// operand puts the output 1e-2 (fp16) to 9e-2 (bf16) of rms away from the
// float64 definition on the oracle's own cases; two parts, 1e-4 .. 7e-4.
//
// Roles of k_prefill_attn (224 threads): warp 0 loads Q once and the key
// tiles, warp 2 the value tiles (TMA, 128-byte swizzle), warp 1 allocates TMEM
// and one of its threads issues every MMA, warps 3-6 run the softmax (warp w
// reads TMEM lanes 32 (w % 4) .. + 31: one query row per thread) and the
// epilogue.  Every wait is bounded as in the split kernels.
#include <cuda.h>

#include <cstring>

#include "internal.cuh"
#include "tc_common.cuh"

namespace qsvd {
namespace {

constexpr int kPaThreads = 224;
constexpr int kPaD = 128;                    // head dimension
constexpr int kPaBoxQ = 128 * 128;           // one 64-channel box of 128 rows, 16-bit
constexpr float kPaRescale = 8.f;            // P <= 2^8 before a rescale

// P enters the P V product as two 16-bit parts for both types: with fp16
// alone (one part) the rotary cases sit at the 2e-3 bar.
template <bool BF16>
struct PaCfg {
  static constexpr int BN = 64;                        // keys per tile
  static constexpr int PS = 2;                         // P parts (hi, lo)
  static constexpr int NST = 2;                        // stages of the key and value rings
  static constexpr int KVBox = BN * 128;               // one 64-channel box of BN rows
  static constexpr int KVStage = 4 * KVBox;            // hi and lo, two boxes each
  static constexpr int PPart = BN * 256;               // P part: BN / 64 boxes of 128 rows
  static constexpr int Q0 = 0;                         // Q hi, Q lo: 2 x 32 KB
  static constexpr int K0 = 4 * kPaBoxQ;
  static constexpr int V0 = K0 + NST * KVStage;
  static constexpr int P0 = V0 + NST * KVStage;
  static constexpr int BAR = P0 + PS * PPart;
  static constexpr int SMEM = 1024 + BAR + 256;
  static constexpr int SCOLS = BN;                     // TMEM columns of one S buffer
  static constexpr int OCOL = 2 * BN;                  // O accumulator (128 columns)
};
static_assert(PaCfg<false>::SMEM <= 227 * 1024 && PaCfg<true>::SMEM <= 227 * 1024, "shared memory");

// Q, K or V: rotary (queries and keys), then two 16-bit parts.  src [n][E]
// float32, row i = (b max_len + t); rows with t >= len_b are written as
// zeros.  grid (n), block 256: thread k handles pairs (k + 256 u) of the
// row, pair p = (h, i) -> channels h d + i and h d + i + d/2.
template <typename T>
__global__ void __launch_bounds__(256)
k_qkv_parts(const float* __restrict__ src, const int32_t* __restrict__ lengths,
            const float* __restrict__ rope_tab, int rope, T* __restrict__ hi, T* __restrict__ lo,
            int E, int d, int max_len) {
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  const size_t i = blockIdx.x;
  const int b = int(i / max_len), t = int(i % max_len);
  const int len = min(max(lengths[b], 0), max_len);
  const int half = d / 2;
  const float* row = src + i * E;
  T* hr = hi + i * E;
  T* lr = lo + i * E;
  for (int p = threadIdx.x; p < E / 2; p += 256) {
    const int h = p / half, k = p % half;
    const int e0 = h * d + k, e1 = e0 + half;
    float x0 = 0.f, x1 = 0.f;
    if (t < len) {
      x0 = row[e0];
      x1 = row[e1];
      if (rope) {
        const float cs = rope_tab[(size_t(t) * half + k) * 2];
        const float sn = rope_tab[(size_t(t) * half + k) * 2 + 1];
        const float y0 = x0 * cs - x1 * sn, y1 = x1 * cs + x0 * sn;
        x0 = y0;
        x1 = y1;
      }
    }
    const T h0 = dev::from_f<T>(x0), h1 = dev::from_f<T>(x1);
    hr[e0] = h0;
    hr[e1] = h1;
    lr[e0] = dev::from_f<T>(x0 - dev::to_f(h0));
    lr[e1] = dev::from_f<T>(x1 - dev::to_f(h1));
  }
}

// grid (ceil(max_len / 128), H, B): query tile qi = gridDim.x - 1 - blockIdx.x
// (the longest key ranges first).  Q/K/V parts [B max_len][E] 16-bit; out
// [B max_len][E] OT, rows t < len_b of head h's d columns.
template <bool BF16, typename OT>
__global__ void __launch_bounds__(kPaThreads, 1)
k_prefill_attn(const __grid_constant__ CUtensorMap tm_qh, const __grid_constant__ CUtensorMap tm_ql,
               const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_kl,
               const __grid_constant__ CUtensorMap tm_vh, const __grid_constant__ CUtensorMap tm_vl,
               const int32_t* __restrict__ lengths, OT* __restrict__ out, int32_t* __restrict__ status,
               int E, int max_len, float sl2) {
  using C = PaCfg<BF16>;
  constexpr int BN = C::BN, PS = C::PS, NST = C::NST;
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;            // [NST]
  uint64_t* k_empty = k_full + NST;       // [NST]
  uint64_t* v_full = k_empty + NST;       // [NST]
  uint64_t* v_empty = v_full + NST;       // [NST]
  uint64_t* s_full = v_empty + NST;       // [2]
  uint64_t* s_free = s_full + 2;          // [2]
  uint64_t* p_full = s_free + 2;
  uint64_t* o_done = p_full + 1;
  uint64_t* drain = o_done + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int qi = int(gridDim.x) - 1 - int(blockIdx.x);
  const int len = min(max(lengths[b], 0), max_len);
  const int q0 = qi * 128;
  if (q0 >= len) return;   // uniform across the CTA, before any barrier or TMEM use
  const int nk = (min(q0 + 128, len) + BN - 1) / BN;   // key tiles at or before the last query
  const int rb = b * max_len;                           // first row of the prompt
  const uint32_t s0 = saddr(base);

  if (threadIdx.x == 0) {
    mbar_init(saddr(q_full), 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(saddr(&k_full[i]), 1);
      mbar_init(saddr(&k_empty[i]), 1);
      mbar_init(saddr(&v_full[i]), 1);
      mbar_init(saddr(&v_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(saddr(&s_full[i]), 1);
      mbar_init(saddr(&s_free[i]), 1);
    }
    mbar_init(saddr(p_full), 1);
    mbar_init(saddr(o_done), 1);
    mbar_init(saddr(drain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     saddr(tmem_holder))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int col = h * kPaD;

  if (warp == 0 || warp == 2) {
    // ---------------------------------------------------------- producers
    const bool keys = warp == 0;
    bool ok = true;
    int issued = 0;
    if (lane == 0) {
      if (keys) {
        mbar_expect_tx(saddr(q_full), uint32_t(4 * kPaBoxQ));
        tma_load_2d(s0 + C::Q0, &tm_qh, col, rb + q0, saddr(q_full));
        tma_load_2d(s0 + C::Q0 + kPaBoxQ, &tm_qh, col + 64, rb + q0, saddr(q_full));
        tma_load_2d(s0 + C::Q0 + 2 * kPaBoxQ, &tm_ql, col, rb + q0, saddr(q_full));
        tma_load_2d(s0 + C::Q0 + 3 * kPaBoxQ, &tm_ql, col + 64, rb + q0, saddr(q_full));
      }
      uint64_t* full = keys ? k_full : v_full;
      uint64_t* empty = keys ? k_empty : v_empty;
      const CUtensorMap* th = keys ? &tm_kh : &tm_vh;
      const CUtensorMap* tl = keys ? &tm_kl : &tm_vl;
      const uint32_t ring = s0 + (keys ? C::K0 : C::V0);
      for (int j = 0; j < nk; ++j) {
        const int st = j % NST;
        if (!mbar_wait(saddr(&empty[st]), (uint32_t(j / NST) & 1u) ^ 1u)) { ok = false; break; }
        if (*abort_flag) { ok = false; break; }
        const uint32_t dst = ring + uint32_t(st * C::KVStage);
        const uint32_t fb = saddr(&full[st]);
        const int row = rb + j * BN;
        mbar_expect_tx(fb, uint32_t(C::KVStage));
        tma_load_2d(dst, th, col, row, fb);
        tma_load_2d(dst + C::KVBox, th, col + 64, row, fb);
        tma_load_2d(dst + 2 * C::KVBox, tl, col, row, fb);
        tma_load_2d(dst + 3 * C::KVBox, tl, col + 64, row, fb);
        ++issued;
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(status, QSVD_STATUS_TIMEOUT);
      }
      // every copy this warp issued has landed before the CTA may leave
      if (keys) mbar_wait(saddr(q_full), 0);
      for (int j = issued > NST ? issued - NST : 0; j < issued; ++j)
        mbar_wait(saddr(&full[j % NST]), uint32_t(j / NST) & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_f16(128, BN, BF16, false, false);
      constexpr uint32_t id_o = idesc_f16(128, kPaD, BF16, false, true);   // V: MN-major B
      const uint32_t qh = s0 + C::Q0, ql = qh + 2 * kPaBoxQ;
      bool ok = mbar_wait(saddr(q_full), 0);
      auto pv = [&](int i) -> bool {
        if (!mbar_wait(saddr(p_full), uint32_t(i) & 1u)) return false;
        if (!mbar_wait(saddr(&v_full[i % NST]), uint32_t(i / NST) & 1u)) return false;
        tc_fence_after();
        const uint32_t vh = s0 + C::V0 + uint32_t((i % NST) * C::KVStage), vl = vh + 2 * C::KVBox;
        int n = 0;
#pragma unroll
        for (int prod = 0; prod < (PS == 2 ? 3 : 2); ++prod) {
          const uint32_t pa = s0 + C::P0 + uint32_t((prod == 2 ? 1 : 0) * C::PPart);
          const uint32_t vb = prod == 1 ? vl : vh;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk, ++n) {   // K = 16 keys per MMA
            const uint64_t a = sdesc(pa + uint32_t((kk >> 2) * kPaBoxQ + (kk & 3) * 32), 16, 1024);
            const uint64_t bd = sdesc(vb + uint32_t(kk * 16 * 128), C::KVBox, 1024);
            tc_mma(tmem + uint32_t(C::OCOL), a, bd, id_o, (i > 0 || n > 0) ? 1u : 0u);
          }
        }
        tc_commit(saddr(o_done));
        tc_commit(saddr(&v_empty[i % NST]));
        return true;
      };
      for (int j = 0; j < nk && ok; ++j) {
        const int sb = j & 1;
        if (!mbar_wait(saddr(&k_full[j % NST]), uint32_t(j / NST) & 1u)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(saddr(&s_free[sb]), uint32_t((j - 2) >> 1) & 1u)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kh = s0 + C::K0 + uint32_t((j % NST) * C::KVStage), kl = kh + 2 * C::KVBox;
        int n = 0;
#pragma unroll
        for (int prod = 0; prod < 3; ++prod) {   // Q_hi K_hi, Q_hi K_lo, Q_lo K_hi
          const uint32_t qa = prod == 2 ? ql : qh, kb = prod == 1 ? kl : kh;
#pragma unroll
          for (int kk = 0; kk < kPaD / 16; ++kk, ++n) {   // K = 16 channels per MMA
            const uint32_t off = uint32_t((kk & 3) * 32);   // 16 channels = 32 bytes along a row
            const uint64_t a = sdesc(qa + uint32_t((kk >> 2) * kPaBoxQ) + off, 16, 1024);
            const uint64_t bd = sdesc(kb + uint32_t((kk >> 2) * C::KVBox) + off, 16, 1024);
            tc_mma(tmem + uint32_t(sb * C::SCOLS), a, bd, id_s, n > 0 ? 1u : 0u);
          }
        }
        tc_commit(saddr(&s_full[sb]));
        tc_commit(saddr(&k_empty[j % NST]));
        if (j >= 1 && !pv(j - 1)) ok = false;
        if (*abort_flag) ok = false;
      }
      if (ok) ok = pv(nk - 1);
      if (!ok) {
        *abort_flag = 1;
        atomicOr(status, QSVD_STATUS_TIMEOUT);
      }
      tc_commit(saddr(drain));
      mbar_wait(saddr(drain), 0);
    }
    __syncwarp();
  } else {
    // --------------------------------------------- softmax and epilogue
    const int t = 32 * (warp & 3) + lane;    // query row in the tile == TMEM lane
    const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
    const int qrow = q0 + t;                 // position of this query in the prompt
    float m_ref = -INFINITY, l = 0.f;
    bool failed = false;
    for (int j = 0; j < nk; ++j) {
      const int sb = j & 1;
      if (group_or(!mbar_wait(saddr(&s_full[sb]), uint32_t(j >> 1) & 1u))) { failed = true; break; }
      tc_fence_after();
      float sv[BN];
#pragma unroll
      for (int c = 0; c < BN / 16; ++c) tmem_ld16(tmem + lane_off + uint32_t(sb * C::SCOLS + 16 * c), sv + 16 * c);
      tmem_wait_ld();
      tc_fence_before();
      group_sync();
      if (t == 0) mbar_arrive(saddr(&s_free[sb]));
      const int k0 = j * BN;
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        const int kj = k0 + c;
        sv[c] = (kj <= qrow && kj < len) ? sv[c] * sl2 : -INFINITY;
        mt = fmaxf(mt, sv[c]);
      }
      const bool need = mt > m_ref + kPaRescale;   // also true on the first valid tile
      bool waited = false;
      if (__any_sync(0xffffffffu, need)) {
        const float mn = need ? mt : m_ref;
        const float alpha = need ? exp2f(m_ref - mn) : 1.f;   // 0 while no key was seen
        if (j > 0) {
          // the previous P V must be complete before O is rescaled (warp-uniform:
          // the TMEM accesses below are warp-collective)
          if (!__all_sync(0xffffffffu, mbar_wait(saddr(o_done), uint32_t(j - 1) & 1u))) failed = true;
          waited = true;
          if (!failed) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < kPaD / 16; ++c) {
              float o[16];
              const uint32_t ta = tmem + lane_off + uint32_t(C::OCOL + 16 * c);
              tmem_ld16(ta, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] *= alpha;
              tmem_st16(ta, o);
            }
            tmem_wait_st();
          }
        }
        l *= alpha;
        m_ref = mn;
      }
      if (group_or(failed)) { failed = true; break; }
      // P = 2^(s - m) as the A operand of P V: row t, keys K-major, 128B swizzle
      float ls = 0.f;
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        const float p = sv[c] == -INFINITY ? 0.f : exp2f(sv[c] - m_ref);
        sv[c] = p;
        ls += p;
      }
      l += ls;
      if (j > 0 && !waited && !mbar_wait(saddr(o_done), uint32_t(j - 1) & 1u)) failed = true;
      if (group_or(failed)) { failed = true; break; }
      uint8_t* prow = base + C::P0 + t * 128;
#pragma unroll
      for (int c8 = 0; c8 < BN / 8; ++c8) {
        const int box = c8 >> 3, chunk = c8 & 7;
        uint32_t w[4], wl[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = sv[8 * c8 + 2 * e], x1 = sv[8 * c8 + 2 * e + 1];
          if (BF16) {
            const __nv_bfloat162 hv = __floats2bfloat162_rn(x0, x1);
            w[e] = *reinterpret_cast<const uint32_t*>(&hv);
            const float2 hf = __bfloat1622float2(hv);
            const __nv_bfloat162 lv = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
            wl[e] = *reinterpret_cast<const uint32_t*>(&lv);
          } else {
            const __half2 hv = __floats2half2_rn(x0, x1);
            w[e] = *reinterpret_cast<const uint32_t*>(&hv);
            const float2 hf = __half22float2(hv);
            const __half2 lv = __floats2half2_rn(x0 - hf.x, x1 - hf.y);
            wl[e] = *reinterpret_cast<const uint32_t*>(&lv);
          }
        }
        uint8_t* dst = prow + box * kPaBoxQ + ((chunk ^ (t & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        if (PS == 2) *reinterpret_cast<uint4*>(dst + C::PPart) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
      }
      fence_proxy_async();   // generic-proxy stores -> visible to the tensor core
      tc_fence_before();
      group_sync();
      if (t == 0) mbar_arrive(saddr(p_full));
    }
    if (failed) {
      if (t == 0) {
        *abort_flag = 1;
        atomicOr(status, QSVD_STATUS_TIMEOUT);
      }
    } else if (!group_or(!mbar_wait(saddr(o_done), uint32_t(nk - 1) & 1u))) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      OT* orow = out + (size_t(rb) + qrow) * E + col;
#pragma unroll 1
      for (int c = 0; c < kPaD / 16; ++c) {
        float o[16];
        tmem_ld16(tmem + lane_off + uint32_t(C::OCOL + 16 * c), o);
        tmem_wait_ld();
        if (qrow < len) {
#pragma unroll
          for (int e = 0; e < 16; ++e) orow[16 * c + e] = dev::from_f<OT>(o[e] * inv);
        }
      }
    } else if (t == 0) {
      *abort_flag = 1;
      atomicOr(status, QSVD_STATUS_TIMEOUT);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

bool encode_rows(CUtensorMap* tm, bool bf16, const void* p, size_t rows, int E, int box_rows) {
  TensorMapEncode enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cuuint64_t(E), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(E) * 2};
  const cuuint32_t box[2] = {64, cuuint32_t(box_rows)};
  const cuuint32_t es[2] = {1, 1};
  memset(tm, 0, sizeof(*tm));
  return enc(tm, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
             const_cast<void*>(p), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool BF16, typename OT>
cudaError_t attn_t(const qsvd_dims& d, const PrefillAttnWs& w, const int32_t* lengths, void* out,
                   int32_t* status, float sl2, cudaStream_t s) {
  using C = PaCfg<BF16>;
  const size_t n = size_t(d.batch) * d.max_len;
  CUtensorMap tq[2], tk[2], tv[2];
  for (int p = 0; p < 2; ++p)
    if (!encode_rows(&tq[p], BF16, w.q[p], n, d.E, 128) || !encode_rows(&tk[p], BF16, w.k[p], n, d.E, C::BN) ||
        !encode_rows(&tv[p], BF16, w.v[p], n, d.E, C::BN))
      return cudaErrorInvalidValue;
  auto kern = k_prefill_attn<BF16, OT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const dim3 grid((d.max_len + 127) / 128, d.H, d.batch);
  {
    const cudaError_t le = launch_pdl(kern, grid, dim3(kPaThreads), size_t(C::SMEM), s, tq[0], tq[1], tk[0],
                                      tk[1], tv[0], tv[1], lengths, static_cast<OT*>(out), status, d.E,
                                      d.max_len, sl2);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return check_launch();
}

template <bool BF16>
cudaError_t attn_ot(const qsvd_dims& d, const PrefillAttnWs& w, const int32_t* lengths, void* out,
                    int32_t* status, float sl2, cudaStream_t s) {
  switch (d.out_dtype) {
    case QSVD_F32: return attn_t<BF16, float>(d, w, lengths, out, status, sl2, s);
    case QSVD_F16: return attn_t<BF16, __half>(d, w, lengths, out, status, sl2, s);
    case QSVD_BF16: return attn_t<BF16, __nv_bfloat16>(d, w, lengths, out, status, sl2, s);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T>
cudaError_t parts_t(const qsvd_dims& d, const float* src, const int32_t* lengths, const float* rope_tab,
                    int rope, void* hi, void* lo, cudaStream_t s) {
  const unsigned n = unsigned(size_t(d.batch) * d.max_len);
  const cudaError_t le = launch_pdl(k_qkv_parts<T>, dim3(n), dim3(256), 0, s, src, lengths, rope_tab, rope,
                                    static_cast<T*>(hi), static_cast<T*>(lo), d.E, d.d_h, d.max_len);
  if (le != cudaSuccess) return le;
  note_launch();
  return check_launch();
}

}  // namespace

bool prefill_attention_supported(const qsvd_dims& d) {
  return d.d_h == kPaD && (d.cache_dtype == QSVD_F16 || d.cache_dtype == QSVD_BF16) &&
         d.weight_dtype == d.cache_dtype && d.E % 256 == 0 && d.r % 64 == 0;
}

PrefillAttnWs prefill_attention_ws(const qsvd_dims& d, void* workspace) {
  PrefillAttnWs w{};
  const size_t n = size_t(d.batch) * d.max_len;
  size_t o = 0;
  uint8_t* p = static_cast<uint8_t*>(workspace);
  w.stage = reinterpret_cast<float*>(p ? p + o : nullptr);
  o = align256(o + n * d.E * 4);
  void** parts[6] = {&w.q[0], &w.q[1], &w.k[0], &w.k[1], &w.v[0], &w.v[1]};
  for (void** q : parts) {
    *q = p ? p + o : nullptr;
    o = align256(o + n * d.E * 2);
  }
  w.total = o;
  return w;
}

cudaError_t launch_prefill_attention(const qsvd_dims& d, const void* wuq, const void* wuk, const void* wuv,
                                     const float* rope_tab, const void* cache, const int32_t* lengths,
                                     const PrefillAttnWs& w, void* out, int32_t* status, float sl2,
                                     cudaStream_t s) {
  // Q, K, V = C W^u_{q,k,v}: the prefill GEMM with K = r, N = E, float32 rows
  qsvd_dims g = d;
  g.E = d.r;
  g.r = d.E;
  g.cache_dtype = QSVD_F32;
  g.h2 = 0;
  const int n = d.batch * d.max_len;
  const void* ws[3] = {wuq, wuk, wuv};
  void* const* dst[3] = {w.q, w.k, w.v};
  const bool bf = d.cache_dtype == QSVD_BF16;
  for (int m = 0; m < 3; ++m) {
    cudaError_t e = launch_prefill(g, ws[m], cache, n, nullptr, w.stage, nullptr, nullptr, status, s);
    if (e != cudaSuccess) return e;
    const int rope = d.rope && m < 2;
    e = bf ? parts_t<__nv_bfloat16>(d, w.stage, lengths, rope_tab, rope, dst[m][0], dst[m][1], s)
           : parts_t<__half>(d, w.stage, lengths, rope_tab, rope, dst[m][0], dst[m][1], s);
    if (e != cudaSuccess) return e;
  }
  return bf ? attn_ot<true>(d, w, lengths, out, status, sl2, s) : attn_ot<false>(d, w, lengths, out, status, sl2, s);
}

}  // namespace qsvd
