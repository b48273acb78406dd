// Prologue of a decode step: the query side.
//
//   q   = c_new W^u_q                      (QSVD digest, Method, Step 1: Q is
//                                            rebuilt from the shared latent)
//   qt_h = (tau * log2 e) W^u_{k,h} q_h    (no rotary embedding: the query is
//                                            absorbed into latent space so the
//                                            scores are C qt_h)
//   q_h <- (tau * log2 e) R(len-1) q_h     (rotary mode: WSVD digest, Method
//                                            3.4, rotary keys; the query is
//                                            rotated at its own position)
//
// These read W^u_q and W^u_k once per step (batched GEMVs, HBM-bound on the
// weights) and are small next to the split phase.
#include "internal.cuh"
#include "gemv.cuh"

namespace qsvd {
namespace {

using dev::to_f;

// ---------------------------------------------------------------------------
// qt[b][h][j] = scale * sum_d W^u_k[j][h*d_h + d] * q[b][h*d_h + d]
// grid (H, ceil(r/128)), block 128.  A thread computes 4 rows x 4 sequences.
// ---------------------------------------------------------------------------
template <typename WT, typename QT16>
__global__ void __launch_bounds__(128)
k_absorb(const float* __restrict__ q, const WT* __restrict__ W, float scale,
         float* __restrict__ qt32, QT16* __restrict__ qt16, int B, int H, int d_h, int r,
         int E) {
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  extern __shared__ float sm[];
  const int h = blockIdx.x;
  const int j0 = blockIdx.y * 128;
  const int jn = min(128, r - j0);
  const int ld = d_h + 4;                  // padded row stride (floats)
  float* ws = sm;                          // [128][ld]
  float* qs = sm + 128 * ld;               // [32][ld]
  // stage the W^u_k tile (rows j0.., columns of head h) as float, 16-byte loads
  {
    constexpr int V = 16 / int(sizeof(WT));
    const int vpr = d_h / V;
    for (int i = threadIdx.x; i < 128 * vpr; i += 128) {
      const int jr = i / vpr, v = i % vpr;
      float f[V];
      if (jr < jn) {
        const uint4 raw = *reinterpret_cast<const uint4*>(W + size_t(j0 + jr) * E + h * d_h + v * V);
        const WT* e = reinterpret_cast<const WT*>(&raw);
#pragma unroll
        for (int k = 0; k < V; ++k) f[k] = to_f(e[k]);
      } else {
#pragma unroll
        for (int k = 0; k < V; ++k) f[k] = 0.f;
      }
#pragma unroll
      for (int k = 0; k < V; ++k) ws[jr * ld + v * V + k] = f[k];
    }
  }
  const int tr = threadIdx.x / 4;    // rows tr + 32a, a < 4 (conflict-free float4 reads)
  const int tb = threadIdx.x % 4;    // sequences b0 + tb + 4c, c < 4
  for (int b0 = 0; b0 < B; b0 += 16) {
    __syncthreads();
    for (int i = threadIdx.x; i < 16 * (d_h / 4); i += 128) {
      const int bb = i / (d_h / 4), d = 4 * (i % (d_h / 4));
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (b0 + bb < B) v = *reinterpret_cast<const float4*>(q + size_t(b0 + bb) * E + h * d_h + d);
      *reinterpret_cast<float4*>(&qs[bb * ld + d]) = v;
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
    for (int d = 0; d < d_h; d += 4) {
      float4 wv[4], qv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) wv[a] = *reinterpret_cast<const float4*>(&ws[(tr + 32 * a) * ld + d]);
#pragma unroll
      for (int c = 0; c < 4; ++c) qv[c] = *reinterpret_cast<const float4*>(&qs[(tb + 4 * c) * ld + d]);
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          acc[a][c] = fmaf(wv[a].x, qv[c].x, acc[a][c]);
          acc[a][c] = fmaf(wv[a].y, qv[c].y, acc[a][c]);
          acc[a][c] = fmaf(wv[a].z, qv[c].z, acc[a][c]);
          acc[a][c] = fmaf(wv[a].w, qv[c].w, acc[a][c]);
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int j = j0 + tr + 32 * a, b = b0 + tb + 4 * c;
        if (j - j0 < jn && b < B) {
          const float v = acc[a][c] * scale;
          const size_t o = (size_t(b) * H + h) * r + j;
          if (qt32) qt32[o] = v;
          if (qt16) {
            // 16-bit copy for the tensor cores, [B][2][H][r]: the rounded value
            // and its rounding residual (hi + lo carries ~2x the mantissa bits;
            // one 16-bit part alone perturbs peaked softmaxes by ~1e-2)
            const QT16 hi = dev::from_f<QT16>(v);
            const size_t o2 = ((size_t(b) * 2) * H + h) * r + j;
            qt16[o2] = hi;
            qt16[o2 + size_t(H) * r] = dev::from_f<QT16>(v - dev::to_f(hi));
          }
        }
      }
  }
}

// ---------------------------------------------------------------------------
// Absorbed query on the tensor cores, for 16-bit weights and d_h a multiple
// of 64:  qt[b][h][j] = scale * sum_dd q[b][h d_h + dd] W^u_k[j][h d_h + dd].
// Per head a 16-row product (M = 16 sequences, N = 128 rows j of W^u_k per
// CTA, K = d_h), so it takes the GEMV's form: the W^u_k tile arrives by TMA
// into 128-byte-swizzled rows whose d_h values are K-contiguous (ldmatrix
// gives the B fragments directly), q enters as a 16-bit part plus its
// rounding residual, with fp16 weights scaled per sequence by a power of two.
// grid (H, ceil(r / 128)), block 128.
// ---------------------------------------------------------------------------
template <typename WT, typename QT16>
__global__ void __launch_bounds__(128)
k_absorb_mma(const __grid_constant__ CUtensorMap tm_w, const float* __restrict__ q, float scale,
             float* __restrict__ qt32, QT16* __restrict__ qt16, int B, int H, int d_h, int r, int E,
             int32_t* status) {
  using namespace gemv_mma;
  constexpr bool BF16 = std::is_same<WT, __nv_bfloat16>::value;
  constexpr bool SCALE = !BF16;           // fp16 range needs the power-of-two scale
  extern __shared__ uint8_t asm_raw[];
  uint8_t* tile = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(asm_raw) + 1023) &
                                             ~uintptr_t(1023));   // [d_h / 64][128 rows][128 B]
  const int XP = d_h * 2 + 16;            // activation row pitch (bytes, padded)
  uint8_t* xs = tile + d_h * 256;         // [2][16][XP]
  __shared__ __align__(8) uint64_t bar;
  __shared__ float inv_scale[16];
  __shared__ unsigned smax[16];
  const int h = blockIdx.x, j0 = blockIdx.y * 128, jn = min(128, r - j0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t tile_s = static_cast<uint32_t>(__cvta_generic_to_shared(tile));
  const uint32_t bar_s = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
  const int NBOX = d_h / 64;
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_s) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_s),
                 "r"(uint32_t(d_h * 256)) : "memory");
    for (int c = 0; c < NBOX; ++c)
      asm volatile(
          "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
          " [%0], [%1, {%2, %3}], [%4];" ::"r"(tile_s + c * 16384),
          "l"(reinterpret_cast<uint64_t>(&tm_w)), "r"(h * d_h + 64 * c), "r"(j0), "r"(bar_s)
          : "memory");
  }
  // the weight tile is in flight; what follows reads what earlier kernels wrote
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  const int mrow = (lane & 7) + 8 * ((lane >> 3) & 1);   // ldmatrix: this lane's row of its 8x8 matrix
  const int mcol = 8 * (lane >> 4);
  const uint32_t xs_s = static_cast<uint32_t>(__cvta_generic_to_shared(xs));
  bool waited = false;
  for (int b0 = 0; b0 < B; b0 += 16) {
    const int bn = min(16, B - b0);
    // q slice of head h: thread tid holds dd = tid + 128 u of every sequence
    float xv[16][2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int dd = tid + 128 * u;
      const int ddc = dd < d_h ? dd : 0;   // clamped: the loads stay unconditional
#pragma unroll
      for (int j = 0; j < 16; ++j)
        xv[j][u] = __ldg(q + size_t(b0 + (j < bn ? j : 0)) * E + h * d_h + ddc);
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (!(j < bn && dd < d_h)) xv[j][u] = 0.f;
    }
    if (SCALE) {
      if (tid < 16) smax[tid] = 0u;
      float m[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) m[j] = fmaxf(fabsf(xv[j][0]), fabsf(xv[j][1]));
      const float wm = dev::warp_reduce_transposed<16>(m, lane, dev::OpMax());   // lane L: sequence L % 16
      __syncthreads();
      if (lane < 16) atomicMax(&smax[lane], __float_as_uint(wm));   // non-negative floats order as integers
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float s = 1.f, inv = 1.f;
      if (SCALE) {
        const unsigned mb = smax[j];
        if (mb != 0u) {
          const int e = max(int((mb >> 23) & 0xFFu) - 127, -112);
          s = __uint_as_float(unsigned(141 - e) << 23);
          inv = __uint_as_float(unsigned(113 + e) << 23);
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int dd = tid + 128 * u;
        if (dd < d_h) {
          const float v = xv[j][u] * s;
          const WT hi = dev::from_f<WT>(v);
          reinterpret_cast<WT*>(xs + j * XP)[dd] = hi;
          reinterpret_cast<WT*>(xs + (16 + j) * XP)[dd] = dev::from_f<WT>(v - dev::to_f(hi));
        }
      }
      if (tid == 0) inv_scale[j] = inv;
    }
    if (!waited) {   // the W^u_k tile (bounded wait: 2 s; on expiry flag it and stop)
      bool ok = mbar_try(bar_s, 0);
      if (!ok) {
        const uint64_t t0 = gtimer();
        while (!(ok = mbar_try(bar_s, 0)))
          if (gtimer() - t0 > 2000000000ull) break;
      }
      if (!__syncthreads_and(ok)) {
        if (tid == 0 && status) atomicOr(status, QSVD_STATUS_TIMEOUT);
        return;
      }
      waited = true;
    } else {
      __syncthreads();
    }
    // warp w: rows j 32 w .. 32 w + 31 (4 n-tiles), k over d_h
    float acc[4][4];
#pragma unroll
    for (int t = 0; t < 4; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
    for (int kk = 0; kk < d_h / 16; ++kk) {
      uint32_t a[2][4];
#pragma unroll
      for (int p = 0; p < 2; ++p) ldsm_x4(xs_s + (p * 16 + mrow) * XP + (16 * kk + mcol) * 2, a[p]);
      const int dd = 16 * kk + 8 * ((lane >> 3) & 1);
      const int c = dd >> 6, chunk = (dd & 63) >> 3;
#pragma unroll
      for (int jp = 0; jp < 2; ++jp) {
        const int j = 32 * warp + 8 * (2 * jp + (lane >> 4)) + (lane & 7);
        uint32_t bfr[4];   // n-tile 2 jp: k lo, k hi; n-tile 2 jp + 1: k lo, k hi
        ldsm_x4(tile_s + c * 16384 + j * 128 + ((chunk ^ (j & 7)) << 4), bfr);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          mma16816<BF16>(acc[2 * jp], a[p], bfr[0], bfr[1]);
          mma16816<BF16>(acc[2 * jp + 1], a[p], bfr[2], bfr[3]);
        }
      }
    }
    // fragment: (row g = sequence, cols 2t, 2t+1 = rows j) and (row g + 8)
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int jl = 32 * warp + 8 * t + 2 * t4;
      if (jl >= jn) continue;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int bb = g + 8 * half;
        if (bb >= bn) continue;
        const int b = b0 + bb;
        const float sc = scale * inv_scale[bb];
        const float v0 = acc[t][2 * half] * sc, v1 = acc[t][2 * half + 1] * sc;
        const size_t o = (size_t(b) * H + h) * r + j0 + jl;
        if (qt32) *reinterpret_cast<float2*>(qt32 + o) = make_float2(v0, v1);
        if (!qt16) continue;
        // 16-bit copy for the tensor cores, [B][2][H][r]: the rounded value
        // and its rounding residual
        const QT16 h0 = dev::from_f<QT16>(v0), h1 = dev::from_f<QT16>(v1);
        const QT16 l0 = dev::from_f<QT16>(v0 - dev::to_f(h0)), l1 = dev::from_f<QT16>(v1 - dev::to_f(h1));
        const size_t o2 = ((size_t(b) * 2) * H + h) * r + j0 + jl;
        QT16 hv[2] = {h0, h1}, lv[2] = {l0, l1};
        *reinterpret_cast<uint32_t*>(qt16 + o2) = *reinterpret_cast<const uint32_t*>(hv);
        *reinterpret_cast<uint32_t*>(qt16 + o2 + size_t(H) * r) = *reinterpret_cast<const uint32_t*>(lv);
      }
    }
    __syncthreads();   // xs is restaged for the next 16 sequences
  }
}

// ---------------------------------------------------------------------------
// Quantised latents on the tensor cores: the absorbed query of each
// (sequence, head) as three int8 parts with one power-of-two scale,
//   qt = s (Q0 + Q1 / 128 + Q2 / 16384),  s = 2^ceil(log2(max_j |qt_j| / 127)),
// Q0 = rint(qt / s) (|Q0| <= 127), Q1 = rint(128 (qt - s Q0) / s), Q2 likewise
// (|Q1|, |Q2| <= 64; remainder <= s / 32768): the integer MMAs of the split
// kernel take the parts, the softmax applies s once per head.  qp [B][3][H][r]
// int8, qs [B][H].  grid (H, B), block 128.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
k_quant_query(const float* __restrict__ qt, int8_t* __restrict__ qp, float* __restrict__ qs, int H, int r) {
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  __shared__ float red[4];
  const int h = blockIdx.x, b = blockIdx.y;
  const float* row = qt + (size_t(b) * H + h) * r;
  float m = 0.f;
  for (int j = threadIdx.x; j < r; j += 128) m = fmaxf(m, fabsf(row[j]));
  m = dev::warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  // the smallest power of two >= m / 127 (1 for an all-zero query)
  const float f = m / 127.f;
  const float sq = f > 0.f ? __uint_as_float((__float_as_uint(f) + 0x007FFFFFu) & 0xFF800000u) : 1.f;
  const float isq = 1.f / sq;   // exact: a power of two
  if (threadIdx.x == 0) qs[size_t(b) * H + h] = sq;
  int8_t* p0 = qp + ((size_t(b) * 3 + 0) * H + h) * r;
  int8_t* p1 = qp + ((size_t(b) * 3 + 1) * H + h) * r;
  int8_t* p2 = qp + ((size_t(b) * 3 + 2) * H + h) * r;
  for (int j = threadIdx.x; j < r; j += 128) {
    const float v = row[j];
    const float q0 = rintf(v * isq);
    const float r1 = v - sq * q0;
    const float q1 = rintf(r1 * isq * 128.f);
    const float r2 = r1 - sq * (1.f / 128.f) * q1;
    const float q2 = rintf(r2 * isq * 16384.f);
    p0[j] = int8_t(q0);
    p1[j] = int8_t(q1);
    p2[j] = int8_t(q2);
  }
}

// ---------------------------------------------------------------------------
// Rotary query: q_h <- scale * R(len_b - 1) q_h, pairs (i, i + d_h/2).
// grid (B), block 256.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
k_rope_query(const float* __restrict__ q, const int32_t* __restrict__ sched,
             const float* __restrict__ tab, float scale, float* __restrict__ qrot, int B,
             int H, int d_h, int E) {
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  const int b = blockIdx.x;
  const int n = sched[B + 1 + b];
  const int pos = n > 0 ? n - 1 : 0;
  const int half = d_h / 2;
  for (int i = threadIdx.x; i < H * half; i += blockDim.x) {
    const int h = i / half, k = i % half;
    const int e0 = h * d_h + k, e1 = e0 + half;
    const float a = q[size_t(b) * E + e0];
    const float c = q[size_t(b) * E + e1];
    const float cs = tab[(size_t(pos) * half + k) * 2 + 0];
    const float sn = tab[(size_t(pos) * half + k) * 2 + 1];
    qrot[size_t(b) * E + e0] = (a * cs - c * sn) * scale;
    qrot[size_t(b) * E + e1] = (c * cs + a * sn) * scale;
  }
}

// ---------------------------------------------------------------------------
// Split-KV schedule: clamped lengths and the tile prefix over sequences.
// sched[0..B] = tiles before sequence b (sched[B] = total), sched[B+1+b] = len.
// grid 1, block 32 .. 1024 (a multiple of 32).  Also records G in the workspace header.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024)
k_schedule(const int32_t* __restrict__ lengths, int B, int max_len, int G,
           int32_t* __restrict__ sched, WsHeader* hdr, int kernel,
           int32_t* __restrict__ tickets, int n_tickets) {
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  for (int i = threadIdx.x; i < n_tickets; i += blockDim.x) tickets[i] = 0;
  __shared__ int32_t wsum[32];
  __shared__ int32_t carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (threadIdx.x == 0) {
    carry = 0;
    hdr->status = 0;   // reset before any thread flags a clamped length
    hdr->G = G;
    hdr->tile = kTile;
    hdr->kernel = kernel;
  }
  __syncthreads();
  for (int b0 = 0; b0 < B; b0 += blockDim.x) {
    const int b = b0 + threadIdx.x;
    int nt = 0;
    if (b < B) {
      const int n = dev::clamp_len(lengths[b], max_len, &hdr->status);
      sched[B + 1 + b] = n;
      nt = dev::tiles_of(n);
    }
    // inclusive scan: within each warp by shuffles, then over the warp totals
    int v = nt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (lane == 31) wsum[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int t = lane < nw ? wsum[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += u;
      }
      if (lane < nw) wsum[lane] = t;
    }
    __syncthreads();
    const int incl = v + (warp > 0 ? wsum[warp - 1] : 0);
    if (b < B) sched[b + 1] = carry + incl;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry += incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) sched[0] = 0;
}

template <typename WT>
cudaError_t q_partial_t(const qsvd_dims& d, const float* qin, const void* wuq, float* qpart,
                        int KS, float* q, int32_t* tickets, int32_t* status, cudaStream_t s) {
  return launch_gemv<float, WT>(qin, static_cast<const WT*>(wuq), qpart, d.batch, d.r, d.E, KS, q,
                                tickets, status, s);
}

template <typename WT, typename QT16>
cudaError_t absorb_t(const qsvd_dims& d, const float* q, const void* wuk, float scale,
                     float* qt32, void* qt16, int32_t* status, cudaStream_t s) {
  if constexpr (sizeof(WT) == 2) {
    if (d.d_h % 64 == 0 && d.d_h <= 256) {
      TensorMapEncode enc = tensor_map_encoder();
      if (!enc) return cudaErrorNotSupported;
      CUtensorMap tm;
      const cuuint64_t dims[2] = {cuuint64_t(d.E), cuuint64_t(d.r)};
      const cuuint64_t strides[1] = {cuuint64_t(d.E) * 2};
      const cuuint32_t box[2] = {64, 128};
      const cuuint32_t es[2] = {1, 1};
      const CUtensorMapDataType dt = std::is_same<WT, __nv_bfloat16>::value
                                         ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
      if (enc(&tm, dt, 2, const_cast<void*>(wuk), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
      const int smem = 1024 + d.d_h * 256 + 2 * 16 * (d.d_h * 2 + 16);
      auto kern = k_absorb_mma<WT, QT16>;
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      dim3 grid(d.H, (d.r + 127) / 128);
      {
        const cudaError_t le = launch_pdl(kern, dim3(grid), dim3(128), smem, s,
                                         tm, q, scale, qt32, static_cast<QT16*>(qt16), d.batch, d.H, d.d_h, d.r, d.E, status);
        if (le != cudaSuccess) return le;
      }
      note_launch();
      return check_launch();
    }
  }
  const size_t smem = size_t(128 + 16) * (d.d_h + 4) * 4;
  auto kern = k_absorb<WT, QT16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(d.H, (d.r + 127) / 128);
  {
    const cudaError_t le = launch_pdl(kern, dim3(grid), dim3(128), smem, s,
                                     q, static_cast<const WT*>(wuk), scale, qt32, static_cast<QT16*>(qt16), d.batch, d.H, d.d_h, d.r, d.E);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return check_launch();
}

}  // namespace

int prologue_ksplit(const qsvd_dims& d) { return gemv_ksplit(d.r, d.weight_dtype); }
int prologue_tickets(const qsvd_dims& d) { return gemv_tickets(d.E, d.batch, d.weight_dtype); }
int gemv_tickets_vup(const qsvd_dims& d) { return gemv_tickets(d.E, d.batch, d.weight_dtype); }

cudaError_t launch_schedule(const qsvd_dims& d, const int32_t* lengths, int G, int32_t* sched,
                            WsHeader* hdr, int kernel, int32_t* tickets, int n_tickets,
                            cudaStream_t s) {
  {
    const int threads = d.batch <= 1024 ? (d.batch + 31) / 32 * 32 : 1024;   // a warp for small batches
    const cudaError_t le = launch_pdl(k_schedule, dim3(1), dim3(threads), 0, s,
                                     lengths, d.batch, d.max_len, G, sched, hdr, kernel, tickets, n_tickets);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return check_launch();
}

cudaError_t launch_q_partial(const qsvd_dims& d, const float* qin, const void* wuq,
                             float* qpart, int KS, float* q, int32_t* tickets, int32_t* status,
                             cudaStream_t s) {
  switch (d.weight_dtype) {
    case QSVD_F32: return q_partial_t<float>(d, qin, wuq, qpart, KS, q, tickets, status, s);
    case QSVD_F16: return q_partial_t<__half>(d, qin, wuq, qpart, KS, q, tickets, status, s);
    case QSVD_BF16: return q_partial_t<__nv_bfloat16>(d, qin, wuq, qpart, KS, q, tickets, status, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_absorb(const qsvd_dims& d, const float* q, const void* wuk, float scale,
                          float* qt32, void* qt16, int32_t* status, cudaStream_t s) {
  const bool bf = d.cache_dtype == QSVD_BF16;
  switch (d.weight_dtype) {
    case QSVD_F32:
      return bf ? absorb_t<float, __nv_bfloat16>(d, q, wuk, scale, qt32, qt16, status, s)
                : absorb_t<float, __half>(d, q, wuk, scale, qt32, qt16, status, s);
    case QSVD_F16:
      return bf ? absorb_t<__half, __nv_bfloat16>(d, q, wuk, scale, qt32, qt16, status, s)
                : absorb_t<__half, __half>(d, q, wuk, scale, qt32, qt16, status, s);
    case QSVD_BF16:
      return bf ? absorb_t<__nv_bfloat16, __nv_bfloat16>(d, q, wuk, scale, qt32, qt16, status, s)
                : absorb_t<__nv_bfloat16, __half>(d, q, wuk, scale, qt32, qt16, status, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_quant_query(const qsvd_dims& d, const float* qt, int8_t* qp, float* qs, cudaStream_t s) {
  {
    const cudaError_t le = launch_pdl(k_quant_query, dim3(d.H, d.batch), dim3(128), 0, s, qt, qp, qs, d.H, d.r);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return check_launch();
}

cudaError_t launch_rope_query(const qsvd_dims& d, const float* q, const int32_t* sched,
                              const float* rope_tab, float scale, float* qrot,
                              cudaStream_t s) {
  {
    const cudaError_t le = launch_pdl(k_rope_query, dim3(d.batch), dim3(256), 0, s,
                                     q, sched, rope_tab, scale, qrot, d.batch, d.H, d.d_h, d.E);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return check_launch();
}

}  // namespace qsvd
