// Batched GEMV with split-K: out[b][n] = sum_k x[b][k] * W[k][n], W row-major
// K x N.  HBM-bound on W for the small batches of a decode step, so the
// kernel is built for bytes in flight: each lane loads 8 consecutive weights
// (16 bytes for 16-bit weights) per row, 8 rows at a time, and keeps
// 16 sequences x 8 columns of accumulators; the 8 warps of a CTA split the
// rows and add their results in a fixed order.  CTAs split K (KS ways) and
// write partials part[ks][b][n]; with `ticket` non-null, the last CTA of each
// column block (atomic ticket, no waiting) adds the KS partials in split order
// into `out` and resets its ticket, so the result is deterministic.
//
// grid (ceil(N/256), KS, ceil(B/16)), block 256.
#pragma once
#include "internal.cuh"

namespace qsvd {

template <typename XT, typename WT>
__global__ void __launch_bounds__(256)
k_gemv_partial(const XT* __restrict__ x, const WT* __restrict__ W, float* __restrict__ part,
               int B, int K, int N, int KS, float* __restrict__ out,
               int32_t* __restrict__ ticket) {
  constexpr int BC = 16;     // sequences per CTA
  constexpr int KC = 64;     // rows staged per chunk
  constexpr int CW = 8;      // columns per lane
  constexpr int CT = 32 * CW;   // columns per CTA
  __shared__ __align__(16) float xs[KC][BC];
  __shared__ float red[BC][CT];
  __shared__ int last_cta;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col0 = blockIdx.x * CT;
  const int col = col0 + CW * lane;
  const bool col_ok = col < N;      // N % 32 == 0 and N % 8 == 0: a lane's columns are all in or out
  const int ks = blockIdx.y;
  const int b0 = blockIdx.z * BC;
  const int bn = min(BC, B - b0);
  const int rs = K / KS;
  const int row0 = ks * rs;

  float acc[BC][CW];
#pragma unroll
  for (int b = 0; b < BC; ++b)
#pragma unroll
    for (int c = 0; c < CW; ++c) acc[b][c] = 0.f;

  for (int kc = 0; kc < rs; kc += KC) {
    const int kn = min(KC, rs - kc);
    __syncthreads();
    for (int i = threadIdx.x; i < KC * BC; i += 256) {
      const int kk = i / BC, b = i % BC;
      xs[kk][b] = (b < bn && kk < kn) ? dev::to_f(x[size_t(b0 + b) * K + row0 + kc + kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = warp; kk < kn; kk += 8) {
      float w[CW];
#pragma unroll
      for (int c = 0; c < CW; ++c) w[c] = 0.f;
      if (col_ok) {
        const WT* wp = W + size_t(row0 + kc + kk) * N + col;
#pragma unroll
        for (int v = 0; v < int(CW * sizeof(WT)) / 16; ++v) {
          const uint4 raw = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(wp) + 16 * v);
          const WT* e = reinterpret_cast<const WT*>(&raw);
#pragma unroll
          for (int c = 0; c < int(16 / sizeof(WT)); ++c) w[v * (16 / sizeof(WT)) + c] = dev::to_f(e[c]);
        }
      }
      const float4* xv = reinterpret_cast<const float4*>(&xs[kk][0]);
#pragma unroll
      for (int q4 = 0; q4 < BC / 4; ++q4) {
        const float4 xq = xv[q4];
        const float xb[4] = {xq.x, xq.y, xq.z, xq.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
          for (int c = 0; c < CW; ++c) acc[4 * q4 + e][c] = fmaf(xb[e], w[c], acc[4 * q4 + e][c]);
      }
    }
  }
  // deterministic cross-warp sum: warps add in order
  for (int wi = 0; wi < 8; ++wi) {
    __syncthreads();
    if (warp == wi) {
#pragma unroll
      for (int b = 0; b < BC; ++b)
#pragma unroll
        for (int c = 0; c < CW; ++c) {
          float& dst = red[b][CW * lane + c];
          dst = (wi == 0) ? acc[b][c] : dst + acc[b][c];
        }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < bn * CT; i += 256) {
    const int b = i / CT, c = i % CT;
    if (col0 + c < N) part[(size_t(ks) * B + b0 + b) * N + col0 + c] = red[b][c];
  }
  if (ticket == nullptr) return;
  // last CTA of this column block adds the KS partials in order
  __threadfence();
  __syncthreads();
  int32_t* tk = ticket + blockIdx.z * gridDim.x + blockIdx.x;
  if (threadIdx.x == 0) last_cta = (atomicAdd(tk, 1) == KS - 1);
  __syncthreads();
  if (!last_cta) return;
  __threadfence();
  for (int i = threadIdx.x; i < bn * CT; i += 256) {
    const int b = i / CT, c = i % CT;
    if (col0 + c >= N) continue;
    float s = 0.f;
    for (int k = 0; k < KS; ++k)
      s += __ldcg(part + (size_t(k) * B + b0 + b) * N + col0 + c);
    out[size_t(b0 + b) * N + col0 + c] = s;
  }
  if (threadIdx.x == 0) *tk = 0;   // ready for the next call
}

// Split-K factor: about two CTAs per SM of a 148-SM B200 over the (N/256)
// column blocks, at most `cap`, dividing K into whole 32-row multiples.  It
// depends on the shapes only, so workspace layouts do not depend on the GPU.
inline int gemv_ksplit(int K, int N, int B, int cap) {
  const int cols = (N + 255) / 256;
  const int bch = (B + 15) / 16;
  int ks = 296 / (cols * bch);
  if (ks < 1) ks = 1;
  if (ks > cap) ks = cap;
  while (ks > 1 && (K % ks || (K / ks) % 32)) --ks;
  return ks;
}

inline int gemv_tickets(int N, int B) { return ((N + 255) / 256) * ((B + 15) / 16); }

}  // namespace qsvd
