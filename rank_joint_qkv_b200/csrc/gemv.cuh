// Batched GEMV with split-K partials: part[ks][b][n] = sum_{k in split ks}
// x[b][k] * W[k][n], W row-major K x N.  HBM-bound on W; each W element is
// read once per batch chunk of 32 rows of x.
//
// grid (ceil(N/64), KS, ceil(B/32)), block 256 = 8 warps; lane owns 2
// columns (N is even, so a lane's pair is either fully inside or outside).
#pragma once
#include "internal.cuh"

namespace qsvd {

template <typename XT, typename WT>
__global__ void __launch_bounds__(256)
k_gemv_partial(const XT* __restrict__ x, const WT* __restrict__ W, float* __restrict__ part,
               int B, int K, int N, int KS) {
  constexpr int BC = 32;
  __shared__ float xs[BC][64];
  __shared__ float red[BC][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col0 = blockIdx.x * 64;
  const int ks = blockIdx.y;
  const int b0 = blockIdx.z * BC;
  const int bn = min(BC, B - b0);
  const int rs = K / KS;
  const int row0 = ks * rs;
  const bool col_ok = col0 + 2 * lane < N;

  float acc[BC][2];
#pragma unroll
  for (int b = 0; b < BC; ++b) { acc[b][0] = 0.f; acc[b][1] = 0.f; }

  for (int kc = 0; kc < rs; kc += 64) {
    const int kn = min(64, rs - kc);
    for (int i = threadIdx.x; i < BC * 64; i += 256) {
      const int b = i / 64, kk = i % 64;
      xs[b][kk] = (b < bn && kk < kn) ? dev::to_f(x[size_t(b0 + b) * K + row0 + kc + kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = warp; kk < kn; kk += 8) {
      const WT* wrow = W + size_t(row0 + kc + kk) * N + col0 + 2 * lane;
      const float w0 = col_ok ? dev::to_f(wrow[0]) : 0.f;
      const float w1 = col_ok ? dev::to_f(wrow[1]) : 0.f;
#pragma unroll
      for (int b = 0; b < BC; ++b) {
        const float xv = xs[b][kk];
        acc[b][0] = fmaf(xv, w0, acc[b][0]);
        acc[b][1] = fmaf(xv, w1, acc[b][1]);
      }
    }
    __syncthreads();
  }
  // deterministic cross-warp sum (warps add in order)
  for (int w = 0; w < 8; ++w) {
    if (warp == w) {
#pragma unroll
      for (int b = 0; b < BC; ++b) {
        if (w == 0) { red[b][2 * lane] = acc[b][0]; red[b][2 * lane + 1] = acc[b][1]; }
        else { red[b][2 * lane] += acc[b][0]; red[b][2 * lane + 1] += acc[b][1]; }
      }
    }
    __syncthreads();
  }
  for (int i = threadIdx.x; i < bn * 64; i += 256) {
    const int b = i / 64, c = i % 64;
    if (col0 + c < N) part[(size_t(ks) * B + b0 + b) * N + col0 + c] = red[b][c];
  }
}

}  // namespace qsvd
