// Batched GEMV with split-K: out[b][n] = sum_k x[b][k] * W[k][n], W row-major
// K x N.  HBM-bound on W for the small batches of a decode step, so the kernel
// is built for bytes in flight: a CTA owns a tile of up to 64 KB of W (kGemvRows
// rows x 256 columns) and pulls the whole tile into shared memory at once with
// one bulk copy per row (cp.async.bulk, completion on one mbarrier), while its
// threads stage the matching slice of x.  Each thread then owns one column
// and accumulates 16 sequences over the tile's rows -- no reduction inside the
// CTA.  CTAs split K and write partials part[ks][b][n]; with `ticket`
// non-null, the last CTA of each column block (atomic ticket, no waiting)
// adds the KS partials in split order into `out` and resets its ticket, so the
// result is deterministic.
//
// grid (ceil(N/256), KS, ceil(B/16)), block 256.
#pragma once
#include "internal.cuh"

namespace qsvd {

namespace gemv_detail {
__device__ __forceinline__ uint32_t saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
}  // namespace gemv_detail

// rows of W per CTA: a 64 KB tile
template <typename WT>
__host__ __device__ constexpr int gemv_rows() { return 65536 / (256 * int(sizeof(WT))); }

template <typename XT, typename WT>
__global__ void __launch_bounds__(256)
k_gemv_partial(const XT* __restrict__ x, const WT* __restrict__ W, float* __restrict__ part,
               int B, int K, int N, int KS, float* __restrict__ out,
               int32_t* __restrict__ ticket, int32_t* status) {
  using namespace gemv_detail;
  constexpr int BC = 16;                 // sequences per CTA
  constexpr int RT = gemv_rows<WT>();    // rows per CTA
  extern __shared__ __align__(128) uint8_t gsm[];
  WT* tile = reinterpret_cast<WT*>(gsm);                          // RT x 256
  float* xs = reinterpret_cast<float*>(gsm + RT * 256 * sizeof(WT));   // RT x BC
  __shared__ __align__(8) uint64_t bar;
  __shared__ int last_cta;
  const int col0 = blockIdx.x * 256;
  const int ncols = min(256, N - col0);
  const int ks = blockIdx.y;
  const int row0 = ks * RT;
  const int rows = min(RT, K - row0);
  const int b0 = blockIdx.z * BC;
  const int bn = min(BC, B - b0);

  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(&bar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const uint32_t row_bytes = uint32_t(ncols) * sizeof(WT);   // multiple of 16
    if (threadIdx.x == 0)
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(&bar)),
                   "r"(row_bytes * uint32_t(rows))
                   : "memory");
    __syncwarp();
    for (int rr = threadIdx.x; rr < rows; rr += 32) {
      const WT* src = W + size_t(row0 + rr) * N + col0;
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
          ::"r"(saddr(tile + rr * 256)), "l"(src), "r"(row_bytes), "r"(saddr(&bar))
          : "memory");
    }
  }
  for (int i = threadIdx.x; i < RT * BC; i += 256) {
    const int kk = i / BC, b = i % BC;
    xs[i] = (b < bn && kk < rows) ? dev::to_f(x[size_t(b0 + b) * K + row0 + kk]) : 0.f;
  }
  __syncthreads();
  // bounded wait for the tile (2 s); on expiry flag it and leave the tile unused
  bool ok = mbar_try(saddr(&bar), 0);
  if (!ok) {
    const uint64_t t0 = gtimer();
    while (!(ok = mbar_try(saddr(&bar), 0)))
      if (gtimer() - t0 > 2000000000ull) break;
  }
  ok = __syncthreads_and(ok);   // one decision for the whole CTA
  if (!ok) {
    if (threadIdx.x == 0 && status) atomicOr(status, QSVD_STATUS_TIMEOUT);
    return;
  }
  const int c = threadIdx.x;
  float acc[BC];
#pragma unroll
  for (int b = 0; b < BC; ++b) acc[b] = 0.f;
  if (c < ncols) {
#pragma unroll 4
    for (int kk = 0; kk < rows; ++kk) {
      const float w = dev::to_f(tile[kk * 256 + c]);
      const float4* xv = reinterpret_cast<const float4*>(xs + kk * BC);
#pragma unroll
      for (int q4 = 0; q4 < BC / 4; ++q4) {
        const float4 xq = xv[q4];
        acc[4 * q4 + 0] = fmaf(xq.x, w, acc[4 * q4 + 0]);
        acc[4 * q4 + 1] = fmaf(xq.y, w, acc[4 * q4 + 1]);
        acc[4 * q4 + 2] = fmaf(xq.z, w, acc[4 * q4 + 2]);
        acc[4 * q4 + 3] = fmaf(xq.w, w, acc[4 * q4 + 3]);
      }
    }
    for (int b = 0; b < bn; ++b) part[(size_t(ks) * B + b0 + b) * N + col0 + c] = acc[b];
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
  if (c < ncols) {
    for (int b = 0; b < bn; ++b)
      out[size_t(b0 + b) * N + col0 + c] =
          dev::sum_strided(part + size_t(b0 + b) * N + col0 + c, size_t(B) * N, KS);
  }
  if (threadIdx.x == 0) *tk = 0;   // ready for the next call
}

template <typename WT>
inline size_t gemv_smem() { return size_t(gemv_rows<WT>()) * (256 * sizeof(WT) + 16 * 4); }

// Split of K: one 64 KB tile of rows per CTA (shape-only, device-independent).
inline int gemv_ksplit(int K, qsvd_dtype wt) {
  const int rt = wt == QSVD_F32 ? 64 : 128;
  return (K + rt - 1) / rt;
}

inline int gemv_tickets(int N, int B) { return ((N + 255) / 256) * ((B + 15) / 16); }

}  // namespace qsvd
