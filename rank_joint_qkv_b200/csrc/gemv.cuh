// Batched GEMV with split-K: out[b][n] = sum_k x[b][k] * W[k][n], W row-major
// K x N.  HBM-bound on W for the small batches of a decode step, so the kernel
// is built for bytes in flight: a CTA owns a tile of up to 64 KB of W (RT rows
// x 256 columns) and requests the whole tile at once with 16-byte
// asynchronous copies, while its threads stage the matching slice of x.  Each
// of its 128 threads then owns two adjacent columns and accumulates 16
// sequences over the tile's rows -- no reduction inside the CTA -- with few
// enough registers that three CTAs share an SM.  CTAs split K and write partials part[ks][b][n]; with `ticket`
// non-null, the last CTA of each column block (atomic ticket, no waiting)
// adds the KS partials in split order into `out` and resets its ticket, so the
// result is deterministic.
//
// grid (ceil(N/256), KS, ceil(B/16)), block kGemvThreads.
#pragma once
#include <type_traits>

#include "internal.cuh"

namespace qsvd {


// rows of W per CTA: a 64 KB tile
template <typename WT>
__host__ __device__ constexpr int gemv_rows() { return 65536 / (256 * int(sizeof(WT))); }

constexpr int kGemvThreads = 128;   // each thread owns 2 adjacent columns of the 256

// Two adjacent elements of W as floats.
__device__ __forceinline__ float2 load2(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ float2 load2(const __half* p) {
  return __half22float2(*reinterpret_cast<const __half2*>(p));
}
__device__ __forceinline__ float2 load2(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}

// Four consecutive elements, loaded as one 16- or 8-byte vector, as floats
// (the pointer argument only selects the element type).
__device__ __forceinline__ void unpack4(const float4& q, float (&v)[4], const float*) {
  v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
}
__device__ __forceinline__ void unpack4(const uint2& q, float (&v)[4], const __half*) {
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&q.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&q.y));
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
__device__ __forceinline__ void unpack4(const uint2& q, float (&v)[4], const __nv_bfloat16*) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.y));
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}

template <typename XT, typename WT>
__global__ void __launch_bounds__(kGemvThreads)
k_gemv_partial(const XT* __restrict__ x, const WT* __restrict__ W, float* __restrict__ part,
               int B, int K, int N, int KS, float* __restrict__ out,
               int32_t* __restrict__ ticket, int32_t* status) {
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  (void)status;                          // no waits left to time out
  constexpr int BC = 16;                 // sequences per CTA
  constexpr int RT = gemv_rows<WT>();    // rows per CTA
  extern __shared__ __align__(128) uint8_t gsm[];
  WT* tile = reinterpret_cast<WT*>(gsm);                               // RT x 256
  float* xs = reinterpret_cast<float*>(gsm + RT * 256 * sizeof(WT));   // RT x BC
  __shared__ int last_cta;
  const int col0 = blockIdx.x * 256;
  const int ncols = min(256, N - col0);
  const int ks = blockIdx.y;
  const int row0 = ks * RT;
  const int rows = min(RT, K - row0);
  const int b0 = blockIdx.z * BC;
  const int bn = min(BC, B - b0);

  // Stage the tile with 16-byte asynchronous copies (cp.async: no registers
  // held while in flight, so the whole 64 KB is requested at once).  Rows are
  // 16-byte aligned: N is a multiple of 16 / sizeof(WT).
  constexpr int VPR = 256 * int(sizeof(WT)) / 16;   // 16-byte vectors per tile row
  constexpr int EPV = 16 / int(sizeof(WT));         // elements per vector
  for (int idx = threadIdx.x; idx < RT * VPR; idx += kGemvThreads) {
    const int rr = idx / VPR, cv = idx % VPR;
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(tile)) + 16u * idx;
    if (rr < rows && cv * EPV < ncols) {
      const WT* src = W + size_t(row0 + rr) * N + col0 + cv * EPV;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
    } else {
      reinterpret_cast<uint4*>(tile)[idx] = make_uint4(0, 0, 0, 0);
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (int i = threadIdx.x; i < RT * BC; i += kGemvThreads) {
    const int kk = i / BC, b = i % BC;
    xs[i] = (b < bn && kk < rows) ? dev::to_f(x[size_t(b0 + b) * K + row0 + kk]) : 0.f;
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();

  const int c = 2 * threadIdx.x;   // first of this thread's two columns
  float acc[BC][2];
#pragma unroll
  for (int b = 0; b < BC; ++b) acc[b][0] = acc[b][1] = 0.f;
#pragma unroll 2
  for (int kk = 0; kk < rows; ++kk) {
    const float2 w = load2(tile + kk * 256 + c);
    const float4* xv = reinterpret_cast<const float4*>(xs + kk * BC);
#pragma unroll
    for (int q4 = 0; q4 < BC / 4; ++q4) {
      const float4 xq = xv[q4];
      acc[4 * q4 + 0][0] = fmaf(xq.x, w.x, acc[4 * q4 + 0][0]);
      acc[4 * q4 + 0][1] = fmaf(xq.x, w.y, acc[4 * q4 + 0][1]);
      acc[4 * q4 + 1][0] = fmaf(xq.y, w.x, acc[4 * q4 + 1][0]);
      acc[4 * q4 + 1][1] = fmaf(xq.y, w.y, acc[4 * q4 + 1][1]);
      acc[4 * q4 + 2][0] = fmaf(xq.z, w.x, acc[4 * q4 + 2][0]);
      acc[4 * q4 + 2][1] = fmaf(xq.z, w.y, acc[4 * q4 + 2][1]);
      acc[4 * q4 + 3][0] = fmaf(xq.w, w.x, acc[4 * q4 + 3][0]);
      acc[4 * q4 + 3][1] = fmaf(xq.w, w.y, acc[4 * q4 + 3][1]);
    }
  }
  if (c < ncols) {
#pragma unroll
    for (int b = 0; b < BC; ++b)   // unrolled with a guard: acc stays in registers
      if (b < bn)
        *reinterpret_cast<float2*>(part + (size_t(ks) * B + b0 + b) * N + col0 + c) =
            make_float2(acc[b][0], acc[b][1]);
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
    // every sequence's partial of one split is loaded together, so the KS
    // rounds of loads overlap instead of running one sequence at a time;
    // each output still adds its partials in split order
    float sum[BC][2];
#pragma unroll
    for (int b = 0; b < BC; ++b) sum[b][0] = sum[b][1] = 0.f;
    const float* pp = part + size_t(b0) * N + col0 + c;
#pragma unroll 1
    for (int k = 0; k < KS; ++k) {
      float2 v[BC];
#pragma unroll
      for (int b = 0; b < BC; ++b)
        v[b] = b < bn ? __ldcg(reinterpret_cast<const float2*>(pp + (size_t(k) * B + b) * N))
                      : make_float2(0.f, 0.f);
#pragma unroll
      for (int b = 0; b < BC; ++b) { sum[b][0] += v[b].x; sum[b][1] += v[b].y; }
    }
#pragma unroll
    for (int b = 0; b < BC; ++b)
      if (b < bn)
        *reinterpret_cast<float2*>(out + size_t(b0 + b) * N + col0 + c) = make_float2(sum[b][0], sum[b][1]);
  }
  if (threadIdx.x == 0) *tk = 0;   // ready for the next call
}

template <typename WT>
inline size_t gemv_smem() { return size_t(gemv_rows<WT>()) * (256 * sizeof(WT) + 16 * 4); }

// ---------------------------------------------------------------------------
// Tensor-core variant for 16-bit weights (mma.sync m16n8k16, fp32 accumulate).
// At 16 sequences a CUDA-core GEMV does 16 FMAs per weight element and is
// issue-bound well before HBM; here the 16 sequences are the M = 16 rows of
// the MMA and the weight tile is read from shared memory once with ldmatrix,
// so the kernel is bound by its loads.  A CTA owns a tall, narrow tile (512
// rows x 64 columns, 64 KB) and its four warps split the rows, so K is split
// across few CTAs (ceil(K / 512)) and the split-K reduction stays small.
// The tile arrives by TMA (two boxes of 256 rows) into 128-byte-swizzled
// rows that ldmatrix reads conflict-free.  An fp32 activation enters as a 16-bit part plus its 16-bit rounding
// residual (two MMAs into the same accumulator); with fp16 weights it is
// first scaled by a power of two per sequence and CTA (largest |x| of the
// slice in [2^14, 2^15)) so that both parts stay in fp16 range, and the
// partial is scaled back exactly.
namespace gemv_mma {
constexpr int RT = 512;                      // rows (K) per CTA
constexpr int CT = 64;                       // columns per CTA: 8 n-tiles of 8
constexpr int TSTRIDE = CT * 2;              // tile row: 128 bytes, TMA 128-byte swizzle
constexpr int TBOX = 256;                    // rows per TMA box (box dims are at most 256)
constexpr int XSTRIDE = RT * 2 + 16;         // activation row pitch in bytes (padded: ldmatrix rows hit distinct banks)
template <int NPART>
__host__ __device__ constexpr int smem_bytes() { return 1024 + RT * TSTRIDE + NPART * 16 * XSTRIDE; }

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

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
template <bool BF16>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if (BF16)
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
                 "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  else
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
                 "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
}  // namespace gemv_mma

// grid (ceil(N/64), KS = ceil(K/512), ceil(B/16)), block 128.  Writes partials
// part[ks][b][n]; with `ticket` non-null the last CTA of each (column block,
// sequence block) adds the KS partials in split order into `out` (converted
// to OT).  Activation row of sequence b for output column n:
// x + b * xg.row + (n / xg.cols) * xg.step (xg.cols a multiple of 64); the
// plain GEMV has row = K, step = 0.
struct XGroups {
  long long row;    // elements between sequences
  int cols;         // output columns sharing one activation row
  long long step;   // elements between consecutive column groups' rows
};
template <typename XT, typename WT, typename OT = float>
__global__ void __launch_bounds__(128)
k_gemv_mma(const __grid_constant__ CUtensorMap tm_w, const XT* __restrict__ x, XGroups xg,
           float* __restrict__ part, int B, int K, int N, int KS, OT* __restrict__ out,
           int32_t* __restrict__ ticket, int32_t* status, const uint8_t* __restrict__ pf,
           unsigned long long pf_bytes) {
  using namespace gemv_mma;
  constexpr bool BF16 = std::is_same<WT, __nv_bfloat16>::value;
  constexpr bool SPLIT = !std::is_same<XT, WT>::value;   // activation wider than the weights
  constexpr bool SCALE = SPLIT && !BF16;                  // fp16 range needs the power-of-two scale
  constexpr int NPART = SPLIT ? 2 : 1;
  extern __shared__ uint8_t gsm_raw[];
  uint8_t* tile = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gsm_raw) + 1023) &
                                             ~uintptr_t(1023));   // swizzle atoms need 1024-byte alignment
  uint8_t* xs = tile + RT * TSTRIDE;      // [NPART][16][XSTRIDE bytes]
  __shared__ __align__(8) uint64_t bar;
  __shared__ float inv_scale[16];
  __shared__ unsigned smax[16];
  __shared__ int last_cta;
  const int col0 = blockIdx.x * CT, ncols = min(CT, N - col0);
  const int ks = blockIdx.y, row0 = ks * RT, rows = min(RT, K - row0);
  const int b0 = blockIdx.z * 16, bn = min(16, B - b0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // weight tile: two TMA boxes of 256 rows x 64 columns (zeros outside the
  // matrix), swizzled 128-byte rows; completion on one mbarrier
  const uint32_t tile_s = static_cast<uint32_t>(__cvta_generic_to_shared(tile));
  const uint32_t bar_s = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_s) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_s),
                 "r"(uint32_t(RT * TSTRIDE)) : "memory");
#pragma unroll
    for (int h = 0; h < RT / TBOX; ++h)
      asm volatile(
          "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
          " [%0], [%1, {%2, %3}], [%4];" ::"r"(tile_s + h * TBOX * TSTRIDE),
          "l"(reinterpret_cast<uint64_t>(&tm_w)), "r"(col0), "r"(row0 + h * TBOX), "r"(bar_s)
          : "memory");
  }

  // the next kernel's weights towards L2 (constant: no need to wait for anything)
  if (pf_bytes && tid == 32) dev::l2_prefetch_share(pf, pf_bytes);
  // the weight tile is in flight; everything below reads what earlier kernels wrote
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();

  // activation slice, row k of sequence j at xs[j][k]; thread tid covers
  // k = 4 tid .. 4 tid + 3 of every sequence with one vector load each, all
  // 16 issued before any is used (rows is a multiple of 32)
  static_assert(RT == 4 * 128, "four activation rows per thread");
  // The loads are unconditional (a clamped, valid address) and masked after,
  // so that nothing stands between them.
  using Raw = typename std::conditional<sizeof(XT) == 4, float4, uint2>::type;
  const bool kin = 4 * tid < rows;
  const XT* xrow = x + size_t(b0) * xg.row + size_t(col0 / xg.cols) * xg.step + row0 + (kin ? 4 * tid : 0);
  Raw raw[16];
#pragma unroll
  for (int j = 0; j < 16; ++j)
    raw[j] = __ldg(reinterpret_cast<const Raw*>(xrow + size_t(j < bn ? j : 0) * xg.row));
  float xv[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    unpack4(raw[j], xv[j], static_cast<const XT*>(nullptr));
    if (!(j < bn && kin)) xv[j][0] = xv[j][1] = xv[j][2] = xv[j][3] = 0.f;
  }
  if (SCALE) {
    if (tid < 16) smax[tid] = 0u;
    float m[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
      m[j] = fmaxf(fmaxf(fabsf(xv[j][0]), fabsf(xv[j][1])), fmaxf(fabsf(xv[j][2]), fabsf(xv[j][3])));
    const float wm = dev::warp_reduce_transposed<16>(m, lane, dev::OpMax());   // lane L: sequence L % 16
    __syncthreads();
    if (lane < 16) atomicMax(&smax[lane], __float_as_uint(wm));   // non-negative floats order as integers
    __syncthreads();
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    // s = 2^(14 - e), e = exponent of the largest |x| (clamped so that s and
    // 1/s are normal floats), built from exponent bits
    float s = 1.f, inv = 1.f;
    if (SCALE) {
      const unsigned mb = smax[j];
      if (mb != 0u) {
        const int e = max(int((mb >> 23) & 0xFFu) - 127, -112);
        s = __uint_as_float(unsigned(141 - e) << 23);
        inv = __uint_as_float(unsigned(113 + e) << 23);
      }
    }
    WT hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float v = xv[j][e] * s;
      hi[e] = dev::from_f<WT>(v);
      lo[e] = dev::from_f<WT>(v - dev::to_f(hi[e]));
    }
    *reinterpret_cast<uint2*>(xs + j * XSTRIDE + 8 * tid) = *reinterpret_cast<const uint2*>(hi);
    if (SPLIT) *reinterpret_cast<uint2*>(xs + (16 + j) * XSTRIDE + 8 * tid) = *reinterpret_cast<const uint2*>(lo);
    if (tid == 0) inv_scale[j] = inv;
  }
  // wait for the tile (bounded: 2 s); on expiry flag it and skip the work
  __syncthreads();   // the barrier is initialised before anyone polls it
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

  // warp w: k-steps w, w + 4, ... over all 8 n-tiles
  float acc[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  const uint32_t xs_s = static_cast<uint32_t>(__cvta_generic_to_shared(xs));
  const int mrow = (lane & 7) + 8 * ((lane >> 3) & 1);   // ldmatrix: this lane's row of its 8x8 matrix
  const int mcol = 8 * (lane >> 4);
#pragma unroll 2
  for (int kk = warp; kk < RT / 16; kk += 4) {
    uint32_t a[NPART][4];
#pragma unroll
    for (int p = 0; p < NPART; ++p)
      ldsm_x4(xs_s + (p * 16 + mrow) * XSTRIDE + (16 * kk + mcol) * 2, a[p]);
#pragma unroll
    for (int jp = 0; jp < 4; ++jp) {
      uint32_t bfr[4];   // k rows 16 kk + (0..7 | 8..15), n-tiles 2 jp and 2 jp + 1
      const int row = 16 * kk + mrow, chunk = 2 * jp + (lane >> 4);   // 16-byte chunk of the row
      ldsm_x4_t(tile_s + row * TSTRIDE + ((chunk ^ (row & 7)) << 4), bfr);
#pragma unroll
      for (int p = 0; p < NPART; ++p) {
        mma16816<BF16>(acc[2 * jp], a[p], bfr[0], bfr[1]);
        mma16816<BF16>(acc[2 * jp + 1], a[p], bfr[2], bfr[3]);
      }
    }
  }
  // the four warps' partial tiles, summed in shared memory (over the tile,
  // no longer needed); fragment: (row g, cols 2t, 2t+1) and (row g + 8)
  __syncthreads();
  float* red = reinterpret_cast<float*>(tile);   // [4][16][CT]
  {
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      *reinterpret_cast<float2*>(red + (warp * 16 + g) * CT + 8 * j + 2 * t4) = make_float2(acc[j][0], acc[j][1]);
      *reinterpret_cast<float2*>(red + (warp * 16 + g + 8) * CT + 8 * j + 2 * t4) = make_float2(acc[j][2], acc[j][3]);
    }
  }
  __syncthreads();
  const int ob = tid >> 3, oc = 8 * (tid & 7);   // this thread's 8 outputs: sequence ob, columns oc..oc+7
  float o[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int i = ob * CT + oc + e;
    o[e] = (red[i] + red[16 * CT + i] + red[32 * CT + i] + red[48 * CT + i]) * inv_scale[ob];
  }
  const bool live = ob < bn && oc < ncols;   // ncols is a multiple of 32
  float* prow = part + (size_t(ks) * B + b0 + ob) * N + col0 + oc;
  if (live) {
    reinterpret_cast<float4*>(prow)[0] = make_float4(o[0], o[1], o[2], o[3]);
    reinterpret_cast<float4*>(prow)[1] = make_float4(o[4], o[5], o[6], o[7]);
  }
  if (ticket == nullptr) return;
  __threadfence();
  __syncthreads();
  int32_t* tk = ticket + blockIdx.z * gridDim.x + blockIdx.x;
  if (tid == 0) last_cta = (atomicAdd(tk, 1) == KS - 1);
  __syncthreads();
  if (!last_cta) return;
  __threadfence();
  if (live) {
    // partials added in split order; all splits' loads are in flight together
    const float* pp = part + size_t(b0 + ob) * N + col0 + oc;
    float sum[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) sum[e] = 0.f;
    for (int k = 0; k < KS; k += 4) {
      float4 v[4][2];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool ok = k + u < KS;
        const float4* src = reinterpret_cast<const float4*>(pp + size_t(k + u) * B * N);
        v[u][0] = ok ? __ldcg(src) : make_float4(0.f, 0.f, 0.f, 0.f);
        v[u][1] = ok ? __ldcg(src + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        sum[0] += v[u][0].x; sum[1] += v[u][0].y; sum[2] += v[u][0].z; sum[3] += v[u][0].w;
        sum[4] += v[u][1].x; sum[5] += v[u][1].y; sum[6] += v[u][1].z; sum[7] += v[u][1].w;
      }
    }
    OT* orow = out + size_t(b0 + ob) * N + col0 + oc;
    if constexpr (std::is_same<OT, float>::value) {
      reinterpret_cast<float4*>(orow)[0] = make_float4(sum[0], sum[1], sum[2], sum[3]);
      reinterpret_cast<float4*>(orow)[1] = make_float4(sum[4], sum[5], sum[6], sum[7]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) orow[e] = dev::from_f<OT>(sum[e]);
    }
  }
  if (tid == 0) *tk = 0;   // ready for the next call
}

// Launch the GEMV: tensor cores for 16-bit weights, CUDA cores for fp32.
// Per-group activation rows (xg) and a non-float output need the tensor-core
// variant (16-bit weights).  pf / pf_bytes: constant bytes the next kernel
// reads (its weights), requested into L2 while this one runs (tensor-core
// variant; a hint only).
template <typename XT, typename WT, typename OT = float>
cudaError_t launch_gemv(const XT* x, const WT* W, float* part, int B, int K, int N, int KS,
                        OT* out, int32_t* ticket, int32_t* status, cudaStream_t s,
                        XGroups xg = XGroups{0, 0, 0}, const void* pf = nullptr, size_t pf_bytes = 0) {
  if (xg.cols == 0) xg = XGroups{K, N, 0};
  cudaError_t e;
  if constexpr (sizeof(WT) == 2) {
    const dim3 grid((N + gemv_mma::CT - 1) / gemv_mma::CT, KS, (B + 15) / 16);
    constexpr int NPART = std::is_same<XT, WT>::value ? 1 : 2;
    TensorMapEncode enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap tm;
    const cuuint64_t dims[2] = {cuuint64_t(N), cuuint64_t(K)};
    const cuuint64_t strides[1] = {cuuint64_t(N) * sizeof(WT)};
    const cuuint32_t box[2] = {gemv_mma::CT, gemv_mma::TBOX};
    const cuuint32_t es[2] = {1, 1};
    const CUtensorMapDataType dt = std::is_same<WT, __nv_bfloat16>::value
                                       ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (enc(&tm, dt, 2, const_cast<WT*>(W), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    auto kern = k_gemv_mma<XT, WT, OT>;
    const int smem = gemv_mma::smem_bytes<NPART>();
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    {
      const cudaError_t le = launch_pdl(kern, dim3(grid), dim3(128), smem, s, tm, x, xg, part, B, K, N, KS,
                                       out, ticket, status, static_cast<const uint8_t*>(pf),
                                       (unsigned long long)pf_bytes);
      if (le != cudaSuccess) return le;
    }
  } else {
    static_assert(std::is_same<OT, float>::value, "CUDA-core GEMV writes fp32");
    if (xg.step != 0 || xg.row != K) return cudaErrorInvalidValue;
    const dim3 grid((N + 255) / 256, KS, (B + 15) / 16);
    auto kern = k_gemv_partial<XT, WT>;
    const size_t smem = gemv_smem<WT>();
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    {
      const cudaError_t le = launch_pdl(kern, dim3(grid), dim3(kGemvThreads), smem, s,
                                       x, W, part, B, K, N, KS, out, ticket, status);
      if (le != cudaSuccess) return le;
    }
  }
  note_launch();
  return check_launch();
}

}  // namespace qsvd
