// Prefill of the latent cache: c = x W^d for every token of a prompt, rounded
// to the cache type (or quantised per 128-channel group) and stored at the
// token's cache row -- the cached latent of the QSVD paper notes (关键设计:
// only C = X W^d is kept) and its quantisation (QSVD digest, Method, Step 3),
// for many tokens at once.  The same per-token arithmetic as
// qsvd_append_latent: fp32 accumulation, then fp16/bf16 round-to-nearest, or
// amax / qmax -> fp16 scale -> round-half-even codes.
//
// One dense GEMM on the tensor cores: rows of x (M = 128 per tile) times
// W^d (N = 256 columns of r per tile, K = E), tcgen05 with the accumulator
// in TMEM (two buffers of 256 columns), operands staged by TMA: x as K-major
// boxes [128 rows][64], W^d read in place as the MN-major B operand (its
// [E][r] rows are K).  Persistent CTAs walk the (row tile, column block)
// units round-robin.
//
// Roles (192 threads): warp 0 producer, warp 1 TMEM allocation and the MMA
// thread, warps 2-5 epilogue (TMEM lane = row of the tile; warp w reads lanes
// 32 (w % 4)): TMEM -> registers -> rounding or quantisation -> the row's 256
// channels (and, for int4/int8, its two group scales) in the cache.  Every
// wait is bounded as in the split kernels.
#include <cuda.h>

#include <cstring>

#include "internal.cuh"
#include "tc_common.cuh"

namespace qsvd {
namespace {

constexpr int kPfThreads = 192;
constexpr int kPfN = 256;                          // columns of r per unit
constexpr int kPfABytes = 128 * 128;              // x box: 128 rows x 64 channels x 2 bytes
constexpr int kPfBBytes = 4 * 64 * 128;           // W^d: 4 chunks of [64 K rows][64 N] x 2 bytes
constexpr int kPfSlot = kPfABytes + kPfBBytes;    // 48 KB
constexpr int kPfMaxSlots = 4;

// Quantise one group of 128 channels of one row (thread-local), with the
// append path's arithmetic: s32 = amax / qmax (IEEE), saturated to the fp16
// range (flagged), s16 = fp16_rn(s32), code = clamp(rint_half_even(v / s16)).
template <int CT>
__device__ __forceinline__ void pf_quant_group(const float* v, uint8_t* cache, __half* scales, size_t row,
                                               int r, int c0, int32_t* status) {
  constexpr int qmax = CT == QSVD_I4 ? 7 : 127;
  float a = 0.f;
#pragma unroll
  for (int e = 0; e < 128; ++e) a = fmaxf(a, fabsf(v[e]));
  float s32 = __fdiv_rn(a, float(qmax));
  if (s32 > 65504.f) {
    s32 = 65504.f;
    if (status) atomicOr(status, QSVD_STATUS_SCALE_SAT);
  }
  const __half s16 = __float2half_rn(s32);
  const float sf = __half2float(s16);
  scales[row * (r / 128) + c0 / 128] = s16;
  if (CT == QSVD_I8) {
    int8_t* dst = reinterpret_cast<int8_t*>(cache) + row * r + c0;
#pragma unroll
    for (int e0 = 0; e0 < 128; e0 += 16) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float x = v[e0 + 4 * k + i];
          const int q = sf != 0.f ? max(-qmax, min(qmax, __float2int_rn(__fdiv_rn(x, sf)))) : 0;
          word |= uint32_t(uint8_t(int8_t(q))) << (8 * i);
        }
        w[k] = word;
      }
      *reinterpret_cast<uint4*>(dst + e0) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else {
    uint8_t* dst = cache + row * (r / 2) + c0 / 2;
#pragma unroll
    for (int e0 = 0; e0 < 128; e0 += 32) {   // 32 channels -> 16 bytes
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {   // element 2j in the low nibble of byte j
          const float x = v[e0 + 8 * k + i];
          const int q = sf != 0.f ? max(-qmax, min(qmax, __float2int_rn(__fdiv_rn(x, sf)))) : 0;
          word |= uint32_t(q & 0xF) << (4 * i);
        }
        w[k] = word;
      }
      *reinterpret_cast<uint4*>(dst + e0 / 2) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

template <bool BF16, int CT>
__global__ void __launch_bounds__(kPfThreads, 1)
k_prefill(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
          const int32_t* __restrict__ dst_rows, uint8_t* __restrict__ cache, __half* __restrict__ scales,
          float* __restrict__ c_out, int32_t* __restrict__ status, int n_rows, int E, int r,
          int n_dst_rows, int ns) {
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = base;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + size_t(ns) * kPfSlot);
  uint64_t* full = bars;                    // [kPfMaxSlots]
  uint64_t* empty = bars + kPfMaxSlots;     // [kPfMaxSlots]
  uint64_t* afull = bars + 2 * kPfMaxSlots; // [2] accumulator complete
  uint64_t* aempty = afull + 2;             // [2] accumulator read by the epilogue
  uint64_t* drain = aempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NB = r / kPfN;                          // column blocks
  const int units = ((n_rows + 127) / 128) * NB;
  const int KI = E / 64;                            // k items per unit
  const int mine = units > int(blockIdx.x) ? (units - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
  if (mine == 0) return;   // uniform across the CTA

  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(saddr(&full[i]), 1);
      mbar_init(saddr(&empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(saddr(&afull[i]), 1);
      mbar_init(saddr(&aempty[i]), 1);
    }
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
  const uint32_t ring0 = saddr(ring);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint64_t wpol = policy_evict_last();   // each W^d column block serves every row tile
    Ring rg(ns);
    long long k = 0;
    bool ok = true;
    for (int j = 0; j < mine && ok; ++j) {
      const int u = int(blockIdx.x) + j * int(gridDim.x);
      const int m0 = (u / NB) * 128, n0 = (u % NB) * kPfN;
      for (int ki = 0; ki < KI; ++ki) {
        if (!__all_sync(0xffffffffu, mbar_wait(saddr(&empty[rg.slot]), rg.phase ^ 1u))) { ok = false; break; }
        const uint32_t dst = ring0 + uint32_t(rg.slot) * kPfSlot;
        const uint32_t fb = saddr(&full[rg.slot]);
        if (lane == 0) mbar_expect_tx(fb, uint32_t(kPfSlot));
        __syncwarp();
        const int ln = int(k & 15) * 2;   // rotating issuing lanes
        // x rows past n_rows arrive as zeros (outside the map)
        if (lane == ln) tma_load_2d(dst, &tm_x, 64 * ki, m0, fb);
        if (lane == ln + 1) tma_load_3d_hint(dst + kPfABytes, &tm_w, 0, 64 * ki, n0 / 64, fb, wpol);
        __syncwarp();
        rg.advance();
        ++k;
      }
      if (__any_sync(0xffffffffu, *abort_flag)) ok = false;
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      if (status) atomicOr(status, QSVD_STATUS_TIMEOUT);
      for (long long kk = (k > ns ? k - ns : 0); kk < k; ++kk)
        mbar_wait(saddr(&full[int(kk % ns)]), uint32_t(kk / ns) & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t id = idesc_f16(128, kPfN, BF16, false, true);   // B MN-major
      const uint64_t da0 = sdesc(ring0, 16, 1024);                        // x: K-major
      const uint64_t db0 = sdesc(ring0 + kPfABytes, 64 * 128, 1024);      // W^d: MN-major, 64-column chunks
      Ring rg(ns);
      bool ok = true;
      for (int j = 0; j < mine && ok; ++j) {
        const int ab = j & 1;
        if (j >= 2 && !mbar_wait(saddr(&aempty[ab]), uint32_t((j - 2) >> 1) & 1u)) { ok = false; break; }
        const uint32_t d = tmem + uint32_t(ab * kPfN);
        for (int ki = 0; ki < KI; ++ki) {
          if (!mbar_wait(saddr(&full[rg.slot]), rg.phase)) { ok = false; break; }
          tc_fence_after();
          const uint64_t off = uint64_t((rg.slot * kPfSlot) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)   // K = 16 per MMA: x 32 bytes along a row, W^d 16 rows
            tc_mma(d, da0 + off + uint64_t((kk * 32) >> 4), db0 + off + uint64_t((kk * 16 * 128) >> 4), id,
                   (ki | kk) != 0);
          tc_commit(saddr(&empty[rg.slot]));
          rg.advance();
        }
        if (!ok) break;
        tc_commit(saddr(&afull[ab]));
        if (*abort_flag) ok = false;
      }
      if (!ok) {
        *abort_flag = 1;
        if (status) atomicOr(status, QSVD_STATUS_TIMEOUT);
      }
      tc_commit(saddr(drain));
      mbar_wait(saddr(drain), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int t = 32 * q + lane;   // row of the tile == TMEM lane
    const uint32_t lane_off = uint32_t(32 * q) << 16;
    for (int j = 0; j < mine; ++j) {
      const int u = int(blockIdx.x) + j * int(gridDim.x);
      const int m0 = (u / NB) * 128, n0 = (u % NB) * kPfN;
      const int ab = j & 1;
      const int fail = group_or(!mbar_wait(saddr(&afull[ab]), uint32_t(j >> 1) & 1u));
      if (fail) {
        if (t == 0) { *abort_flag = 1; if (status) atomicOr(status, QSVD_STATUS_TIMEOUT); }
        break;
      }
      tc_fence_after();
      const int m = m0 + t;
      long long row = -1;
      if (m < n_rows) {
        const int dr = dst_rows ? dst_rows[m] : m;   // no row list: row m of the output
        if (dr >= 0 && dr < n_dst_rows) row = dr;
        else if (status) atomicOr(status, QSVD_STATUS_POS_OOB);
      }
      const uint32_t ta = tmem + lane_off + uint32_t(ab * kPfN);
      // two groups of 128 channels, 16 columns per TMEM load
#pragma unroll 1
      for (int g = 0; g < kPfN / 128; ++g) {
        float v[128];
#pragma unroll
        for (int c = 0; c < 8; ++c) tmem_ld16(ta + uint32_t(128 * g + 16 * c), v + 16 * c);
        tmem_wait_ld();
        if (row >= 0) {
          const int c0 = n0 + 128 * g;
          if (c_out) {
            float4* co = reinterpret_cast<float4*>(c_out + size_t(m) * r + c0);
#pragma unroll
            for (int e = 0; e < 32; ++e) co[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
          }
          if (CT == QSVD_F32) {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(cache) + size_t(row) * r + c0);
#pragma unroll
            for (int e = 0; e < 32; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
          } else if (CT == QSVD_F16 || CT == QSVD_BF16) {
            uint4* dst = reinterpret_cast<uint4*>(cache + (size_t(row) * r + c0) * 2);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              uint32_t w[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float x0 = v[8 * e + 2 * k], x1 = v[8 * e + 2 * k + 1];
                if (CT == QSVD_F16) {
                  const __half2 h = __halves2half2(__float2half_rn(x0), __float2half_rn(x1));
                  w[k] = *reinterpret_cast<const uint32_t*>(&h);
                } else {
                  const __nv_bfloat162 h = __halves2bfloat162(__float2bfloat16_rn(x0), __float2bfloat16_rn(x1));
                  w[k] = *reinterpret_cast<const uint32_t*>(&h);
                }
              }
              dst[e] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          } else {
            pf_quant_group<CT>(v, cache, scales, size_t(row), r, c0, status);
          }
        }
      }
      tc_fence_before();
      group_sync();
      if (t == 0) mbar_arrive(saddr(&aempty[ab]));
      if (group_or(*abort_flag)) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

template <bool BF16, int CT>
cudaError_t prefill_t(const qsvd_dims& d, const void* wd, const void* x, int n_rows, const int32_t* dst_rows,
                      void* cache, void* scales, float* c_out, int32_t* status, cudaStream_t s) {
  TensorMapEncode enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt = BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap tx, tw;
  memset(&tx, 0, sizeof(tx));
  memset(&tw, 0, sizeof(tw));
  {
    // x [n_rows][E]: one box {64 channels, 128 rows}
    const cuuint64_t dims[2] = {cuuint64_t(d.E), cuuint64_t(n_rows)};
    const cuuint64_t strides[1] = {cuuint64_t(d.E) * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&tx, dt, 2, const_cast<void*>(x), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // W^d [E][r] seen as {64 columns, row of E, 64-column chunk}: one box
    // {64, 64, 4} is 64 K rows x 256 columns, smem [chunk][row][64]
    const cuuint64_t dims[3] = {64, cuuint64_t(d.E), cuuint64_t(d.r / 64)};
    const cuuint64_t strides[2] = {cuuint64_t(d.r) * 2, 128};
    const cuuint32_t box[3] = {64, 64, 4};
    const cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tw, dt, 3, const_cast<void*>(wd), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int units = ((n_rows + 127) / 128) * (d.r / kPfN);
  const int grid = units < sms ? units : sms;
  constexpr int ns = kPfMaxSlots;
  const size_t smem = 1024 + size_t(ns) * kPfSlot + (2 * kPfMaxSlots + 5) * 8 + 16;
  auto kern = k_prefill<BF16, CT>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  {
    const cudaError_t le = launch_pdl(kern, dim3(grid), dim3(kPfThreads), smem, s, tx, tw, dst_rows,
                                      static_cast<uint8_t*>(cache), static_cast<__half*>(scales), c_out,
                                      status, n_rows, d.E, d.r, d.batch * d.max_len, ns);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return check_launch();
}

template <bool BF16>
cudaError_t prefill_ct(const qsvd_dims& d, const void* wd, const void* x, int n_rows, const int32_t* dst_rows,
                       void* cache, void* scales, float* c_out, int32_t* status, cudaStream_t s) {
  switch (d.cache_dtype) {
    case QSVD_F32: return prefill_t<BF16, QSVD_F32>(d, wd, x, n_rows, dst_rows, cache, scales, c_out, status, s);
    case QSVD_F16: return prefill_t<BF16, QSVD_F16>(d, wd, x, n_rows, dst_rows, cache, scales, c_out, status, s);
    case QSVD_BF16: return prefill_t<BF16, QSVD_BF16>(d, wd, x, n_rows, dst_rows, cache, scales, c_out, status, s);
    case QSVD_I8: return prefill_t<BF16, QSVD_I8>(d, wd, x, n_rows, dst_rows, cache, scales, c_out, status, s);
    case QSVD_I4: return prefill_t<BF16, QSVD_I4>(d, wd, x, n_rows, dst_rows, cache, scales, c_out, status, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool prefill_supported(const qsvd_dims& d) {
  return (d.weight_dtype == QSVD_F16 || d.weight_dtype == QSVD_BF16) && d.r % kPfN == 0 && d.E % 64 == 0 &&
         !d.h2;
}

cudaError_t launch_prefill(const qsvd_dims& d, const void* wd, const void* x, int n_rows,
                           const int32_t* dst_rows, void* cache, void* scales, float* c_out,
                           int32_t* status, cudaStream_t s) {
  if (!prefill_supported(d)) return cudaErrorInvalidConfiguration;
  return d.weight_dtype == QSVD_BF16
             ? prefill_ct<true>(d, wd, x, n_rows, dst_rows, cache, scales, c_out, status, s)
             : prefill_ct<false>(d, wd, x, n_rows, dst_rows, cache, scales, c_out, status, s);
}

}  // namespace qsvd
