// Append one new token per sequence to the latent cache.
//
//   c = x W^d                        (QSVD digest, Method, Step 1: the latent
//                                      C_qkv = X W^d is what is buffered)
//   c <- H2 c    (optional)          (QSVD paper notes, 关键设计: the H2
//                                      rotation sits between W^d and W^u)
//   quantise per token and group     (QSVD digest, Method, Step 3; A8/A4 rows
//                                      of the QSVD paper notes' tables)
//
// The quantiser is the integer step of the path and is bit-exact against its
// float32 definition: IEEE division (__fdiv_rn), fp16 round-to-nearest-even
// scale, round-half-even codes (__float2int_rn), symmetric clamp.
#include "internal.cuh"
#include "gemv.cuh"

namespace qsvd {
namespace {

// H2 = H_n (x) Q_m applied in place to v[r] (n = r/m): fast Walsh-Hadamard
// transform along a (element m*a + beta), scaled by 1/sqrt(n), then the m x m
// factor along beta.
__device__ void apply_h2_smem(float* v, int r, int m, const float* q, float scale) {
  const int n = r / m;
  for (int len = 1; len < n; len <<= 1) {
    for (int k = threadIdx.x; k < (n / 2) * m; k += blockDim.x) {
      const int beta = k % m, p = k / m;
      const int a0 = (p / len) * 2 * len + (p % len);
      const int i0 = a0 * m + beta, i1 = (a0 + len) * m + beta;
      const float u = v[i0], w = v[i1];
      v[i0] = u + w;
      v[i1] = u - w;
    }
    __syncthreads();
  }
  for (int a = threadIdx.x; a < n; a += blockDim.x) {
    float x[16], y[16];
    for (int b = 0; b < m; ++b) x[b] = v[a * m + b] * scale;
    for (int b = 0; b < m; ++b) {
      float s = 0.f;
      for (int bb = 0; bb < m; ++bb) s = fmaf(q[b * m + bb], x[bb], s);
      y[b] = s;
    }
    for (int b = 0; b < m; ++b) v[a * m + b] = y[b];
  }
  __syncthreads();
}

// grid (B), block 256.  cpart: KS x B x r partials of x W^d.
template <qsvd_dtype CT>
__global__ void __launch_bounds__(256)
k_append_finish(const float* __restrict__ cpart, int KS, const float* __restrict__ h2q,
                float h2_scale, int h2_m, int use_h2, const int32_t* __restrict__ pos,
                uint8_t* __restrict__ cache, __half* __restrict__ scales,
                float* __restrict__ c_out, int32_t* status, int B, int r, int max_len,
                int group) {
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  extern __shared__ float v[];   // r
  __shared__ float qm[256];
  const int b = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int j = threadIdx.x; j < r; j += 256)
    v[j] = dev::sum_strided(cpart + size_t(b) * r + j, size_t(B) * r, KS);
  if (use_h2) {
    for (int i = threadIdx.x; i < h2_m * h2_m; i += 256) qm[i] = h2q[i];
  }
  __syncthreads();
  if (use_h2) apply_h2_smem(v, r, h2_m, qm, h2_scale);
  if (c_out)
    for (int j = threadIdx.x; j < r; j += 256) c_out[size_t(b) * r + j] = v[j];
  const int p = pos[b];
  if (p < 0 || p >= max_len) {
    if (threadIdx.x == 0 && status) atomicOr(status, QSVD_STATUS_POS_OOB);
    return;
  }
  if (CT == QSVD_F32 || CT == QSVD_F16 || CT == QSVD_BF16) {
    for (int j = threadIdx.x; j < r; j += 256) {
      if (CT == QSVD_F32) reinterpret_cast<float*>(cache)[(size_t(b) * max_len + p) * r + j] = v[j];
      if (CT == QSVD_F16) reinterpret_cast<__half*>(cache)[(size_t(b) * max_len + p) * r + j] = __float2half_rn(v[j]);
      if (CT == QSVD_BF16) reinterpret_cast<__nv_bfloat16*>(cache)[(size_t(b) * max_len + p) * r + j] = __float2bfloat16_rn(v[j]);
    }
    return;
  }
  const int qmax = (CT == QSVD_I4) ? 7 : 127;
  const int ng = r / group;
  const size_t row = size_t(b) * max_len + p;
  // one warp per group
  for (int g = warp; g < ng; g += 8) {
    float amax = 0.f;
    for (int i = lane; i < group; i += 32) amax = fmaxf(amax, fabsf(v[g * group + i]));
    amax = dev::warp_max(amax);
    float s32 = __fdiv_rn(amax, float(qmax));
    if (s32 > 65504.f) {
      s32 = 65504.f;
      if (lane == 0 && status) atomicOr(status, QSVD_STATUS_SCALE_SAT);
    }
    const __half s16 = __float2half_rn(s32);
    const float sf = __half2float(s16);
    if (lane == 0) scales[row * ng + g] = s16;
    if (CT == QSVD_I8) {
      int8_t* dst = reinterpret_cast<int8_t*>(cache) + row * r + g * group;
      for (int i = lane; i < group; i += 32) {
        int q = 0;
        if (sf != 0.f) q = max(-qmax, min(qmax, __float2int_rn(__fdiv_rn(v[g * group + i], sf))));
        dst[i] = int8_t(q);
      }
    } else {
      uint8_t* dst = cache + row * (r / 2) + (g * group) / 2;
      for (int i = lane; i < group / 2; i += 32) {
        int q0 = 0, q1 = 0;
        if (sf != 0.f) {
          q0 = max(-qmax, min(qmax, __float2int_rn(__fdiv_rn(v[g * group + 2 * i], sf))));
          q1 = max(-qmax, min(qmax, __float2int_rn(__fdiv_rn(v[g * group + 2 * i + 1], sf))));
        }
        dst[i] = uint8_t((q0 & 0xF) | ((q1 & 0xF) << 4));
      }
    }
  }
}

// Without online H2 every group is independent: grid (B, r / chunk), one
// thread per channel of the chunk (chunk = the quantisation group for int
// caches).  Sums the split-K partials, writes c_out and the cache row.
template <qsvd_dtype CT>
__global__ void __launch_bounds__(1024)
k_append_chunk(const float* __restrict__ cpart, int KS, const int32_t* __restrict__ pos,
               uint8_t* __restrict__ cache, __half* __restrict__ scales,
               float* __restrict__ c_out, int32_t* status, int B, int r, int max_len,
               int chunk) {
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  __shared__ float wmax[32];
  const int b = blockIdx.x;
  const int j = blockIdx.y * chunk + threadIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float v = dev::sum_strided(cpart + size_t(b) * r + j, size_t(B) * r, KS);
  if (c_out) c_out[size_t(b) * r + j] = v;
  const int p = pos[b];
  if (p < 0 || p >= max_len) {
    if (threadIdx.x == 0 && blockIdx.y == 0 && status) atomicOr(status, QSVD_STATUS_POS_OOB);
    return;
  }
  const size_t row = size_t(b) * max_len + p;
  if (CT == QSVD_F32) { reinterpret_cast<float*>(cache)[row * r + j] = v; return; }
  if (CT == QSVD_F16) { reinterpret_cast<__half*>(cache)[row * r + j] = __float2half_rn(v); return; }
  if (CT == QSVD_BF16) {
    reinterpret_cast<__nv_bfloat16*>(cache)[row * r + j] = __float2bfloat16_rn(v);
    return;
  }
  // group amax over the chunk (== group)
  float a = dev::warp_max(fabsf(v));
  if (lane == 0) wmax[warp] = a;
  __syncthreads();
  if (warp == 0) {
    a = lane < int(blockDim.x >> 5) ? wmax[lane] : 0.f;
    a = dev::warp_max(a);
    if (lane == 0) wmax[0] = a;
  }
  __syncthreads();
  const int qmax = (CT == QSVD_I4) ? 7 : 127;
  float s32 = __fdiv_rn(wmax[0], float(qmax));
  if (s32 > 65504.f) {
    s32 = 65504.f;
    if (threadIdx.x == 0 && status) atomicOr(status, QSVD_STATUS_SCALE_SAT);
  }
  const __half s16 = __float2half_rn(s32);
  const float sf = __half2float(s16);
  if (threadIdx.x == 0) scales[row * (r / chunk) + blockIdx.y] = s16;
  int q = 0;
  if (sf != 0.f) q = max(-qmax, min(qmax, __float2int_rn(__fdiv_rn(v, sf))));
  if (CT == QSVD_I8) {
    reinterpret_cast<int8_t*>(cache)[row * r + j] = int8_t(q);
  } else {
    const int hi = __shfl_down_sync(0xffffffffu, q, 1);   // partner element j + 1
    if ((j & 1) == 0) cache[row * (r / 2) + j / 2] = uint8_t((q & 0xF) | ((hi & 0xF) << 4));
  }
}

template <typename WT>
cudaError_t gemv_t(const qsvd_dims& d, const void* x, const void* wd, float* cpart, int KS,
                   int32_t* status, cudaStream_t s) {
  // W^u_q and W^u_k follow W^d in the packed weights: the decode's query
  // GEMV and absorption read them next, so they are requested into L2 here
  const PackedLayout L = packed_layout(d);
  const uint8_t* wq = static_cast<const uint8_t*>(wd) + (L.wuq - L.wd);
  const size_t pf_bytes = L.wuk + size_t(d.E) * d.r * sizeof(WT) - L.wuq;
  return launch_gemv<WT, WT>(static_cast<const WT*>(x), static_cast<const WT*>(wd), cpart, d.batch,
                             d.E, d.r, KS, static_cast<float*>(nullptr), nullptr, status, s, XGroups{0, 0, 0},
                             wq, pf_bytes);
}

int append_chunk(const qsvd_dims& d) {
  if (d.cache_dtype == QSVD_I8 || d.cache_dtype == QSVD_I4) return d.group;
  for (int c : {256, 128, 64, 32})
    if (d.r % c == 0) return c;
  return 32;
}

template <qsvd_dtype CT>
cudaError_t finish_t(const qsvd_dims& d, const float* cpart, int KS, const float* h2q,
                     float h2_scale, const int32_t* pos, void* cache, void* scales,
                     float* c_out, int32_t* status, cudaStream_t s) {
  if (!d.h2) {
    const int chunk = append_chunk(d);
    dim3 grid(d.batch, d.r / chunk);
    {
      const cudaError_t le = launch_pdl(k_append_chunk<CT>, dim3(grid), dim3(chunk), 0, s,
                                       cpart, KS, pos, static_cast<uint8_t*>(cache), static_cast<__half*>(scales), c_out, status, d.batch, d.r, d.max_len, chunk);
      if (le != cudaSuccess) return le;
    }
    note_launch();
    return check_launch();
  }
  const size_t smem = size_t(d.r) * 4;
  auto kern = k_append_finish<CT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  {
    const cudaError_t le = launch_pdl(kern, dim3(d.batch), dim3(256), smem, s,
                                     cpart, KS, h2q, h2_scale, d.h2_m, d.h2 ? 1 : 0, pos, static_cast<uint8_t*>(cache), static_cast<__half*>(scales), c_out, status, d.batch, d.r, d.max_len, d.group);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return check_launch();
}

}  // namespace

int append_ksplit(const qsvd_dims& d) { return gemv_ksplit(d.E, d.weight_dtype); }

cudaError_t launch_append(const qsvd_dims& d, const void* x, const void* wd,
                          const float* h2q, float h2_scale, const int32_t* pos,
                          void* cache, void* scales, float* c_out, float* cpart,
                          int KS, int32_t* status, cudaStream_t s) {
  cudaError_t e;
  switch (d.weight_dtype) {
    case QSVD_F32: e = gemv_t<float>(d, x, wd, cpart, KS, status, s); break;
    case QSVD_F16: e = gemv_t<__half>(d, x, wd, cpart, KS, status, s); break;
    case QSVD_BF16: e = gemv_t<__nv_bfloat16>(d, x, wd, cpart, KS, status, s); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  switch (d.cache_dtype) {
    case QSVD_F32: return finish_t<QSVD_F32>(d, cpart, KS, h2q, h2_scale, pos, cache, scales, c_out, status, s);
    case QSVD_F16: return finish_t<QSVD_F16>(d, cpart, KS, h2q, h2_scale, pos, cache, scales, c_out, status, s);
    case QSVD_BF16: return finish_t<QSVD_BF16>(d, cpart, KS, h2q, h2_scale, pos, cache, scales, c_out, status, s);
    case QSVD_I8: return finish_t<QSVD_I8>(d, cpart, KS, h2q, h2_scale, pos, cache, scales, c_out, status, s);
    case QSVD_I4: return finish_t<QSVD_I4>(d, cpart, KS, h2q, h2_scale, pos, cache, scales, c_out, status, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace qsvd
