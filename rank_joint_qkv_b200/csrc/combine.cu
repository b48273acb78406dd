// Combine phase: merge the split partials of each sequence and apply the
// value up-projection once per step.
//
//   M = max_s m_s,  w_s = 2^(m_s - M),  z_h = sum_s w_s z_s,h / sum_s w_s l_s,h
//   o_h = z_h W^u_{v,h}
//
// Flash decoding's log-sum-exp merge (WSVD digest, Method 3.4) in the latent
// space; values are never materialised, V = C W^u_v is applied to the merged
// latent (QSVD digest, Method, Step 1).  W^u_v is read exactly once per step:
// CTA (h, js) owns rows [256 js, 256 js + 256) of head h's columns and
// handles every sequence.
#include "internal.cuh"

namespace qsvd {
namespace {

constexpr int kJ = 256;   // latent rows per CTA

template <typename WT>
__global__ void __launch_bounds__(256)
k_combine_vup(const WsHeader* __restrict__ hdr, const int32_t* __restrict__ sched,
              const float* __restrict__ pm, const float* __restrict__ pl,
              const float* __restrict__ pz, const WT* __restrict__ wuv,
              float* __restrict__ opart, int B, int H, int d_h, int r, int E) {
  extern __shared__ float sm[];
  float* ws = sm;                 // [kJ][d_h]
  float* zsm = ws + kJ * d_h;     // [kJ]
  float* osm = zsm + kJ;          // [2][d_h]
  const int h = blockIdx.x;
  const int js = blockIdx.y;
  const int j0 = js * kJ;
  const int jn = min(kJ, r - j0);
  const long long G = hdr->G;
  const int32_t* tstart = sched;
  const long long T = tstart[B];

  for (int i = threadIdx.x; i < kJ * d_h; i += 256) {
    const int jj = i / d_h, dd = i % d_h;
    ws[i] = jj < jn ? dev::to_f(wuv[size_t(j0 + jj) * E + h * d_h + dd]) : 0.f;
  }
  const int j = j0 + threadIdx.x;
  for (int b = 0; b < B; ++b) {
    const long long t0 = tstart[b], t1 = tstart[b + 1];
    float z = 0.f;
    if (t1 > t0) {
      const long long c0 = dev::split_of_tile(t0, G, T);
      const long long c1 = dev::split_of_tile(t1 - 1, G, T);
      float M = -INFINITY;
      for (long long c = c0; c <= c1; ++c) {
        if (dev::split_begin(c, G, T) == dev::split_begin(c + 1, G, T)) continue;
        M = fmaxf(M, pm[(size_t(c) + b) * H + h]);
      }
      float L = 0.f, acc = 0.f;
      for (long long c = c0; c <= c1; ++c) {
        if (dev::split_begin(c, G, T) == dev::split_begin(c + 1, G, T)) continue;
        const size_t slot = size_t(c) + b;
        const float w = exp2f(pm[slot * H + h] - M);
        L = fmaf(w, pl[slot * H + h], L);
        if (threadIdx.x < jn) acc = fmaf(w, pz[(slot * H + h) * r + j], acc);
      }
      z = L > 0.f ? acc / L : 0.f;
    }
    __syncthreads();
    zsm[threadIdx.x] = threadIdx.x < jn ? z : 0.f;
    __syncthreads();
    // o[d] = sum_jj z[jj] * W[jj][d]; two threads per output dim
    for (int i = threadIdx.x; i < 2 * d_h; i += 256) {
      const int dd = i % d_h, half = i / d_h;
      float o = 0.f;
      const int jb = half * (kJ / 2);
      for (int jj = jb; jj < jb + kJ / 2; ++jj) o = fmaf(zsm[jj], ws[jj * d_h + dd], o);
      osm[half * d_h + dd] = o;
    }
    __syncthreads();
    for (int dd = threadIdx.x; dd < d_h; dd += 256)
      opart[(size_t(js) * B + b) * E + h * d_h + dd] = osm[dd] + osm[d_h + dd];
  }
}

template <typename OT>
__global__ void __launch_bounds__(256)
k_combine_out(const float* __restrict__ opart, int JS, OT* __restrict__ out, size_t n) {
  const size_t i = size_t(blockIdx.x) * 256 + threadIdx.x;
  if (i >= n) return;
  float s = 0.f;
  for (int k = 0; k < JS; ++k) s += opart[size_t(k) * n + i];
  out[i] = dev::from_f<OT>(s);
}

template <typename WT>
cudaError_t vup_t(const qsvd_dims& d, const WsHeader* hdr, const int32_t* sched,
                  const float* pm, const float* pl, const float* pz, const void* wuv,
                  float* opart, int JS, cudaStream_t s) {
  const size_t smem = (size_t(kJ) * d.d_h + kJ + 2 * d.d_h) * 4;
  auto kern = k_combine_vup<WT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(d.H, JS);
  kern<<<grid, 256, smem, s>>>(hdr, sched, pm, pl, pz, static_cast<const WT*>(wuv), opart,
                               d.batch, d.H, d.d_h, d.r, d.E);
  note_launch();
  return check_launch();
}

template <typename OT>
cudaError_t out_t(const qsvd_dims& d, const float* opart, int JS, void* out, cudaStream_t s) {
  const size_t n = size_t(d.batch) * d.E;
  k_combine_out<OT><<<unsigned((n + 255) / 256), 256, 0, s>>>(opart, JS, static_cast<OT*>(out), n);
  note_launch();
  return check_launch();
}

}  // namespace

cudaError_t launch_combine(const qsvd_dims& d, const WsHeader* hdr, const int32_t* sched,
                           const float* pm, const float* pl, const float* pz,
                           const void* wuv, float* opart, int JS, void* out,
                           cudaStream_t s) {
  cudaError_t e;
  switch (d.weight_dtype) {
    case QSVD_F32: e = vup_t<float>(d, hdr, sched, pm, pl, pz, wuv, opart, JS, s); break;
    case QSVD_F16: e = vup_t<__half>(d, hdr, sched, pm, pl, pz, wuv, opart, JS, s); break;
    case QSVD_BF16: e = vup_t<__nv_bfloat16>(d, hdr, sched, pm, pl, pz, wuv, opart, JS, s); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  switch (d.out_dtype) {
    case QSVD_F32: return out_t<float>(d, opart, JS, out, s);
    case QSVD_F16: return out_t<__half>(d, opart, JS, out, s);
    case QSVD_BF16: return out_t<__nv_bfloat16>(d, opart, JS, out, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qsvd
