// Weight preparation (one-off per model layer).
//
// Copies the joint-SVD factors into one packed device buffer, optionally
// folds the rotation H2 = H_n (x) Q_m into them (QSVD paper notes, 关键设计:
// Y = (X H1^T)(H1 W^d H2^T)(H2 W^u)), stores W^u_k transposed for the rotary
// tensor-core kernel and a float32 cos/sin table whose angles are formed in
// float64 (positions up to 32k lose ~2^-9 rad if formed in float32).
#include <algorithm>
#include <cmath>

#include "internal.cuh"

namespace qsvd {
namespace {

// Apply H2 to NV vectors of length r stored with element stride es and
// vector stride vs: v <- H2 v.  grid ceil(nvec/NV), block 256.
template <typename WT>
__global__ void __launch_bounds__(256)
k_h2_fold(WT* __restrict__ base, int nvec, size_t es, size_t vs, int r, int m,
          const float* __restrict__ q, float scale) {
  constexpr int NV = 4;
  extern __shared__ float v[];   // NV x r
  __shared__ float qm[256];
  const int v0 = blockIdx.x * NV;
  const int nv = min(NV, nvec - v0);
  for (int i = threadIdx.x; i < m * m; i += 256) qm[i] = q[i];
  for (int i = threadIdx.x; i < NV * r; i += 256) {
    const int k = i / r, j = i % r;
    v[i] = k < nv ? dev::to_f(base[size_t(v0 + k) * vs + size_t(j) * es]) : 0.f;
  }
  __syncthreads();
  const int n = r / m;
  for (int len = 1; len < n; len <<= 1) {
    for (int idx = threadIdx.x; idx < NV * (n / 2) * m; idx += 256) {
      const int k = idx / ((n / 2) * m), rem = idx % ((n / 2) * m);
      const int beta = rem % m, p = rem / m;
      const int a0 = (p / len) * 2 * len + (p % len);
      float* vk = v + k * r;
      const int i0 = a0 * m + beta, i1 = (a0 + len) * m + beta;
      const float u = vk[i0], w = vk[i1];
      vk[i0] = u + w;
      vk[i1] = u - w;
    }
    __syncthreads();
  }
  for (int idx = threadIdx.x; idx < NV * n; idx += 256) {
    const int k = idx / n, a = idx % n;
    float* vk = v + k * r;
    float x[16], y[16];
    for (int b = 0; b < m; ++b) x[b] = vk[a * m + b] * scale;
    for (int b = 0; b < m; ++b) {
      float s = 0.f;
      for (int bb = 0; bb < m; ++bb) s = fmaf(qm[b * m + bb], x[bb], s);
      y[b] = s;
    }
    for (int b = 0; b < m; ++b) vk[a * m + b] = y[b];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < NV * r; i += 256) {
    const int k = i / r, j = i % r;
    if (k < nv) base[size_t(v0 + k) * vs + size_t(j) * es] = dev::from_f<WT>(v[i]);
  }
}

// dst[e][j] = src[j][e]  (src r x E)
template <typename WT>
__global__ void k_transpose(const WT* __restrict__ src, WT* __restrict__ dst, int r, int E) {
  __shared__ WT t[32][33];
  const int e0 = blockIdx.x * 32, j0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int j = j0 + i, e = e0 + threadIdx.x;
    if (j < r && e < E) t[i][threadIdx.x] = src[size_t(j) * E + e];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int e = e0 + i, j = j0 + threadIdx.x;
    if (j < r && e < E) dst[size_t(e) * r + j] = t[threadIdx.x][i];
  }
}

// tab[pos][i] = {cos, sin}(pos * base^(-2i/d_h)), angles in float64.
__global__ void k_rope_table(float* __restrict__ tab, int max_len, int half, double log_base,
                             int d_h) {
  const size_t n = size_t(max_len) * half;
  for (size_t idx = size_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < n;
       idx += size_t(gridDim.x) * blockDim.x) {
    const int pos = int(idx / half), i = int(idx % half);
    const double theta = exp(-(2.0 * i / d_h) * log_base);
    double s, c;
    sincos(double(pos) * theta, &s, &c);
    tab[idx * 2 + 0] = float(c);
    tab[idx * 2 + 1] = float(s);
  }
}

// Per-head fold of the value up-projection into the output projection (WSVD
// digest, Method, fused kernel §3.4): F[h r + j][n] = sum_i V_h[j][i]
// W_O[h d_h + i][n], with V_h[j][i] at v[j sj + h sh + i]: the head's d_h
// columns of the shared W^u_v (sj = E, sh = d_h) or the per-head factor
// B_{Vh} stacked by head (sj = d_h, sh = r d_h).  One 64 x 64 tile of F per
// CTA (grid ceil(E/64), ceil(r/64), H; block 16 x 16, 4 x 4 outputs per
// thread); i runs in order, fp32 fma, rounded once to WT.
template <typename WT>
__global__ void __launch_bounds__(256)
k_fold_vo(const WT* __restrict__ wuv, const WT* __restrict__ wo, WT* __restrict__ f, int E, int r,
          int d_h, long long sj, long long sh) {
  __shared__ float as[64][33];   // [j][i]
  __shared__ float bs[32][65];   // [i][n]
  const int n0 = blockIdx.x * 64, j0 = blockIdx.y * 64, h = blockIdx.z;
  const int tx = threadIdx.x, ty = threadIdx.y, t = ty * 16 + tx;
  float acc[4][4] = {};
  for (int i0 = 0; i0 < d_h; i0 += 32) {
    for (int k = t; k < 64 * 32; k += 256) {
      const int jj = k / 32, ii = k % 32;
      const int j = j0 + jj, i = i0 + ii;
      as[jj][ii] = (j < r && i < d_h) ? dev::to_f(wuv[size_t(j) * sj + size_t(h) * sh + i]) : 0.f;
    }
    for (int k = t; k < 32 * 64; k += 256) {
      const int ii = k / 64, nn = k % 64;
      const int i = i0 + ii, n = n0 + nn;
      bs[ii][nn] = (i < d_h && n < E) ? dev::to_f(wo[(size_t(h) * d_h + i) * E + n]) : 0.f;
    }
    __syncthreads();
    const int iend = min(32, d_h - i0);
    for (int ii = 0; ii < iend; ++ii) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) { a[u] = as[ty * 4 + u][ii]; b[u] = bs[ii][tx * 4 + u]; }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = j0 + ty * 4 + u;
    if (j >= r) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int n = n0 + tx * 4 + v;
      if (n < E) f[(size_t(h) * r + j) * E + n] = dev::from_f<WT>(acc[u][v]);
    }
  }
}

template <typename WT>
cudaError_t fold_vo_t(const qsvd_dims& d, const void* wuv, const void* wo, void* f, cudaStream_t s,
                      bool per_head = false) {
  const dim3 grid((d.E + 63) / 64, (d.r + 63) / 64, d.H);
  const long long sj = per_head ? d.d_h : d.E, sh = per_head ? (long long)d.r * d.d_h : d.d_h;
  k_fold_vo<WT><<<grid, dim3(16, 16), 0, s>>>(static_cast<const WT*>(wuv), static_cast<const WT*>(wo),
                                              static_cast<WT*>(f), d.E, d.r, d.d_h, sj, sh);
  note_launch();
  return check_launch();
}

template <typename WT>
cudaError_t fold_t(WT* base, int nvec, size_t es, size_t vs, int r, int m, const float* q,
                   float scale, cudaStream_t s) {
  const size_t smem = size_t(4) * r * 4;
  auto kern = k_h2_fold<WT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  kern<<<(nvec + 3) / 4, 256, smem, s>>>(base, nvec, es, vs, r, m, q, scale);
  note_launch();
  return check_launch();
}

template <typename WT>
cudaError_t prepare_t(const qsvd_dims& d, const float* h2q_host, uint8_t* P,
                      const PackedLayout& L, cudaStream_t s) {
  cudaError_t e;
  WT* wd = reinterpret_cast<WT*>(P + L.wd);
  WT* wu[3] = {reinterpret_cast<WT*>(P + L.wuq), reinterpret_cast<WT*>(P + L.wuk),
               reinterpret_cast<WT*>(P + L.wuv)};
  float* q = reinterpret_cast<float*>(P + L.h2q);
  if (h2q_host) {
    const int m = d.h2_m;
    e = cudaMemcpyAsync(q, h2q_host, size_t(m) * m * 4, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return e;
    const double n = double(d.r / m);
    const float scale = float(1.0 / std::sqrt(n));
    for (int k = 0; k < 3; ++k) {   // W^u_* <- H2 W^u_*: columns are vectors
      e = fold_t<WT>(wu[k], d.E, size_t(d.E), 1, d.r, m, q, scale, s);
      if (e != cudaSuccess) return e;
    }
    if (!d.h2) {                     // W^d <- W^d H2^T: rows are vectors
      e = fold_t<WT>(wd, d.E, 1, size_t(d.r), d.r, m, q, scale, s);
      if (e != cudaSuccess) return e;
    }
  }
  if (d.rope) {
    dim3 grid((d.E + 31) / 32, (d.r + 31) / 32);
    k_transpose<WT><<<grid, dim3(32, 8), 0, s>>>(wu[1], reinterpret_cast<WT*>(P + L.wukT), d.r, d.E);
    note_launch();
    if ((e = check_launch()) != cudaSuccess) return e;
    const int half = d.d_h / 2;
    const size_t n = size_t(d.max_len) * half;
    const unsigned blocks = unsigned(std::min<size_t>((n + 255) / 256, 4096));
    k_rope_table<<<blocks, 256, 0, s>>>(reinterpret_cast<float*>(P + L.rope), d.max_len, half,
                                        std::log(double(d.rope_base)), d.d_h);
    note_launch();
    if ((e = check_launch()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_prepare(const qsvd_dims& d, const void* wd, const void* wuq,
                           const void* wuk, const void* wuv, const float* h2q_host,
                           void* packed, const PackedLayout& L, cudaStream_t s) {
  uint8_t* P = static_cast<uint8_t*>(packed);
  const size_t mat = size_t(d.E) * d.r * dtype_bytes(d.weight_dtype);
  const void* src[4] = {wd, wuq, wuk, wuv};
  const size_t off[4] = {L.wd, L.wuq, L.wuk, L.wuv};
  for (int k = 0; k < 4; ++k) {
    cudaError_t e = cudaMemcpyAsync(P + off[k], src[k], mat, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return e;
  }
  switch (d.weight_dtype) {
    case QSVD_F32: return prepare_t<float>(d, h2q_host, P, L, s);
    case QSVD_F16: return prepare_t<__half>(d, h2q_host, P, L, s);
    case QSVD_BF16: return prepare_t<__nv_bfloat16>(d, h2q_host, P, L, s);
    default: return cudaErrorInvalidValue;
  }
}

namespace {

// wd[e][j] = u[e][j] a[j] (E x r); wu_k[j][n] = b[j] vt[j][k E + n] for
// k = q, k, v (r x E each).  Grid-stride over the 4 r E outputs.
template <typename WT>
__global__ void __launch_bounds__(256)
k_split_factors(const float* __restrict__ u, const float* __restrict__ vt, const float* __restrict__ a,
                const float* __restrict__ b, WT* __restrict__ wd, WT* __restrict__ wuq, WT* __restrict__ wuk,
                WT* __restrict__ wuv, int E, int r) {
  const size_t m = size_t(E) * r;
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < 4 * m;
       i += size_t(gridDim.x) * blockDim.x) {
    if (i < m) {
      wd[i] = dev::from_f<WT>(u[i] * a[i % r]);
    } else {
      const size_t t = i - m;
      const int k = int(t / m);              // 0: q, 1: k, 2: v
      const size_t rem = t % m;
      const int j = int(rem / E), n = int(rem % E);
      WT* dst = k == 0 ? wuq : (k == 1 ? wuk : wuv);
      dst[rem] = dev::from_f<WT>(b[j] * vt[size_t(j) * 3 * E + size_t(k) * E + n]);
    }
  }
}

// The split exponents of one beta: a_j = float(sigma_j^beta), b_j =
// float(sigma_j^(1 - beta)), powers in float64.  One CTA, r <= 8192.
__global__ void __launch_bounds__(256)
k_beta_split(const float* __restrict__ sigma, double beta, float* __restrict__ a, float* __restrict__ b, int r) {
  for (int j = threadIdx.x; j < r; j += blockDim.x) {
    const double sj = double(sigma[j]);
    a[j] = float(pow(sj, beta));
    b[j] = float(pow(sj, 1.0 - beta));
  }
}

// sum over i of (y_i - yq_i)^2 in float64, added into *out (zeroed first).
__global__ void __launch_bounds__(256)
k_sq_diff_sum(const float* __restrict__ y, const float* __restrict__ yq, size_t n, double* __restrict__ out) {
  __shared__ double red[8];
  double acc = 0.0;
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += size_t(gridDim.x) * blockDim.x) {
    const double d = double(y[i]) - double(yq[i]);
    acc = fma(d, d, acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < int(blockDim.x >> 5); ++w) t += red[w];
    atomicAdd(out, t);
  }
}

template <typename WT>
cudaError_t split_factors_t(const qsvd_dims& d, const float* u, const float* vt, const float* a,
                            const float* b, void* wd, void* wuq, void* wuk, void* wuv, cudaStream_t s) {
  const size_t n = size_t(4) * d.E * d.r;
  const unsigned blocks = unsigned(std::min<size_t>((n + 255) / 256, 148 * 16));
  k_split_factors<WT><<<blocks, 256, 0, s>>>(u, vt, a, b, static_cast<WT*>(wd), static_cast<WT*>(wuq),
                                             static_cast<WT*>(wuk), static_cast<WT*>(wuv), d.E, d.r);
  note_launch();
  return check_launch();
}

}  // namespace

cudaError_t launch_split_factors(const qsvd_dims& d, const float* u, const float* vt, const float* a,
                                 const float* b, void* wd, void* wuq, void* wuk, void* wuv,
                                 cudaStream_t s) {
  switch (d.weight_dtype) {
    case QSVD_F32: return split_factors_t<float>(d, u, vt, a, b, wd, wuq, wuk, wuv, s);
    case QSVD_F16: return split_factors_t<__half>(d, u, vt, a, b, wd, wuq, wuk, wuv, s);
    case QSVD_BF16: return split_factors_t<__nv_bfloat16>(d, u, vt, a, b, wd, wuq, wuk, wuv, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_beta_split(const float* sigma, double beta, float* a, float* b, int r, cudaStream_t s) {
  k_beta_split<<<1, 256, 0, s>>>(sigma, beta, a, b, r);
  note_launch();
  return check_launch();
}

cudaError_t launch_sq_diff_sum(const float* y, const float* yq, size_t n, double* out, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(out, 0, sizeof(double), s);
  if (e != cudaSuccess) return e;
  const unsigned blocks = unsigned(std::min<size_t>((n + 255) / 256, 148 * 4));
  k_sq_diff_sum<<<blocks > 0 ? blocks : 1, 256, 0, s>>>(y, yq, n, out);
  note_launch();
  return check_launch();
}

cudaError_t launch_prepare_out_proj(const qsvd_dims& d, const void* wo, void* packed,
                                    const PackedLayout& L, cudaStream_t s) {
  uint8_t* P = static_cast<uint8_t*>(packed);
  if (d.out_proj == QSVD_OUT_PROJ_CHAIN)
    return cudaMemcpyAsync(P + L.wo, wo, size_t(d.E) * d.E * dtype_bytes(d.weight_dtype),
                           cudaMemcpyDeviceToDevice, s);
  switch (d.weight_dtype) {
    case QSVD_F16: return fold_vo_t<__half>(d, P + L.wuv, wo, P + L.wo, s);
    case QSVD_BF16: return fold_vo_t<__nv_bfloat16>(d, P + L.wuv, wo, P + L.wo, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_per_head_fold(const qsvd_dims& d, const void* bv, const void* wo, void* f, cudaStream_t s) {
  switch (d.weight_dtype) {
    case QSVD_F16: return fold_vo_t<__half>(d, bv, wo, f, s, true);
    case QSVD_BF16: return fold_vo_t<__nv_bfloat16>(d, bv, wo, f, s, true);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_rope_table(float* tab, int max_len, int d_h, float base, cudaStream_t s) {
  const int half = d_h / 2;
  const size_t n = size_t(max_len) * half;
  const unsigned blocks = unsigned(std::min<size_t>((n + 255) / 256, 4096));
  k_rope_table<<<blocks, 256, 0, s>>>(tab, max_len, half, std::log(double(base)), d_h);
  note_launch();
  return check_launch();
}

}  // namespace qsvd
