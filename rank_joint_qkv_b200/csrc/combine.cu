// Combine phase: merge the split partials of each sequence and apply the
// value up-projection once per step.
//
//   M = max_s m_s,  w_s = 2^(m_s - M),  z_h = sum_s w_s z_s,h / sum_s w_s l_s,h
//   o_h = z_h W^u_{v,h}
//
// Flash decoding's log-sum-exp merge (WSVD digest, Method 3.4) in the latent
// space; values are never materialised, V = C W^u_v is applied to the merged
// latent (QSVD digest, Method, Step 1).  W^u_v is read exactly once per step:
// CTA (h, js) owns rows [128 js, 128 js + 128) of head h's columns and
// handles every sequence.  The per-split weights are computed first (one warp
// per sequence), so the partial loads that follow are independent.
#include "internal.cuh"

namespace qsvd {
namespace {

constexpr int kJ = 128;   // latent rows (of W^u_v) per CTA
constexpr int kBC = 16;   // sequences per pass

// grid (H, ceil(r / kJ)), block 256.
// smem: ws[kJ][d_h] W^u_v tile (float), zs[kBC][kJ] merged latents,
//       red[KSP][kBC][d_h] partial outputs, wt[P] per-slot merge weight
//       2^(m_s - M) / L (indexed by slot), seg[B][2] slot ranges.
template <typename WT>
__global__ void __launch_bounds__(256)
k_combine_vup(const WsHeader* __restrict__ hdr, const int32_t* __restrict__ sched,
              const float* __restrict__ pm, const float* __restrict__ pl,
              const float* __restrict__ pz, const WT* __restrict__ wuv,
              float* __restrict__ opart, int B, int H, int d_h, int r, int E, int P) {
  extern __shared__ float sm[];
  const int DQ = d_h / 4;                 // output quads per sequence
  const int KSP = 256 / (4 * DQ);         // k-splits of the V-up tile
  float* ws = sm;                         // kJ * d_h
  float* zs = ws + kJ * d_h;              // kBC * kJ
  float* red = zs + kBC * kJ;             // KSP * kBC * d_h
  float* wt = red + KSP * kBC * d_h;      // P
  int* seg = reinterpret_cast<int*>(wt + P);   // B x {c0, c1}
  const int h = blockIdx.x;
  const int js = blockIdx.y;
  const int j0 = js * kJ;
  const int jn = min(kJ, r - j0);
  const long long G = hdr->G;
  const int32_t* tstart = sched;
  const long long T = tstart[B];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // W^u_v tile, 16-byte loads
  {
    constexpr int V = 16 / int(sizeof(WT));
    const int vpr = d_h / V;
    for (int i = threadIdx.x; i < kJ * vpr; i += 256) {
      const int jj = i / vpr, v = i % vpr;
      float f[V];
      if (jj < jn) {
        const uint4 raw = *reinterpret_cast<const uint4*>(wuv + size_t(j0 + jj) * E + h * d_h + v * V);
        const WT* e = reinterpret_cast<const WT*>(&raw);
#pragma unroll
        for (int k = 0; k < V; ++k) f[k] = dev::to_f(e[k]);
      } else {
#pragma unroll
        for (int k = 0; k < V; ++k) f[k] = 0.f;
      }
#pragma unroll
      for (int k = 0; k < V; ++k) ws[jj * d_h + v * V + k] = f[k];
    }
  }
  // merge weights, one warp per sequence; lane i holds slots c0 + i + 32 k
  for (int b = warp; b < B; b += 8) {
    const long long t0 = tstart[b], t1 = tstart[b + 1];
    int c0 = 0, c1 = -1;
    if (t1 > t0) {
      c0 = int(dev::split_of_tile(t0, G, T));
      c1 = int(dev::split_of_tile(t1 - 1, G, T));
    }
    if (lane == 0) { seg[2 * b] = c0; seg[2 * b + 1] = c1; }
    constexpr int NR = 4;
    float mv[NR], lv[NR];
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      const int c = c0 + lane + 32 * k;
      mv[k] = -INFINITY;
      lv[k] = 0.f;
      if (c <= c1 && dev::split_begin(c, G, T) != dev::split_begin(c + 1, G, T)) {
        mv[k] = pm[(size_t(c) + b) * H + h];
        lv[k] = pl[(size_t(c) + b) * H + h];
      }
      M = fmaxf(M, mv[k]);
    }
    for (int c = c0 + lane + 32 * NR; c <= c1; c += 32)   // long runs of splits
      if (dev::split_begin(c, G, T) != dev::split_begin(c + 1, G, T))
        M = fmaxf(M, pm[(size_t(c) + b) * H + h]);
    M = dev::warp_max(M);
    float L = 0.f;
#pragma unroll
    for (int k = 0; k < NR; ++k) L += exp2f(mv[k] - M) * lv[k];
    for (int c = c0 + lane + 32 * NR; c <= c1; c += 32)
      if (dev::split_begin(c, G, T) != dev::split_begin(c + 1, G, T))
        L += exp2f(pm[(size_t(c) + b) * H + h] - M) * pl[(size_t(c) + b) * H + h];
    L = dev::warp_sum(L);
    const float invL = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      const int c = c0 + lane + 32 * k;
      if (c <= c1) wt[c + b] = exp2f(mv[k] - M) * invL;
    }
    for (int c = c0 + lane + 32 * NR; c <= c1; c += 32) {
      const bool live = dev::split_begin(c, G, T) != dev::split_begin(c + 1, G, T);
      wt[c + b] = live ? exp2f(pm[(size_t(c) + b) * H + h] - M) * invL : 0.f;
    }
  }
  __syncthreads();
  const int jj = threadIdx.x & (kJ - 1);
  const int bsub = threadIdx.x / kJ;          // 0 or 1
  // V-up tile: thread -> 4 sequences x 4 output dims over one k-split
  const int ksp = threadIdx.x / (4 * DQ);
  const int bq = (threadIdx.x % (4 * DQ)) / DQ;
  const int dq = threadIdx.x % DQ;
  const int kper = kJ / KSP;
  for (int bc = 0; bc < B; bc += kBC) {
    const int bn = min(kBC, B - bc);
    // merged latent z[b][j] = sum_s w_s z_s[j]; the loads are independent
    for (int bb = bsub; bb < kBC; bb += 2) {
      const int b = bc + bb;
      float z = 0.f;
      if (bb < bn && jj < jn) {
        const int c0 = seg[2 * b], c1 = seg[2 * b + 1];
        // loads in batches of 8 so that they are in flight together
        for (int cb = c0; cb <= c1; cb += 8) {
          float v[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            v[i] = (cb + i <= c1 && wt[cb + i + b] != 0.f)
                       ? __ldcg(pz + ((size_t(cb + i) + b) * H + h) * r + j0 + jj) : 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (cb + i <= c1) z = fmaf(wt[cb + i + b], v[i], z);
        }
      }
      zs[bb * kJ + jj] = z;
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
    const int kend = ksp < KSP ? (ksp + 1) * kper : 0;   // spare threads when 256 % d_h != 0
    for (int k = ksp * kper; k < kend; ++k) {
      const float4 w4 = *reinterpret_cast<const float4*>(&ws[k * d_h + 4 * dq]);
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float z = zs[(4 * bq + a) * kJ + k];
        acc[a][0] = fmaf(z, w4.x, acc[a][0]);
        acc[a][1] = fmaf(z, w4.y, acc[a][1]);
        acc[a][2] = fmaf(z, w4.z, acc[a][2]);
        acc[a][3] = fmaf(z, w4.w, acc[a][3]);
      }
    }
    if (ksp < KSP) {
#pragma unroll
      for (int a = 0; a < 4; ++a)
        *reinterpret_cast<float4*>(&red[(ksp * kBC + 4 * bq + a) * d_h + 4 * dq]) =
            make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < bn * d_h; i += 256) {
      const int bb = i / d_h, dd = i % d_h;
      float o = 0.f;
      for (int k = 0; k < KSP; ++k) o += red[(k * kBC + bb) * d_h + dd];
      opart[(size_t(js) * B + bc + bb) * E + h * d_h + dd] = o;
    }
    __syncthreads();
  }
}

template <typename OT>
__global__ void __launch_bounds__(256)
k_combine_out(const float* __restrict__ opart, int JS, OT* __restrict__ out, size_t n) {
  const size_t i = size_t(blockIdx.x) * 256 + threadIdx.x;
  if (i >= n) return;
  out[i] = dev::from_f<OT>(dev::sum_strided(opart + i, n, JS));
}

template <typename WT>
cudaError_t vup_t(const qsvd_dims& d, const WsHeader* hdr, const int32_t* sched,
                  const float* pm, const float* pl, const float* pz, const void* wuv,
                  float* opart, int JS, int P, cudaStream_t s) {
  const int ksp = 256 / d.d_h;   // k-splits of the V-up tile (4 x 4 outputs per thread)
  const size_t smem = (size_t(kJ) * d.d_h + size_t(kBC) * kJ + size_t(ksp) * kBC * d.d_h + P) * 4 +
                      size_t(d.batch) * 8;
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  auto kern = k_combine_vup<WT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(d.H, JS);
  kern<<<grid, 256, smem, s>>>(hdr, sched, pm, pl, pz, static_cast<const WT*>(wuv), opart,
                               d.batch, d.H, d.d_h, d.r, d.E, P);
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
                           const void* wuv, float* opart, int JS, int P, void* out,
                           cudaStream_t s) {
  cudaError_t e;
  switch (d.weight_dtype) {
    case QSVD_F32: e = vup_t<float>(d, hdr, sched, pm, pl, pz, wuv, opart, JS, P, s); break;
    case QSVD_F16: e = vup_t<__half>(d, hdr, sched, pm, pl, pz, wuv, opart, JS, P, s); break;
    case QSVD_BF16: e = vup_t<__nv_bfloat16>(d, hdr, sched, pm, pl, pz, wuv, opart, JS, P, s); break;
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
