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
#include "gemv.cuh"
#include "internal.cuh"

namespace qsvd {
namespace {

// ----------------------------------------------- merge, then V-up GEMV
//
// For 16-bit weights with d_h a multiple of 64 the two steps run as two
// kernels: the merge, wide (one CTA per 512 channels of one (sequence,
// head), four channels per thread), writes the merged latent
// zm[b][h][r] = sum_s w_s z_s (w_s = 2^(m_s - M) / L); the V-up is the
// tensor-core GEMV with head h's output columns reading row zm[b][h].

constexpr int kMergeCh = 512;   // channels per merge CTA (128 threads x 4)
constexpr int kMergeMaxSplits = kMaxSplits;   // weights kept in shared memory per (b, h): c1 - c0 < G

// grid (ceil(r / 512), H, B), block 128.
__global__ void __launch_bounds__(128)
k_merge(const WsHeader* __restrict__ hdr, const int32_t* __restrict__ sched,
        const float* __restrict__ pm, const float* __restrict__ pl, const float* __restrict__ pz,
        float* __restrict__ zm, int B, int H, int r, const uint8_t* __restrict__ pf,
        unsigned long long pf_bytes) {
  // the following GEMV's weights towards L2 (constant; a hint)
  if (pf_bytes && threadIdx.x == 32) dev::l2_prefetch_share(pf, pf_bytes);
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  __shared__ float wt[kMergeMaxSplits];
  __shared__ int cr[2];
  const int ch = blockIdx.x * kMergeCh + 4 * threadIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long G = hdr->G;
  if (warp == 0) {
    // the slots of sequence b: splits c0..c1 (slot c + b); dead splits weigh 0
    const long long T = sched[B], t0 = sched[b], t1 = sched[b + 1];
    int c0 = 0, c1 = -1;
    if (t1 > t0) {
      c0 = int(dev::split_of_tile(t0, G, T));
      c1 = int(dev::split_of_tile(t1 - 1, G, T));
    }
    float M = -INFINITY;
    for (int c = c0 + lane; c <= c1; c += 32)
      if (dev::split_begin(c, G, T) != dev::split_begin(c + 1, G, T))
        M = fmaxf(M, __ldcg(pm + (size_t(c) + b) * H + h));
    M = dev::warp_max(M);
    float L = 0.f;
    for (int c = c0 + lane; c <= c1; c += 32) {
      float w = 0.f;
      if (dev::split_begin(c, G, T) != dev::split_begin(c + 1, G, T)) {
        w = exp2f(__ldcg(pm + (size_t(c) + b) * H + h) - M);
        L += w * __ldcg(pl + (size_t(c) + b) * H + h);
      }
      wt[c - c0] = w;
    }
    L = dev::warp_sum(L);
    const float invL = L > 0.f ? 1.f / L : 0.f;
    __syncwarp();
    for (int c = c0 + lane; c <= c1; c += 32) wt[c - c0] *= invL;
    if (lane == 0) { cr[0] = c0; cr[1] = c1; }
  }
  __syncthreads();
  if (ch >= r) return;
  const int c0 = cr[0], c1 = cr[1];
  const float* base = pz + size_t(h) * r + ch;
  float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int cb = c0; cb <= c1; cb += 8) {   // eight splits' loads in flight, added in split order
    float4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      v[i] = cb + i <= c1 && wt[cb + i - c0] != 0.f
                 ? __ldcg(reinterpret_cast<const float4*>(base + (size_t(cb + i) + b) * H * r))
                 : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float w = cb + i <= c1 ? wt[cb + i - c0] : 0.f;
      z.x = fmaf(w, v[i].x, z.x); z.y = fmaf(w, v[i].y, z.y);
      z.z = fmaf(w, v[i].z, z.z); z.w = fmaf(w, v[i].w, z.w);
    }
  }
  *reinterpret_cast<float4*>(zm + (size_t(b) * H + h) * r + ch) = z;
}

constexpr int kJ = 128;   // latent rows (of W^u_v) per CTA
constexpr int kBC = 16;   // sequences per pass

// grid (H, ceil(r / kJ)), block 256.
// smem: ws[kJ][d_h] W^u_v tile (16-bit, as stored), zs[kBC][kJ] merged
//       latents, red[KSP][kBC][d_h] partial outputs, wt[P] per-slot merge
//       weight 2^(m_s - M) / L (indexed by slot), ts[B + 1] tile starts,
//       seg[B][2] slot ranges.
// Every stage issues all of a thread's loads before it uses one of them:
// the W^u_v tile by cp.async (it lands while the weights and the merge run),
// the partials of 8 splits per thread at a time; registers are capped for
// three CTAs per SM, so that the whole grid is resident at once.
template <typename WT>
__global__ void __launch_bounds__(256, 3)
k_combine_vup(const WsHeader* __restrict__ hdr, const int32_t* __restrict__ sched,
              const float* __restrict__ pm, const float* __restrict__ pl,
              const float* __restrict__ pz, const WT* __restrict__ wuv,
              float* __restrict__ opart, int B, int H, int d_h, int r, int E, int P) {
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  extern __shared__ __align__(16) uint8_t csm[];
  const int DQ = d_h / 4;                 // output quads per sequence
  const int KSP = 256 / (4 * DQ);         // k-splits of the V-up tile
  WT* ws = reinterpret_cast<WT*>(csm);                                   // kJ * d_h
  float* zs = reinterpret_cast<float*>(csm + size_t(kJ) * d_h * sizeof(WT));   // kBC * kJ
  float* red = zs + kBC * kJ;             // KSP * kBC * d_h
  float* wt = red + KSP * kBC * d_h;      // P
  int* ts = reinterpret_cast<int*>(wt + P);   // B + 1
  int* seg = ts + B + 1;                  // B x {c0, c1}
  const int h = blockIdx.x;
  const int js = blockIdx.y;
  const int j0 = js * kJ;
  const int jn = min(kJ, r - j0);         // a multiple of 32
  const long long G = hdr->G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // W^u_v tile rows j0 .. j0 + jn - 1, head h's columns: 16-byte async copies
  {
    const int vpr = d_h * int(sizeof(WT)) / 16;   // d_h is a multiple of 8
    const uint32_t ws_s = static_cast<uint32_t>(__cvta_generic_to_shared(ws));
    for (int i = threadIdx.x; i < kJ * vpr; i += 256) {
      const int jj = i / vpr, v = i % vpr;
      if (jj < jn) {
        const WT* src = wuv + size_t(j0 + jj) * E + h * d_h + v * (16 / int(sizeof(WT)));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ws_s + 16u * i), "l"(src) : "memory");
      } else {
        reinterpret_cast<uint4*>(ws)[i] = make_uint4(0, 0, 0, 0);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  for (int i = threadIdx.x; i <= B; i += 256) ts[i] = sched[i];
  __syncthreads();
  const long long T = ts[B];
  // merge weights, one warp per sequence; lane i holds slots c0 + i + 32 k
  for (int b = warp; b < B; b += 8) {
    const long long t0 = ts[b], t1 = ts[b + 1];
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
      const bool live = c <= c1 && dev::split_begin(c, G, T) != dev::split_begin(c + 1, G, T);
      mv[k] = live ? __ldcg(pm + (size_t(c) + b) * H + h) : -INFINITY;
      lv[k] = live ? __ldcg(pl + (size_t(c) + b) * H + h) : 0.f;
      M = fmaxf(M, mv[k]);
    }
    for (int c = c0 + lane + 32 * NR; c <= c1; c += 32)   // long runs of splits
      if (dev::split_begin(c, G, T) != dev::split_begin(c + 1, G, T))
        M = fmaxf(M, __ldcg(pm + (size_t(c) + b) * H + h));
    M = dev::warp_max(M);
    float L = 0.f;
#pragma unroll
    for (int k = 0; k < NR; ++k) L += exp2f(mv[k] - M) * lv[k];
    for (int c = c0 + lane + 32 * NR; c <= c1; c += 32)
      if (dev::split_begin(c, G, T) != dev::split_begin(c + 1, G, T))
        L += exp2f(__ldcg(pm + (size_t(c) + b) * H + h) - M) * __ldcg(pl + (size_t(c) + b) * H + h);
    L = dev::warp_sum(L);
    const float invL = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int k = 0; k < NR; ++k) {
      const int c = c0 + lane + 32 * k;
      if (c <= c1) wt[c + b] = exp2f(mv[k] - M) * invL;
    }
    for (int c = c0 + lane + 32 * NR; c <= c1; c += 32) {
      const bool live = dev::split_begin(c, G, T) != dev::split_begin(c + 1, G, T);
      wt[c + b] = live ? exp2f(__ldcg(pm + (size_t(c) + b) * H + h) - M) * invL : 0.f;
    }
  }
  __syncthreads();
  // V-up tile: thread -> 4 sequences x 4 output dims over one k-split
  const int ksp = threadIdx.x / (4 * DQ);
  const int bq = (threadIdx.x % (4 * DQ)) / DQ;
  const int dq = threadIdx.x % DQ;
  const int kper = kJ / KSP;
  // merge: thread -> channel quad qd of sequences mb and mb + 8
  const int mb = threadIdx.x >> 5, qd = threadIdx.x & 31;
  bool waited = false;
  for (int bc = 0; bc < B; bc += kBC) {
    const int bn = min(kBC, B - bc);
#pragma unroll 1
    for (int bb = mb; bb < kBC; bb += 8) {
      const int b = bc + bb;
      float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      if (bb < bn && 4 * qd < jn) {
        const int c0 = seg[2 * b], c1 = seg[2 * b + 1];
        const float* base = pz + size_t(h) * r + j0 + 4 * qd;
        for (int cb = c0; cb <= c1; cb += 8) {
          float4 v[8];
          float w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            w[i] = cb + i <= c1 ? wt[cb + i + b] : 0.f;
            v[i] = w[i] != 0.f
                       ? __ldcg(reinterpret_cast<const float4*>(base + (size_t(cb + i) + b) * H * r))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            z.x = fmaf(w[i], v[i].x, z.x); z.y = fmaf(w[i], v[i].y, z.y);
            z.z = fmaf(w[i], v[i].z, z.z); z.w = fmaf(w[i], v[i].w, z.w);
          }
        }
      }
      reinterpret_cast<float4*>(zs + bb * kJ)[qd] = z;
    }
    if (!waited) {   // the W^u_v tile has landed
      asm volatile("cp.async.wait_all;" ::: "memory");
      waited = true;
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
    const int kend = ksp < KSP ? (ksp + 1) * kper : 0;   // spare threads when 256 % d_h != 0
    for (int k = ksp * kper; k < kend; ++k) {
      float w4[4];
      {
        const WT* wp = ws + k * d_h + 4 * dq;
        w4[0] = dev::to_f(wp[0]); w4[1] = dev::to_f(wp[1]);
        w4[2] = dev::to_f(wp[2]); w4[3] = dev::to_f(wp[3]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float z = zs[(4 * bq + a) * kJ + k];
        acc[a][0] = fmaf(z, w4[0], acc[a][0]);
        acc[a][1] = fmaf(z, w4[1], acc[a][1]);
        acc[a][2] = fmaf(z, w4[2], acc[a][2]);
        acc[a][3] = fmaf(z, w4[3], acc[a][3]);
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
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  const size_t i = size_t(blockIdx.x) * 256 + threadIdx.x;
  if (i >= n) return;
  out[i] = dev::from_f<OT>(dev::sum_strided(opart + i, n, JS));
}

template <typename WT>
cudaError_t vup_t(const qsvd_dims& d, const WsHeader* hdr, const int32_t* sched,
                  const float* pm, const float* pl, const float* pz, const void* wuv,
                  float* opart, int JS, int P, cudaStream_t s) {
  const int ksp = 256 / d.d_h;   // k-splits of the V-up tile (4 x 4 outputs per thread)
  const size_t smem = size_t(kJ) * d.d_h * sizeof(WT) +
                      (size_t(kBC) * kJ + size_t(ksp) * kBC * d.d_h + P) * 4 + size_t(d.batch + 1) * 4 +
                      size_t(d.batch) * 8;
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  auto kern = k_combine_vup<WT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e == cudaSuccess)   // room for three CTAs per SM
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  dim3 grid(d.H, JS);
  {
    const cudaError_t le = launch_pdl(kern, dim3(grid), dim3(256), smem, s,
                                     hdr, sched, pm, pl, pz, static_cast<const WT*>(wuv), opart, d.batch, d.H, d.d_h, d.r, d.E, P);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return check_launch();
}

template <typename OT>
cudaError_t out_t(const qsvd_dims& d, const float* opart, int JS, void* out, cudaStream_t s) {
  const size_t n = size_t(d.batch) * d.E;
  {
    const cudaError_t le = launch_pdl(k_combine_out<OT>, dim3(unsigned((n + 255) / 256)), dim3(256), 0, s,
                                     opart, JS, static_cast<OT*>(out), n);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return check_launch();
}

template <typename WT, typename OT>
cudaError_t merge_vup_t(const qsvd_dims& d, const WsHeader* hdr, const int32_t* sched,
                        const float* pm, const float* pl, const float* pz, const void* wuv,
                        float* zm, float* vpart, int32_t* tickets, int32_t* status, void* out,
                        const OutProj& op, cudaStream_t s) {
  const dim3 grid((d.r + kMergeCh - 1) / kMergeCh, d.H, d.batch);
  {
    // the GEMV after the merge reads F (fold) or W^u_v
    const size_t wb = sizeof(WT);
    const void* pf = d.out_proj == QSVD_OUT_PROJ_FOLD ? op.wo : wuv;
    const size_t pf_bytes = d.out_proj == QSVD_OUT_PROJ_FOLD ? size_t(d.H) * d.r * d.E * wb : size_t(d.r) * d.E * wb;
    const cudaError_t le = launch_pdl(k_merge, dim3(grid), dim3(128), 0, s, hdr, sched, pm, pl, pz, zm,
                                     d.batch, d.H, d.r, static_cast<const uint8_t*>(pf),
                                     (unsigned long long)pf_bytes);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  cudaError_t e = check_launch();
  if (e != cudaSuccess) return e;
  const WT* wo = static_cast<const WT*>(op.wo);
  if (d.out_proj == QSVD_OUT_PROJ_FOLD) {
    // out[b][n] = sum_{h, j} zm[b][h][j] F[h r + j][n]: the merged latents of
    // all heads are one activation row of H r elements
    const int K = d.H * d.r;
    return launch_gemv<float, WT, OT>(zm, wo, op.ypart, d.batch, K, d.E, gemv_ksplit(K, d.weight_dtype),
                                      static_cast<OT*>(out), op.ytickets, status, s);
  }
  // o[b][h d_h + n] = zm[b][h] . W^u_v[:, h d_h + n]: activation row of
  // column group h (d_h columns) is zm + b H r + h r
  const XGroups xg{(long long)d.H * d.r, d.d_h, d.r};
  if (d.out_proj == QSVD_OUT_PROJ_CHAIN) {
    e = launch_gemv<float, WT, float>(zm, static_cast<const WT*>(wuv), vpart, d.batch, d.r, d.E,
                                      gemv_ksplit(d.r, d.weight_dtype), op.ow, tickets, status, s, xg);
    if (e != cudaSuccess) return e;
    // y = o W_O with o kept in fp32 (the GEMV splits it into two 16-bit parts)
    return launch_gemv<float, WT, OT>(op.ow, wo, op.ypart, d.batch, d.E, d.E,
                                      gemv_ksplit(d.E, d.weight_dtype), static_cast<OT*>(out), op.ytickets,
                                      status, s);
  }
  return launch_gemv<float, WT, OT>(zm, static_cast<const WT*>(wuv), vpart, d.batch, d.r, d.E,
                                    gemv_ksplit(d.r, d.weight_dtype), static_cast<OT*>(out), tickets,
                                    status, s, xg);
}

}  // namespace

bool combine_uses_gemv(const qsvd_dims& d) {
  // the merge's weights fit for any G (G <= kMaxSplits, capped by the host);
  // the tile bound is the range of sequence lengths this path supports
  const long long tiles = (d.max_len + kTile - 1) / kTile;
  return (d.weight_dtype == QSVD_F16 || d.weight_dtype == QSVD_BF16) && d.d_h % 64 == 0 &&
         d.r % 32 == 0 && tiles + 1 <= kMergeMaxSplits;
}

cudaError_t launch_combine_gemv(const qsvd_dims& d, const WsHeader* hdr, const int32_t* sched,
                                const float* pm, const float* pl, const float* pz, const void* wuv,
                                float* zm, float* vpart, int32_t* tickets, int32_t* status, void* out,
                                const OutProj& op, cudaStream_t s) {
#define QSVD_MV(WT)                                                                                    \
  switch (d.out_dtype) {                                                                               \
    case QSVD_F32: return merge_vup_t<WT, float>(d, hdr, sched, pm, pl, pz, wuv, zm, vpart, tickets,   \
                                                 status, out, op, s);                                      \
    case QSVD_F16: return merge_vup_t<WT, __half>(d, hdr, sched, pm, pl, pz, wuv, zm, vpart, tickets,  \
                                                  status, out, op, s);                                     \
    case QSVD_BF16: return merge_vup_t<WT, __nv_bfloat16>(d, hdr, sched, pm, pl, pz, wuv, zm, vpart,   \
                                                          tickets, status, out, op, s);                    \
    default: return cudaErrorInvalidValue;                                                             \
  }
  if (d.weight_dtype == QSVD_BF16) { QSVD_MV(__nv_bfloat16) }
  if (d.weight_dtype == QSVD_F16) { QSVD_MV(__half) }
#undef QSVD_MV
  return cudaErrorInvalidValue;
}

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
