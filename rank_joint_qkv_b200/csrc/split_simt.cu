// Split phase on CUDA cores: flash decoding over latent tiles, every dtype.
//
// Each CTA owns a contiguous run of 128-token tiles of the flattened
// (sequence, tile) order and, for every sequence segment in that run, writes
// one partial (m, l, z) per head: m the running max of the log2-domain
// scores, l = sum_t 2^(s_t - m), z = sum_t 2^(s_t - m) c_t (latent space).
//
// Absorbed mode (no rotary embedding): s_t,h = c_t . qt_h with qt_h the
// absorbed query (QSVD digest, Method, Step 1: K = C W^u_k is never built).
// Rotary mode: k_t,h = R(t) (c_t W^u_{k,h}) is rebuilt per sub-tile and
// s_t,h = k_t,h . q_h (WSVD digest, Method 3.4: keys rebuilt on-chip, rotary
// applied, scores and softmax in the same pass).
//
// These kernels are the reference-quality GPU path (every cache dtype, any
// rank multiple of 32); the tensor-core kernel replaces the absorbed one for
// 16-bit caches.
#include "internal.cuh"

namespace qsvd {
namespace {

using dev::CacheVec;

constexpr int kThreads = 256;

// Reduce-scatter over the 32 lanes of N values per lane (N power of two).
// Afterwards lane L holds the lane-sum of index L*(N/32)+p, p < N/32, when
// N >= 32; when N < 32 it holds index L >> log2(32/N) in v[0].
template <int N>
__device__ __forceinline__ void warp_reduce_scatter(float (&v)[N], int lane) {
  int n = N;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (n >= 2) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        if (i < n / 2) {
          const float send = upper ? v[i] : v[i + n / 2];
          const float keep = upper ? v[i + n / 2] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      n >>= 1;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
}

// Locate the first sequence of a tile run: largest b with tstart[b] <= t.
__device__ __forceinline__ int seq_of_tile(const int32_t* tstart, int B, long long t) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tstart[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Stage rows [t0, t0 + nv) of one sequence's cache as float (dequantised)
// into dst[TS][ld]; rows nv..TS-1 are zero.
template <qsvd_dtype CT>
__device__ __forceinline__ void stage_rows(float* dst, int ld, int TS, const uint8_t* seq_base,
                                           const __half* seq_scales, size_t row_bytes, int r,
                                           int group, int t0, int nv) {
  constexpr int N = CacheVec<CT>::N;
  const int vec_per_row = r / N;
  for (int i = threadIdx.x; i < TS * vec_per_row; i += kThreads) {
    const int t = i / vec_per_row, v = i % vec_per_row;
    const int j0 = v * N;
    float o[N];
    if (t < nv) {
      float s = 1.f;
      if (CT == QSVD_I8 || CT == QSVD_I4)
        s = __half2float(seq_scales[size_t(t0 + t) * (r / group) + j0 / group]);
      CacheVec<CT>::load(seq_base + size_t(t0 + t) * row_bytes, j0, s, o);
    } else {
#pragma unroll
      for (int k = 0; k < N; ++k) o[k] = 0.f;
    }
#pragma unroll
    for (int k = 0; k < N; ++k) dst[t * ld + j0 + k] = o[k];
  }
}

// ---------------------------------------------------------------------------
// Absorbed split kernel.  grid (G, H/HB), block 256.
// smem: qs[HB][r], cs[TS][r], zs[HB][r] (float), sc[TS*HB], red[8][64].
// ---------------------------------------------------------------------------
// SG: the scores come precomputed (rotary mode: [B][H][max_len], log2 domain,
// scaled) instead of from the absorbed query.
template <qsvd_dtype CT, int HB, bool SG = false>
__global__ void __launch_bounds__(kThreads)
k_split_abs(const float* __restrict__ qt32, const uint8_t* __restrict__ cache,
            const __half* __restrict__ scales, const int32_t* __restrict__ sched,
            float* __restrict__ pm, float* __restrict__ pl, float* __restrict__ pz,
            int B, int H, int r, int max_len, int group, int G, const float* __restrict__ sgiven = nullptr) {
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  constexpr int TS = 8;             // tokens per sub-tile
  constexpr int NV = TS * HB;       // scores per sub-tile
  extern __shared__ float sm[];
  float* qs = sm;                   // HB * r
  float* cs = qs + HB * r;          // TS * r
  float* zs = cs + TS * r;          // HB * r
  __shared__ float sc[NV];
  __shared__ float red[8][NV > 64 ? NV : 64];
  __shared__ float m_s[HB], l_s[HB], alpha_s[HB];

  const int c = blockIdx.x;
  const int h0 = blockIdx.y * HB;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int32_t* tstart = sched;          // B + 1
  const int32_t* lens = sched + B + 1;    // B
  const long long T = tstart[B];
  const long long tb = dev::split_begin(c, G, T), te = dev::split_begin(c + 1, G, T);
  if (tb >= te) return;

  const size_t row_bytes = (CT == QSVD_F32) ? size_t(r) * 4
                         : (CT == QSVD_I8) ? size_t(r)
                         : (CT == QSVD_I4) ? size_t(r) / 2 : size_t(r) * 2;
  const int ngroups = (CT == QSVD_I8 || CT == QSVD_I4) ? r / group : 1;

  int b = seq_of_tile(tstart, B, tb);
  long long t = tb;
  while (t < te) {
    while (tstart[b + 1] <= t) ++b;       // skip empty sequences
    const long long seg_end = min(te, (long long)tstart[b + 1]);
    const int n = lens[b];
    const int tok0 = int(t - tstart[b]) * kTile;
    const int tok1 = min(n, int(seg_end - tstart[b]) * kTile);
    const uint8_t* seq_base = cache + size_t(b) * max_len * row_bytes;
    const __half* seq_scales = scales ? scales + size_t(b) * max_len * ngroups : nullptr;

    // absorbed queries of this head block; zero the latent accumulators
    __syncthreads();
    for (int i = threadIdx.x; i < HB * r; i += kThreads) {
      const int hh = i / r, j = i % r;
      if (!SG) qs[i] = qt32[(size_t(b) * H + h0 + hh) * r + j];
      zs[i] = 0.f;
    }
    if (threadIdx.x < HB) { m_s[threadIdx.x] = -INFINITY; l_s[threadIdx.x] = 0.f; }

    for (int s0 = tok0; s0 < tok1; s0 += TS) {
      const int nv = min(TS, tok1 - s0);
      __syncthreads();
      stage_rows<CT>(cs, r, TS, seq_base, seq_scales, row_bytes, r, group, s0, nv);
      __syncthreads();
      if (SG) {   // scores given: sc[tt][hh]
        if (threadIdx.x < NV) {
          const int tt = threadIdx.x / HB, hh = threadIdx.x % HB;
          sc[threadIdx.x] = tt < nv ? sgiven[(size_t(b) * H + h0 + hh) * max_len + s0 + tt] : 0.f;
        }
      } else {
      // scores: each thread a strided slice of the channels
      float acc[NV];
#pragma unroll
      for (int i = 0; i < NV; ++i) acc[i] = 0.f;
      for (int j = threadIdx.x; j < r; j += kThreads) {
        float q[HB];
#pragma unroll
        for (int hh = 0; hh < HB; ++hh) q[hh] = qs[hh * r + j];
#pragma unroll
        for (int tt = 0; tt < TS; ++tt) {
          const float cv = cs[tt * r + j];
#pragma unroll
          for (int hh = 0; hh < HB; ++hh) acc[tt * HB + hh] = fmaf(cv, q[hh], acc[tt * HB + hh]);
        }
      }
      warp_reduce_scatter<NV>(acc, lane);
      if (NV >= 32) {
#pragma unroll
        for (int p = 0; p < (NV >= 32 ? NV / 32 : 1); ++p) red[warp][lane * (NV / 32) + p] = acc[p];
      } else {
        constexpr int sh = (NV == 16) ? 1 : (NV == 8) ? 2 : 0;
        if ((lane & ((1 << sh) - 1)) == 0) red[warp][lane >> sh] = acc[0];
      }
      __syncthreads();
      if (threadIdx.x < NV) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) s += red[w][threadIdx.x];
        sc[threadIdx.x] = s;
      }
      }
      __syncthreads();
      // online softmax per head (log2 domain)
      if (threadIdx.x < HB) {
        const int hh = threadIdx.x;
        float mx = -INFINITY;
        for (int tt = 0; tt < nv; ++tt) mx = fmaxf(mx, sc[tt * HB + hh]);
        const float m_old = m_s[hh];
        const float m_new = fmaxf(m_old, mx);
        const float alpha = exp2f(m_old - m_new);
        float l = l_s[hh] * alpha;
        for (int tt = 0; tt < TS; ++tt) {
          const float p = tt < nv ? exp2f(sc[tt * HB + hh] - m_new) : 0.f;
          sc[tt * HB + hh] = p;
          l += p;
        }
        m_s[hh] = m_new; l_s[hh] = l; alpha_s[hh] = alpha;
      }
      __syncthreads();
      // latent accumulation z_h = alpha z_h + sum_t p_t,h c_t
      for (int j = threadIdx.x; j < r; j += kThreads) {
        float cv[TS];
#pragma unroll
        for (int tt = 0; tt < TS; ++tt) cv[tt] = cs[tt * r + j];
#pragma unroll
        for (int hh = 0; hh < HB; ++hh) {
          float z = zs[hh * r + j] * alpha_s[hh];
#pragma unroll
          for (int tt = 0; tt < TS; ++tt) z = fmaf(sc[tt * HB + hh], cv[tt], z);
          zs[hh * r + j] = z;
        }
      }
    }
    __syncthreads();
    const size_t slot = size_t(c) + b;
    for (int i = threadIdx.x; i < HB * r; i += kThreads) {
      const int hh = i / r, j = i % r;
      pz[(slot * H + h0 + hh) * r + j] = zs[i];
    }
    if (threadIdx.x < HB) {
      pm[slot * H + h0 + threadIdx.x] = m_s[threadIdx.x];
      pl[slot * H + h0 + threadIdx.x] = l_s[threadIdx.x];
    }
    t = seg_end;
    ++b;
  }
}

// ---------------------------------------------------------------------------
// Rotary split kernel.  grid (G, H), block 256 = 8 warps.
// Sub-tile of 16 tokens: warp w owns tokens 2w, 2w+1; lane g owns the
// rotary pairs (i, i + d_h/2) with i in [g*NP, g*NP + NP), NP = d_h/64.
// smem: cs[16][r+1], wk[32][d_h], zs[r].
// ---------------------------------------------------------------------------
template <qsvd_dtype CT, typename WT>
__global__ void __launch_bounds__(kThreads)
k_split_rope(const float* __restrict__ qrot, const WT* __restrict__ wuk,
             const float* __restrict__ tab, const uint8_t* __restrict__ cache,
             const __half* __restrict__ scales, const int32_t* __restrict__ sched,
             float* __restrict__ pm, float* __restrict__ pl, float* __restrict__ pz,
             int B, int H, int d_h, int r, int E, int max_len, int group, int G) {
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  constexpr int TS = 16;
  constexpr int JC = 32;
  extern __shared__ float sm[];
  const int ldc = r + 1;
  float* cs = sm;                   // TS * ldc
  float* wk = cs + TS * ldc;        // JC * d_h
  float* zs = wk + JC * d_h;        // r
  __shared__ float sc[TS];
  __shared__ float m_s, l_s, alpha_s;

  const int c = blockIdx.x;
  const int h = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = d_h / 2;
  const int NP = half / 32;         // pairs per lane (1 or 2 for d_h 64/128)
  const int32_t* tstart = sched;
  const int32_t* lens = sched + B + 1;
  const long long T = tstart[B];
  const long long tb = dev::split_begin(c, G, T), te = dev::split_begin(c + 1, G, T);
  if (tb >= te) return;

  const size_t row_bytes = (CT == QSVD_F32) ? size_t(r) * 4
                         : (CT == QSVD_I8) ? size_t(r)
                         : (CT == QSVD_I4) ? size_t(r) / 2 : size_t(r) * 2;
  const int ngroups = (CT == QSVD_I8 || CT == QSVD_I4) ? r / group : 1;

  int b = seq_of_tile(tstart, B, tb);
  long long t = tb;
  while (t < te) {
    while (tstart[b + 1] <= t) ++b;
    const long long seg_end = min(te, (long long)tstart[b + 1]);
    const int n = lens[b];
    const int tok0 = int(t - tstart[b]) * kTile;
    const int tok1 = min(n, int(seg_end - tstart[b]) * kTile);
    const uint8_t* seq_base = cache + size_t(b) * max_len * row_bytes;
    const __half* seq_scales = scales ? scales + size_t(b) * max_len * ngroups : nullptr;
    // this lane's query components (already rotated and scaled)
    float qlo[2], qhi[2];
    for (int k = 0; k < 2; ++k) {
      const int i = lane * NP + k;
      qlo[k] = (k < NP) ? qrot[size_t(b) * E + h * d_h + i] : 0.f;
      qhi[k] = (k < NP) ? qrot[size_t(b) * E + h * d_h + i + half] : 0.f;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < r; j += kThreads) zs[j] = 0.f;
    if (threadIdx.x == 0) { m_s = -INFINITY; l_s = 0.f; }

    for (int s0 = tok0; s0 < tok1; s0 += TS) {
      const int nv = min(TS, tok1 - s0);
      __syncthreads();
      stage_rows<CT>(cs, ldc, TS, seq_base, seq_scales, row_bytes, r, group, s0, nv);
      // keys of tokens 2w, 2w+1 at this lane's dims
      float acc[2][2][2];  // [token][pair slot][lo/hi]
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int k = 0; k < 2; ++k) { acc[a][k][0] = 0.f; acc[a][k][1] = 0.f; }
      for (int j0 = 0; j0 < r; j0 += JC) {
        __syncthreads();
        for (int i = threadIdx.x; i < JC * d_h; i += kThreads) {
          const int jj = i / d_h, dd = i % d_h;
          wk[i] = dev::to_f(wuk[size_t(j0 + jj) * E + h * d_h + dd]);
        }
        __syncthreads();
#pragma unroll 4
        for (int jj = 0; jj < JC; ++jj) {
          const float c0 = cs[(2 * warp) * ldc + j0 + jj];
          const float c1 = cs[(2 * warp + 1) * ldc + j0 + jj];
          for (int k = 0; k < NP; ++k) {
            const int i = lane * NP + k;
            const float wlo = wk[jj * d_h + i], whi = wk[jj * d_h + i + half];
            acc[0][k][0] = fmaf(c0, wlo, acc[0][k][0]);
            acc[0][k][1] = fmaf(c0, whi, acc[0][k][1]);
            acc[1][k][0] = fmaf(c1, wlo, acc[1][k][0]);
            acc[1][k][1] = fmaf(c1, whi, acc[1][k][1]);
          }
        }
      }
      // rotate keys at their positions and score
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const int tt = 2 * warp + a;
        const int pos = s0 + tt;
        float part = 0.f;
        if (tt < nv) {
          for (int k = 0; k < NP; ++k) {
            const int i = lane * NP + k;
            const float cs_ = tab[(size_t(pos) * half + i) * 2 + 0];
            const float sn_ = tab[(size_t(pos) * half + i) * 2 + 1];
            const float lo = acc[a][k][0], hi = acc[a][k][1];
            const float rlo = lo * cs_ - hi * sn_;
            const float rhi = hi * cs_ + lo * sn_;
            part = fmaf(rlo, qlo[k], part);
            part = fmaf(rhi, qhi[k], part);
          }
        }
        part = dev::warp_sum(part);
        if (lane == 0) sc[tt] = part;
      }
      __syncthreads();
      if (warp == 0) {
        const float s = lane < nv ? sc[lane & (TS - 1)] : -INFINITY;
        const float mx = dev::warp_max(lane < TS ? s : -INFINITY);
        const float m_old = m_s;
        const float m_new = fmaxf(m_old, mx);
        const float p = (lane < nv) ? exp2f(s - m_new) : 0.f;
        const float psum = dev::warp_sum(p);
        __syncwarp();
        if (lane < TS) sc[lane] = p;
        if (lane == 0) {
          const float alpha = exp2f(m_old - m_new);
          l_s = l_s * alpha + psum;
          m_s = m_new;
          alpha_s = alpha;
        }
      }
      __syncthreads();
      const float alpha = alpha_s;
      for (int j = threadIdx.x; j < r; j += kThreads) {
        float z = zs[j] * alpha;
#pragma unroll
        for (int tt = 0; tt < TS; ++tt) z = fmaf(sc[tt], cs[tt * ldc + j], z);
        zs[j] = z;
      }
    }
    __syncthreads();
    const size_t slot = size_t(c) + b;
    for (int j = threadIdx.x; j < r; j += kThreads) pz[(slot * H + h) * r + j] = zs[j];
    if (threadIdx.x == 0) { pm[slot * H + h] = m_s; pl[slot * H + h] = l_s; }
    t = seg_end;
    ++b;
  }
}

int head_block(const qsvd_dims& d) {
  for (int hb : {8, 4, 2, 1}) {
    if (d.H % hb) continue;
    const size_t smem = size_t(2 * hb + 8) * d.r * 4;
    if (smem <= 200 * 1024) return hb;
  }
  return 0;
}

template <qsvd_dtype CT, int HB, bool SG = false>
cudaError_t abs_t(const qsvd_dims& d, const float* qt32, const void* cache, const void* scales,
                  const int32_t* sched, int G, float* pm, float* pl, float* pz, cudaStream_t s,
                  const float* sgiven = nullptr) {
  const size_t smem = size_t(2 * HB + 8) * d.r * 4;
  auto kern = k_split_abs<CT, HB, SG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(G, d.H / HB);
  {
    const cudaError_t le = launch_pdl(kern, dim3(grid), dim3(kThreads), smem, s,
                                     qt32, static_cast<const uint8_t*>(cache), static_cast<const __half*>(scales), sched, pm, pl, pz, d.batch, d.H, d.r, d.max_len, d.group, G, sgiven);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return check_launch();
}

template <qsvd_dtype CT>
cudaError_t scores_ct(const qsvd_dims& d, const float* sgiven, const void* cache, const void* scales,
                      const int32_t* sched, int G, float* pm, float* pl, float* pz, cudaStream_t s) {
  switch (head_block(d)) {
    case 8: return abs_t<CT, 8, true>(d, nullptr, cache, scales, sched, G, pm, pl, pz, s, sgiven);
    case 4: return abs_t<CT, 4, true>(d, nullptr, cache, scales, sched, G, pm, pl, pz, s, sgiven);
    case 2: return abs_t<CT, 2, true>(d, nullptr, cache, scales, sched, G, pm, pl, pz, s, sgiven);
    case 1: return abs_t<CT, 1, true>(d, nullptr, cache, scales, sched, G, pm, pl, pz, s, sgiven);
    default: return cudaErrorInvalidConfiguration;
  }
}

template <qsvd_dtype CT>
cudaError_t abs_ct(const qsvd_dims& d, const float* qt32, const void* cache, const void* scales,
                   const int32_t* sched, int G, float* pm, float* pl, float* pz, cudaStream_t s) {
  switch (head_block(d)) {
    case 8: return abs_t<CT, 8>(d, qt32, cache, scales, sched, G, pm, pl, pz, s);
    case 4: return abs_t<CT, 4>(d, qt32, cache, scales, sched, G, pm, pl, pz, s);
    case 2: return abs_t<CT, 2>(d, qt32, cache, scales, sched, G, pm, pl, pz, s);
    case 1: return abs_t<CT, 1>(d, qt32, cache, scales, sched, G, pm, pl, pz, s);
    default: return cudaErrorInvalidConfiguration;
  }
}

template <qsvd_dtype CT, typename WT>
cudaError_t rope_t(const qsvd_dims& d, const float* qrot, const void* wuk, const float* tab,
                   const void* cache, const void* scales, const int32_t* sched, int G,
                   float* pm, float* pl, float* pz, cudaStream_t s) {
  const size_t smem = (size_t(16) * (d.r + 1) + size_t(32) * d.d_h + d.r) * 4;
  auto kern = k_split_rope<CT, WT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(G, d.H);
  {
    const cudaError_t le = launch_pdl(kern, dim3(grid), dim3(kThreads), smem, s,
                                     qrot, static_cast<const WT*>(wuk), tab, static_cast<const uint8_t*>(cache), static_cast<const __half*>(scales), sched, pm, pl, pz, d.batch, d.H, d.d_h, d.r, d.E, d.max_len, d.group, G);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return check_launch();
}

template <qsvd_dtype CT>
cudaError_t rope_ct(const qsvd_dims& d, const float* qrot, const void* wuk, const float* tab,
                    const void* cache, const void* scales, const int32_t* sched, int G,
                    float* pm, float* pl, float* pz, cudaStream_t s) {
  switch (d.weight_dtype) {
    case QSVD_F32: return rope_t<CT, float>(d, qrot, wuk, tab, cache, scales, sched, G, pm, pl, pz, s);
    case QSVD_F16: return rope_t<CT, __half>(d, qrot, wuk, tab, cache, scales, sched, G, pm, pl, pz, s);
    case QSVD_BF16: return rope_t<CT, __nv_bfloat16>(d, qrot, wuk, tab, cache, scales, sched, G, pm, pl, pz, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int split_simt_grid_heads(const qsvd_dims& d) {
  if (d.rope) return d.H;
  const int hb = head_block(d);
  return hb ? d.H / hb : 0;
}

cudaError_t launch_split_simt_absorbed(const qsvd_dims& d, const float* qt32, const void* cache,
                                       const void* scales, const int32_t* sched, int G,
                                       float* pm, float* pl, float* pz, cudaStream_t s) {
  switch (d.cache_dtype) {
    case QSVD_F32: return abs_ct<QSVD_F32>(d, qt32, cache, scales, sched, G, pm, pl, pz, s);
    case QSVD_F16: return abs_ct<QSVD_F16>(d, qt32, cache, scales, sched, G, pm, pl, pz, s);
    case QSVD_BF16: return abs_ct<QSVD_BF16>(d, qt32, cache, scales, sched, G, pm, pl, pz, s);
    case QSVD_I8: return abs_ct<QSVD_I8>(d, qt32, cache, scales, sched, G, pm, pl, pz, s);
    case QSVD_I4: return abs_ct<QSVD_I4>(d, qt32, cache, scales, sched, G, pm, pl, pz, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_split_simt_scores(const qsvd_dims& d, const float* scores, const void* cache,
                                     const void* scales, const int32_t* sched, int G, float* pm,
                                     float* pl, float* pz, cudaStream_t s) {
  switch (d.cache_dtype) {
    case QSVD_F16: return scores_ct<QSVD_F16>(d, scores, cache, scales, sched, G, pm, pl, pz, s);
    case QSVD_BF16: return scores_ct<QSVD_BF16>(d, scores, cache, scales, sched, G, pm, pl, pz, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_split_simt_rope(const qsvd_dims& d, const float* qrot, const void* wuk,
                                   const float* rope_tab, const void* cache, const void* scales,
                                   const int32_t* sched, int G, float* pm, float* pl, float* pz,
                                   cudaStream_t s) {
  switch (d.cache_dtype) {
    case QSVD_F32: return rope_ct<QSVD_F32>(d, qrot, wuk, rope_tab, cache, scales, sched, G, pm, pl, pz, s);
    case QSVD_F16: return rope_ct<QSVD_F16>(d, qrot, wuk, rope_tab, cache, scales, sched, G, pm, pl, pz, s);
    case QSVD_BF16: return rope_ct<QSVD_BF16>(d, qrot, wuk, rope_tab, cache, scales, sched, G, pm, pl, pz, s);
    case QSVD_I8: return rope_ct<QSVD_I8>(d, qrot, wuk, rope_tab, cache, scales, sched, G, pm, pl, pz, s);
    case QSVD_I4: return rope_ct<QSVD_I4>(d, qrot, wuk, rope_tab, cache, scales, sched, G, pm, pl, pz, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace qsvd
