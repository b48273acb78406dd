// Decode-step attention over per-head latents (WSVD paper digest, Method,
// per-head SVD §3.1 and fused kernel §3.4): head h keeps its own key latent
// C_{Kh} (L x r) and value latent C_{Vh} (L x r).  Without rotary embedding
// no key or value is rebuilt: the query is absorbed, qt_h = tau log2e
// B_{Kh} q_h, scores are C_{Kh,t} . qt_h, the value side accumulates
// z_h = p^T C_{Vh} in latent space and is up-projected once, o_h = z_h B_{Vh}.
//
// With a per-head latent one token of one head carries 2 r latent elements
// and 4 r flop (score dot and value accumulate): about one flop per byte of
// a 16-bit latent, an order of magnitude under the CUDA cores' rate per
// byte of HBM, so the kernels run on CUDA cores (a tensor-core tile would
// have one query row).  One CTA per (sequence, head, 256-token chunk):
// a warp per token row for the score dot (coalesced row reads), an exact
// softmax over the chunk, then the value rows read by consecutive threads
// for consecutive channels; a second kernel merges the chunks in the log2
// domain and applies B_{Vh}.
#include "gemv.cuh"
#include "wsvd.cuh"

namespace qsvd {
namespace {

constexpr int kT = 128;   // threads per CTA

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
// Block-wide reductions over kT threads; red holds 4 floats.  Every thread
// gets the result; red is free again after the call returns.
__device__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  const float s = (red[0] + red[1]) + (red[2] + red[3]);
  __syncthreads();
  return s;
}
__device__ float block_max(float v, float* red) {
  v = warp_max(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  const float m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  return m;
}

__device__ __forceinline__ int clamp_len(int len, int max_len) {
  return len < 0 ? 0 : (len > max_len ? max_len : len);
}

// qt[b][h][j] = sl2 sum_i B_K[h][j][i] q[b][h d_h + i].  grid (H, B).
template <typename WT>
__global__ void __launch_bounds__(kT)
k_wsvd_absorb(const WT* __restrict__ bk, const float* __restrict__ q, float* __restrict__ qt,
              int32_t* __restrict__ status, int H, int d_h, int r, float sl2,
              int32_t* __restrict__ tickets, int n_tickets) {
  extern __shared__ float qs[];   // d_h
  const int h = blockIdx.x, b = blockIdx.y;
  if (h == 0 && b == 0) {
    if (threadIdx.x == 0) *status = 0;   // the combine ORs flags in later
    for (int i = threadIdx.x; i < n_tickets; i += kT) tickets[i] = 0;   // the fold GEMV's counters
  }
  const float* qrow = q + (size_t(b) * H + h) * d_h;
  for (int i = threadIdx.x; i < d_h; i += kT) qs[i] = qrow[i];
  __syncthreads();
  for (int j = threadIdx.x; j < r; j += kT) {
    const WT* row = bk + (size_t(h) * r + j) * d_h;
    float acc = 0.f;
    for (int i = 0; i < d_h; ++i) acc = fmaf(dev::to_f(row[i]), qs[i], acc);
    qt[(size_t(b) * H + h) * r + j] = acc * sl2;
  }
}

// One chunk of one (sequence, head).  grid (S, H, B).  Writes the chunk's
// m = max s, l = sum 2^(s - m), z = sum 2^(s - m) C_V,t (log2-domain s).
// Latent row (b, h, t) starts at ((b H + h) max_len + t) r (head-major) or
// ((b max_len + t) H + h) r (token-major); consecutive tokens are r or H r
// elements apart.
template <typename CT>
__global__ void __launch_bounds__(kT)
k_wsvd_split(const CT* __restrict__ ck, const CT* __restrict__ cv, const float* __restrict__ qt,
             const int32_t* __restrict__ lengths, float* __restrict__ pm, float* __restrict__ pl,
             float* __restrict__ pz, int H, int r, int max_len, int S, int token_major) {
  extern __shared__ float sm[];
  float* qs = sm;                   // r
  float* ss = qs + r;               // kWsvdChunk scores, then weights
  float* red = ss + kWsvdChunk;     // 4
  float* zp = red + 4;              // ng x r partial sums (ng r <= max(r, kT))
  const int sp = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int len = clamp_len(lengths[b], max_len);
  const int t0 = sp * kWsvdChunk;
  if (t0 >= len) return;            // the same for every thread of the CTA
  const int n = min(kWsvdChunk, len - t0);
  const size_t bh = size_t(b) * H + h;
  const size_t row0 = token_major ? (size_t(b) * max_len + t0) * H + h : bh * max_len + t0;
  const size_t rs = token_major ? size_t(H) * r : size_t(r);   // elements between tokens
  const CT* kb = ck + row0 * size_t(r);
  const CT* vb = cv + row0 * size_t(r);
  for (int j = threadIdx.x; j < r; j += kT) qs[j] = qt[bh * r + j];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t = warp; t < n; t += kT / 32) {
    const CT* row = kb + size_t(t) * rs;
    float acc = 0.f;
    for (int j = lane; j < r; j += 32) acc = fmaf(dev::to_f(row[j]), qs[j], acc);
    acc = warp_sum(acc);
    if (lane == 0) ss[t] = acc;
  }
  __syncthreads();
  float mx = -INFINITY;
  for (int t = threadIdx.x; t < n; t += kT) mx = fmaxf(mx, ss[t]);
  const float M = block_max(mx, red);
  float ls = 0.f;
  for (int t = threadIdx.x; t < n; t += kT) {
    const float p = exp2f(ss[t] - M);
    ss[t] = p;
    ls += p;
  }
  const float L = block_sum(ls, red);   // its barriers also publish ss
  const size_t slot = bh * S + sp;
  float* zrow = pz + slot * size_t(r);
  const int ng = (r < kT && kT % r == 0) ? kT / r : 1;   // token groups when r divides kT
  if (ng > 1) {
    const int g = threadIdx.x / r, j = threadIdx.x % r;
    float acc = 0.f;
    for (int t = g; t < n; t += ng) acc = fmaf(ss[t], dev::to_f(vb[size_t(t) * rs + j]), acc);
    zp[g * r + j] = acc;
    __syncthreads();
    for (int jj = threadIdx.x; jj < r; jj += kT) {
      float z = 0.f;
      for (int gg = 0; gg < ng; ++gg) z += zp[gg * r + jj];
      zrow[jj] = z;
    }
  } else {
    for (int j = threadIdx.x; j < r; j += kT) {
      float acc = 0.f;
      for (int t = 0; t < n; ++t) acc = fmaf(ss[t], dev::to_f(vb[size_t(t) * rs + j]), acc);
      zrow[j] = acc;
    }
  }
  if (threadIdx.x == 0) {
    pm[slot] = M;
    pl[slot] = L;
  }
}

// The same chunk for 16-bit latents with r in {64, 128, 256}, read with
// 16-byte vectors: a token row is r / 8 vectors, taken by r / 8 consecutive
// threads (thread vj holds channels 8 vj .. 8 vj + 7 of the absorbed query in
// registers), 256 / (r / 8) rows per pass; every row load of the chunk is
// issued before the first is used.  Scores: per-thread partial dots summed
// over the row's threads by shuffles.  Values: per-thread sums over the
// thread's rows, then over the row groups in shared memory.  grid (S, H, B),
// block 256.
constexpr int kTV = 256;
__device__ __forceinline__ void widen8(const uint4& v, float (&f)[8], __half) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 x = __half22float2(h[e]);
    f[2 * e] = x.x;
    f[2 * e + 1] = x.y;
  }
}
__device__ __forceinline__ void widen8(const uint4& v, float (&f)[8], __nv_bfloat16) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {   // a bf16 is the high half of its float
    f[2 * e] = __uint_as_float(w[e] << 16);
    f[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
  }
}
template <typename CT, int R>
__global__ void __launch_bounds__(kTV)
k_wsvd_split_vec(const CT* __restrict__ ck, const CT* __restrict__ cv, const float* __restrict__ qt,
                 const int32_t* __restrict__ lengths, float* __restrict__ pm, float* __restrict__ pl,
                 float* __restrict__ pz, int H, int max_len, int S, int token_major,
                 const float* __restrict__ scores) {
  constexpr int TPR = R / 8;            // threads per row
  constexpr int TPP = kTV / TPR;        // rows per pass
  constexpr int NP = kWsvdChunk / TPP;  // passes per chunk
  __shared__ float ss[kWsvdChunk];      // scores, then weights
  __shared__ float zr[TPP][R];          // per row-group value sums
  __shared__ float red[8];
  const int sp = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int len = clamp_len(lengths[b], max_len);
  const int t0 = sp * kWsvdChunk;
  if (t0 >= len) return;                // the same for every thread of the CTA
  const int n = min(kWsvdChunk, len - t0);
  const size_t bh = size_t(b) * H + h;
  const size_t row0 = token_major ? (size_t(b) * max_len + t0) * H + h : bh * max_len + t0;
  const size_t rs = token_major ? size_t(H) * R : size_t(R);   // elements between tokens
  const int vj = threadIdx.x % TPR, tg = threadIdx.x / TPR;
  const uint4* kb = reinterpret_cast<const uint4*>(ck + row0 * R) + vj;
  const uint4* vb = reinterpret_cast<const uint4*>(cv + row0 * R) + vj;
  const size_t rsv = rs / 8;            // 16-byte vectors between tokens
  uint4 raw[NP];
  if (scores) {
    // rotary mode: the scores were computed from keys rebuilt on the tensor
    // cores ([B][H][max_len], log2 domain); only the values are read here
    for (int t = threadIdx.x; t < kWsvdChunk; t += kTV)
      ss[t] = t < n ? scores[bh * max_len + t0 + t] : -INFINITY;
  } else {
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int t = p * TPP + tg;
    raw[p] = t < n ? __ldg(kb + size_t(t) * rsv) : make_uint4(0, 0, 0, 0);
  }
  float q8[8];
  {
    const float4* qv = reinterpret_cast<const float4*>(qt + bh * R + 8 * vj);
    const float4 a = qv[0], c = qv[1];
    q8[0] = a.x; q8[1] = a.y; q8[2] = a.z; q8[3] = a.w;
    q8[4] = c.x; q8[5] = c.y; q8[6] = c.z; q8[7] = c.w;
  }
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    float f[8];
    widen8(raw[p], f, CT());
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc = fmaf(f[e], q8[e], acc);
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    const int t = p * TPP + tg;
    if (vj == 0) ss[t] = t < n ? acc : -INFINITY;
  }
  }
  // the value rows, in flight while the softmax runs
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int t = p * TPP + tg;
    raw[p] = t < n ? __ldg(vb + size_t(t) * rsv) : make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float mx = ss[threadIdx.x];   // kTV == kWsvdChunk: one score per thread
  mx = warp_max(mx);
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  float M = red[0];
#pragma unroll
  for (int w = 1; w < kTV / 32; ++w) M = fmaxf(M, red[w]);
  const float pt = threadIdx.x < n ? exp2f(ss[threadIdx.x] - M) : 0.f;
  __syncthreads();   // red and ss are rewritten below
  ss[threadIdx.x] = pt;
  float ls = warp_sum(pt);
  if (lane == 0) red[warp] = ls;
  __syncthreads();
  float L = 0.f;
#pragma unroll
  for (int w = 0; w < kTV / 32; ++w) L += red[w];
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const float w = ss[p * TPP + tg];
    float f[8];
    widen8(raw[p], f, CT());
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, f[e], acc[e]);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) zr[tg][8 * vj + e] = acc[e];
  __syncthreads();
  const size_t slot = bh * S + sp;
  for (int j = threadIdx.x; j < R; j += kTV) {
    float z = 0.f;
#pragma unroll 8
    for (int g = 0; g < TPP; ++g) z += zr[g][j];
    pz[slot * size_t(R) + j] = z;
  }
  if (threadIdx.x == 0) {
    pm[slot] = M;
    pl[slot] = L;
  }
}

// Merge the chunks of (b, h) and apply B_V: o[b][h d_h + i] =
// sum_j z[j] B_V[h][j][i], z = sum_s 2^(m_s - M) z_s / sum_s 2^(m_s - M) l_s.
// FOLD: write z to zm[b][h][r] instead (the GEMV by F = [B_{Vh} W_{O,h}]_h
// follows).  grid (H, B).
template <typename WT, typename OT, bool FOLD = false>
__global__ void __launch_bounds__(kT)
k_wsvd_combine(const float* __restrict__ pm, const float* __restrict__ pl, const float* __restrict__ pz,
               const WT* __restrict__ bv, const int32_t* __restrict__ lengths, OT* __restrict__ out,
               int32_t* __restrict__ status, int H, int d_h, int r, int max_len, int S,
               float* __restrict__ zm = nullptr) {
  extern __shared__ float sm[];
  float* ws = sm;          // S chunk weights
  float* zs = ws + S;      // r merged latent
  float* red = zs + r;     // 4
  const int h = blockIdx.x, b = blockIdx.y;
  const int raw = lengths[b];
  const int len = clamp_len(raw, max_len);
  if (h == 0 && threadIdx.x == 0 && raw != len) atomicOr(status, QSVD_STATUS_LEN_CLAMPED);
  OT* orow = out + (size_t(b) * H + h) * d_h;
  float* zrow = FOLD ? zm + (size_t(b) * H + h) * r : nullptr;
  const int su = (len + kWsvdChunk - 1) / kWsvdChunk;
  if (su == 0) {
    if (FOLD) {
      for (int j = threadIdx.x; j < r; j += kT) zrow[j] = 0.f;
    } else {
      for (int i = threadIdx.x; i < d_h; i += kT) orow[i] = dev::from_f<OT>(0.f);
    }
    return;
  }
  const size_t base = (size_t(b) * H + h) * S;
  float mx = -INFINITY;
  for (int s = threadIdx.x; s < su; s += kT) mx = fmaxf(mx, pm[base + s]);
  const float M = block_max(mx, red);
  float ls = 0.f;
  for (int s = threadIdx.x; s < su; s += kT) {
    const float w = exp2f(pm[base + s] - M);
    ws[s] = w;
    ls += w * pl[base + s];
  }
  const float L = block_sum(ls, red);   // its barriers also publish ws
  const float inv = 1.f / L;
  for (int j = threadIdx.x; j < r; j += kT) {
    float acc = 0.f;
    for (int s = 0; s < su; ++s) acc = fmaf(ws[s], pz[(base + s) * size_t(r) + j], acc);
    zs[j] = acc * inv;
    if (FOLD) zrow[j] = acc * inv;
  }
  if (FOLD) return;
  __syncthreads();
  const WT* bvh = bv + size_t(h) * r * d_h;
  for (int i = threadIdx.x; i < d_h; i += kT) {
    float acc = 0.f;
    for (int j = 0; j < r; ++j) acc = fmaf(zs[j], dev::to_f(bvh[size_t(j) * d_h + i]), acc);
    orow[i] = dev::from_f<OT>(acc);
  }
}

template <typename K>
cudaError_t allow_smem(K kern, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
}

// Merge + B_V (one kernel), or with B_{Vh} folded into W_O: merge into zm,
// then the tensor-core GEMV y = zm F (K = H r, N = E; F passed as bv).
template <typename WT, typename OT>
cudaError_t wsvd_combine(const qsvd_dims& d, const float* pm, const float* pl, const float* pz, const void* bv,
                         const int32_t* lengths, void* out, int32_t* status, const WsvdLayout& W, uint8_t* wb,
                         size_t s_comb, cudaStream_t s) {
  cudaError_t e;
  if (d.out_proj != QSVD_OUT_PROJ_FOLD) {
    auto kc = k_wsvd_combine<WT, OT, false>;
    if ((e = allow_smem(kc, s_comb)) != cudaSuccess) return e;
    kc<<<dim3(d.H, d.batch), kT, s_comb, s>>>(pm, pl, pz, static_cast<const WT*>(bv), lengths,
                                              static_cast<OT*>(out), status, d.H, d.d_h, d.r, d.max_len, W.S,
                                              nullptr);
    note_launch();
    return check_launch();
  }
  if constexpr (sizeof(WT) == 2) {
    float* zm = reinterpret_cast<float*>(wb + W.zm);
    auto kc = k_wsvd_combine<WT, OT, true>;
    if ((e = allow_smem(kc, s_comb)) != cudaSuccess) return e;
    kc<<<dim3(d.H, d.batch), kT, s_comb, s>>>(pm, pl, pz, nullptr, lengths, static_cast<OT*>(out), status, d.H,
                                              d.d_h, d.r, d.max_len, W.S, zm);
    note_launch();
    if ((e = check_launch()) != cudaSuccess) return e;
    return launch_gemv<float, WT, OT>(zm, static_cast<const WT*>(bv), reinterpret_cast<float*>(wb + W.ypart),
                                      d.batch, d.H * d.r, d.E, W.KSY, static_cast<OT*>(out),
                                      reinterpret_cast<int32_t*>(wb + W.tickets), status, s);
  } else {
    return cudaErrorInvalidValue;   // the fold needs 16-bit weights (refused on the host)
  }
}

template <typename WT, typename CT, typename OT>
cudaError_t wsvd_t(const qsvd_dims& d, const void* bk, const void* bv, const float* q, const void* ck,
                   const void* cv, const int32_t* lengths, float sl2, void* workspace,
                   const WsvdLayout& W, void* out, int token_major, cudaStream_t s) {
  uint8_t* wb = static_cast<uint8_t*>(workspace);
  int32_t* status = reinterpret_cast<int32_t*>(wb + W.hdr);
  float* qt = reinterpret_cast<float*>(wb + W.qt);
  float* pm = reinterpret_cast<float*>(wb + W.m);
  float* pl = reinterpret_cast<float*>(wb + W.l);
  float* pz = reinterpret_cast<float*>(wb + W.z);
  const size_t s_abs = size_t(d.d_h) * 4;
  const int ng = (d.r < kT && kT % d.r == 0) ? kT / d.r : 1;
  const size_t s_split = (size_t(d.r) + kWsvdChunk + 4 + size_t(ng) * d.r) * 4;
  const size_t s_comb = (size_t(W.S) + d.r + 4) * 4;
  cudaError_t e;
  auto ka = k_wsvd_absorb<WT>;
  auto ks = k_wsvd_split<CT>;
  if ((e = allow_smem(ka, s_abs)) != cudaSuccess || (e = allow_smem(ks, s_split)) != cudaSuccess)
    return e;
  const bool fold = d.out_proj == QSVD_OUT_PROJ_FOLD;
  int32_t* tickets = reinterpret_cast<int32_t*>(wb + W.tickets);
  if (d.rope) {
    // keys rebuilt and rotated on the tensor cores; then the chunk kernel
    // takes the scores and reads only the values
    if constexpr (sizeof(CT) == 2 && std::is_same<CT, WT>::value) {
      if ((e = launch_wsvd_rope_front(d, bk, q, ck, lengths, sl2, workspace, W, token_major, s)) != cudaSuccess)
        return e;
      const float* scores = reinterpret_cast<const float*>(wb + W.scores);
      auto kv = d.r == 64 ? k_wsvd_split_vec<CT, 64> : d.r == 128 ? k_wsvd_split_vec<CT, 128>
                                                                   : k_wsvd_split_vec<CT, 256>;
      kv<<<dim3(W.S, d.H, d.batch), kTV, 0, s>>>(static_cast<const CT*>(ck), static_cast<const CT*>(cv), qt,
                                                 lengths, pm, pl, pz, d.H, d.max_len, W.S, token_major, scores);
      note_launch();
      if ((e = check_launch()) != cudaSuccess) return e;
      return wsvd_combine<WT, OT>(d, pm, pl, pz, bv, lengths, out, status, W, wb, s_comb, s);
    } else {
      return cudaErrorInvalidValue;   // refused on the host (wsvd_rope_supported)
    }
  }
  ka<<<dim3(d.H, d.batch), kT, s_abs, s>>>(static_cast<const WT*>(bk), q, qt, status, d.H, d.d_h, d.r, sl2,
                                          tickets, fold ? W.NT : 0);
  note_launch();
  if ((e = check_launch()) != cudaSuccess) return e;
  if constexpr (sizeof(CT) == 2) {
    if (d.r == 64 || d.r == 128 || d.r == 256) {
      auto kv = d.r == 64 ? k_wsvd_split_vec<CT, 64> : d.r == 128 ? k_wsvd_split_vec<CT, 128>
                                                                   : k_wsvd_split_vec<CT, 256>;
      kv<<<dim3(W.S, d.H, d.batch), kTV, 0, s>>>(static_cast<const CT*>(ck), static_cast<const CT*>(cv), qt,
                                                 lengths, pm, pl, pz, d.H, d.max_len, W.S, token_major,
                                                 nullptr);
      note_launch();
      if ((e = check_launch()) != cudaSuccess) return e;
      return wsvd_combine<WT, OT>(d, pm, pl, pz, bv, lengths, out, status, W, wb, s_comb, s);
    }
  }
  ks<<<dim3(W.S, d.H, d.batch), kT, s_split, s>>>(static_cast<const CT*>(ck), static_cast<const CT*>(cv),
                                                  qt, lengths, pm, pl, pz, d.H, d.r, d.max_len, W.S,
                                                  token_major);
  note_launch();
  if ((e = check_launch()) != cudaSuccess) return e;
  return wsvd_combine<WT, OT>(d, pm, pl, pz, bv, lengths, out, status, W, wb, s_comb, s);
}

template <typename WT, typename CT>
cudaError_t wsvd_out(const qsvd_dims& d, const void* bk, const void* bv, const float* q, const void* ck,
                     const void* cv, const int32_t* lengths, float sl2, void* ws, const WsvdLayout& W,
                     void* out, int tm, cudaStream_t s) {
  switch (d.out_dtype) {
    case QSVD_F32: return wsvd_t<WT, CT, float>(d, bk, bv, q, ck, cv, lengths, sl2, ws, W, out, tm, s);
    case QSVD_F16: return wsvd_t<WT, CT, __half>(d, bk, bv, q, ck, cv, lengths, sl2, ws, W, out, tm, s);
    case QSVD_BF16: return wsvd_t<WT, CT, __nv_bfloat16>(d, bk, bv, q, ck, cv, lengths, sl2, ws, W, out, tm, s);
    default: return cudaErrorInvalidValue;
  }
}

template <typename WT>
cudaError_t wsvd_cache(const qsvd_dims& d, const void* bk, const void* bv, const float* q, const void* ck,
                       const void* cv, const int32_t* lengths, float sl2, void* ws, const WsvdLayout& W,
                       void* out, int tm, cudaStream_t s) {
  switch (d.cache_dtype) {
    case QSVD_F32: return wsvd_out<WT, float>(d, bk, bv, q, ck, cv, lengths, sl2, ws, W, out, tm, s);
    case QSVD_F16: return wsvd_out<WT, __half>(d, bk, bv, q, ck, cv, lengths, sl2, ws, W, out, tm, s);
    case QSVD_BF16: return wsvd_out<WT, __nv_bfloat16>(d, bk, bv, q, ck, cv, lengths, sl2, ws, W, out, tm, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_wsvd_decode(const qsvd_dims& d, const void* bk, const void* bv, const float* q,
                               const void* ck, const void* cv, const int32_t* lengths, float sl2,
                               void* workspace, const WsvdLayout& W, void* out, int token_major,
                               cudaStream_t s) {
  const int tm = token_major;
  switch (d.weight_dtype) {
    case QSVD_F32: return wsvd_cache<float>(d, bk, bv, q, ck, cv, lengths, sl2, workspace, W, out, tm, s);
    case QSVD_F16: return wsvd_cache<__half>(d, bk, bv, q, ck, cv, lengths, sl2, workspace, W, out, tm, s);
    case QSVD_BF16:
      return wsvd_cache<__nv_bfloat16>(d, bk, bv, q, ck, cv, lengths, sl2, workspace, W, out, tm, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qsvd
