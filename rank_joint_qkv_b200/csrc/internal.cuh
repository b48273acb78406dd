// Internal declarations of the joint-QKV latent decode library (sm_100a).
//
// Shared by the C-ABI layer (api.cu) and the kernel files.  Nothing here is
// part of the public interface (include/qsvd.h).
#pragma once

#include <cuda.h>

#include <cstring>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/qsvd.h"

namespace qsvd {

constexpr int kTile = QSVD_TILE_TOKENS;   // tokens per split-KV tile
// Split CTAs per call at most.  A sequence's tiles fall into a contiguous run
// of splits c0..c1; when G exceeds the tiles actually present, empty splits
// lie between them, so the run can span up to G indices.  The merge keeps
// one weight per index of the run in shared memory: the host caps G here.
constexpr int kMaxSplits = 2048;
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- layouts

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline size_t dtype_bytes(qsvd_dtype t) {
  switch (t) {
    case QSVD_F32: return 4;
    case QSVD_F16: case QSVD_BF16: return 2;
    default: return 1;
  }
}

// Bytes of one cache row (without scales).
inline size_t cache_row_bytes(const qsvd_dims& d) {
  switch (d.cache_dtype) {
    case QSVD_F32: return size_t(d.r) * 4;
    case QSVD_F16: case QSVD_BF16: return size_t(d.r) * 2;
    case QSVD_I8: return size_t(d.r);
    case QSVD_I4: return size_t(d.r) / 2;
  }
  return 0;
}

inline bool cache_is_int(const qsvd_dims& d) {
  return d.cache_dtype == QSVD_I8 || d.cache_dtype == QSVD_I4;
}

// Packed weights: one device buffer, 256-byte aligned sections.
struct PackedLayout {
  size_t wd, wuq, wuk, wuv;   // native layouts: W^d E x r, W^u_* r x E
  size_t wukT;                // W^u_k transposed, E x r (rotary tensor-core path)
  size_t h2q;                 // h2_m x h2_m float32 (online H2 in append)
  size_t rope;                // max_len x (d_h/2) x {cos, sin} float32
  size_t wo;                  // output projection: W_O E x E (chain) or F H r x E (fold)
  size_t total;
};

// Rows (K) of the output-projection GEMV: E for the chain, H r for the fold.
inline size_t out_proj_rows(const qsvd_dims& d) {
  return d.out_proj == QSVD_OUT_PROJ_FOLD ? size_t(d.H) * d.r
                                          : d.out_proj == QSVD_OUT_PROJ_CHAIN ? size_t(d.E) : 0;
}

inline PackedLayout packed_layout(const qsvd_dims& d) {
  PackedLayout p{};
  const size_t wb = dtype_bytes(d.weight_dtype);
  const size_t mat = size_t(d.E) * d.r * wb;
  size_t o = 256;  // reserved header
  p.wd = o;  o = align256(o + mat);
  p.wuq = o; o = align256(o + mat);
  p.wuk = o; o = align256(o + mat);
  p.wuv = o; o = align256(o + mat);
  p.wukT = o; if (d.rope) o = align256(o + mat);
  p.h2q = o; o = align256(o + size_t(16) * 16 * 4);
  p.rope = o; if (d.rope) o = align256(o + size_t(d.max_len) * (d.d_h / 2) * 2 * 4);
  p.wo = o;  o = align256(o + out_proj_rows(d) * d.E * wb);
  p.total = o;
  return p;
}

// Workspace of qsvd_decode_attn.
struct WsHeader {
  int32_t status;
  int32_t G;       // split CTAs of the split phase
  int32_t tile;    // tokens per tile
  int32_t kernel;  // split kernel used
};

struct WsLayout {
  size_t hdr, sched, tickets, q, qt32, qt16, qpart, pm, pl, pz, opart, zm, scores, ow, ypart, total;
  int G, P, KS, JS, NT, NTQ, NTV;   // NT tickets in all: NTQ query GEMV, NTV V-up GEMV, then the
                                    // output projection's
  int KSY;                          // split-K of the output-projection GEMV
};

// GEMV (gemv.cuh) split of K: one 64 KB tile per CTA -- 512 rows x 64 columns for 16-bit
// weights (tensor cores), 64 rows x 256 columns for fp32 (CUDA cores).
// Shape-only, device-independent.
inline int gemv_ksplit(int K, qsvd_dtype wt) {
  const int rt = wt == QSVD_F32 ? 64 : 512;
  return (K + rt - 1) / rt;
}

// Ticket counters: one per (column block, block of 16 sequences).
inline int gemv_tickets(int N, int B, qsvd_dtype wt) {
  const int cw = wt == QSVD_F32 ? 256 : 64;
  return ((N + cw - 1) / cw) * ((B + 15) / 16);
}

// Split-K factor of the query projection and j-splits of the combine.
int prologue_ksplit(const qsvd_dims& d);   // split of r in q = c_new W^u_q
inline int combine_jsplit(const qsvd_dims& d) { return (d.r + 127) / 128; }

int prologue_tickets(const qsvd_dims& d);  // ticket counters of that GEMV
int gemv_tickets_vup(const qsvd_dims& d);  // ticket counters of the combine's V-up GEMV

inline WsLayout ws_layout(const qsvd_dims& d, int G) {
  WsLayout w{};
  w.G = G;
  w.P = G + d.batch;
  w.KS = prologue_ksplit(d);
  w.JS = combine_jsplit(d);
  w.NTQ = prologue_tickets(d);
  w.NTV = gemv_tickets_vup(d);          // then the V-up GEMV's (combine)
  w.KSY = d.out_proj ? gemv_ksplit(int(out_proj_rows(d)), d.weight_dtype) : 0;
  w.NT = w.NTQ + w.NTV + (d.out_proj ? gemv_tickets(d.E, d.batch, d.weight_dtype) : 0);
  const size_t B = d.batch, E = d.E, H = d.H, r = d.r;
  size_t o = 0;
  w.hdr = o;   o = align256(o + sizeof(WsHeader));
  w.sched = o; o = align256(o + (2 * B + 1) * 4);
  w.tickets = o; o = align256(o + size_t(w.NT) * 4);
  w.q = o;     o = align256(o + B * E * 4);
  w.qt32 = o;  o = align256(o + (H * r > E ? H * r : E) * B * 4);   // rotary mode: B x E query
  w.qt16 = o;  o = align256(o + 2 * B * H * r * 2);   // [B][2][H][r] for bf16 hi/lo
  w.qpart = o; o = align256(o + size_t(w.KS) * B * E * 4);
  w.pm = o;    o = align256(o + size_t(w.P) * H * 4);
  w.pl = o;    o = align256(o + size_t(w.P) * H * 4);
  w.pz = o;    o = align256(o + size_t(w.P) * H * r * 4);
  w.opart = o; o = align256(o + size_t(w.JS) * B * E * 4);   // also the V-up GEMV's partials
  w.zm = o;    o = align256(o + B * H * r * 4);                 // merged latents [B][H][r]
  w.scores = o; if (d.rope) o = align256(o + B * H * size_t(d.max_len) * 4);   // rotary: [B][H][max_len]
  w.ow = o;    if (d.out_proj == QSVD_OUT_PROJ_CHAIN) o = align256(o + B * E * 4);   // o before W_O
  w.ypart = o; o = align256(o + size_t(w.KSY) * B * E * 4);    // output-projection partials
  w.total = o;
  return w;
}

// -------------------------------------------------------- launch bookkeeping

void note_launch();                 // counts kernels launched by this library
qsvd_status set_error(qsvd_status st, const char* msg);   // records qsvd_last_error()
cudaError_t check_launch();         // cudaGetLastError after a launch

// Programmatic dependent launch.  The decode-step kernels are launched with
// programmatic stream serialisation, so each may start while the previous
// kernel in the stream is still running.  Every such kernel executes
// dev::pdl_wait() -- which returns once the previous grid has completed and
// its memory is visible -- before it reads or writes any global memory that
// an earlier kernel produces or consumes; before the wait it only reads the
// packed weights (written by qsvd_prepare_weights) and sets up its own shared
// memory.  It calls dev::pdl_trigger() after the wait, so a kernel starts
// only once its predecessor's predecessor has completed, and a chain of such
// kernels stays ordered transitively.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// cuTensorMapEncodeTiled, reached through the runtime's driver entry point
// (no link against the driver library); null if the driver lacks it.
using TensorMapEncode = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                     const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                     const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
TensorMapEncode tensor_map_encoder();

// ------------------------------------------------------------ kernel entry

// Prologue (query side).
cudaError_t launch_schedule(const qsvd_dims& d, const int32_t* lengths, int G, int32_t* sched,
                            WsHeader* hdr, int kernel, int32_t* tickets, int n_tickets,
                            cudaStream_t s);
cudaError_t launch_q_partial(const qsvd_dims& d, const float* qin, const void* wuq,
                             float* qpart, int KS, float* q, int32_t* tickets, int32_t* status,
                             cudaStream_t s);
// qt32 (fp32, for the CUDA-core split) and qt16 ([B][2][H][r] hi/lo, for the
// tensor cores) are each written only when non-null.
cudaError_t launch_absorb(const qsvd_dims& d, const float* q, const void* wuk, float scale_log2,
                          float* qt32, void* qt16, int32_t* status, cudaStream_t s);
// Quantised latent on the tensor cores: qt32 [B][H][r] -> three int8 parts
// qp [B][3][H][r] and one power-of-two scale qs [B][H] per (sequence, head).
cudaError_t launch_quant_query(const qsvd_dims& d, const float* qt, int8_t* qp, float* qs, cudaStream_t s);
cudaError_t launch_rope_query(const qsvd_dims& d, const float* q, const int32_t* sched,
                              const float* rope_tab, float scale_log2, float* qrot,
                              cudaStream_t s);

// Split phase.
cudaError_t launch_split_simt_absorbed(const qsvd_dims& d, const float* qt32,
                                       const void* cache, const void* scales,
                                       const int32_t* sched, int G, float* pm,
                                       float* pl, float* pz, cudaStream_t s);
// Rotary mode on the tensor cores: keys rebuilt from the latent, rotated,
// scored against the rotary query into `scores` ([B][H][max_len]); then a
// split kernel runs the softmax and the latent accumulation on them (the
// tensor-core one when split_tc_scores_supported, else the CUDA-core one).
bool rope_tc_supported(const qsvd_dims& d);
cudaError_t launch_rope_scores(const qsvd_dims& d, const void* cache, const void* wukT,
                               const float* qrot, const float* rope_tab, const int32_t* sched,
                               int G, float* scores, int32_t* status, cudaStream_t s);
bool split_tc_scores_supported(const qsvd_dims& d);
int split_tc_scores_parts(const qsvd_dims& d);   // CTAs sharing one split's channels
cudaError_t launch_split_tc_scores(const qsvd_dims& d, const float* scores, const void* cache,
                                   const int32_t* sched, int G, float* pm, float* pl, float* pz,
                                   int32_t* status, cudaStream_t s);
cudaError_t launch_split_simt_scores(const qsvd_dims& d, const float* scores, const void* cache,
                                     const void* scales, const int32_t* sched, int G, float* pm,
                                     float* pl, float* pz, cudaStream_t s);
cudaError_t launch_split_simt_rope(const qsvd_dims& d, const float* qrot,
                                   const void* wuk, const float* rope_tab,
                                   const void* cache, const void* scales,
                                   const int32_t* sched, int G, float* pm,
                                   float* pl, float* pz, cudaStream_t s);
int split_simt_grid_heads(const qsvd_dims& d);   // head blocks per split
bool split_tc_supported(const qsvd_dims& d);
// Absorbed mode, the tile's channels spread over a thread-block cluster;
// G = the number of clusters (split_cl_clusters: as many as fit at once).
bool split_cl_supported(const qsvd_dims& d);
int split_cl_clusters(const qsvd_dims& d);
cudaError_t launch_split_cl(const qsvd_dims& d, const void* cache, const void* qt16, const int32_t* sched,
                            int G, float* pm, float* pl, float* pz, int32_t* status, cudaStream_t s);
// Absorbed mode, one CTA per split (tcgen05).  qt16: the query as 16-bit
// hi/lo parts, or for an int8/int4 latent its int8 parts (launch_quant_query)
// with qsh their per-(sequence, head) scales.
cudaError_t launch_split_tc(const qsvd_dims& d, const void* cache, const void* scales, const void* qt16,
                            const int32_t* sched, int G, float* pm, float* pl, float* pz,
                            int32_t* status, cudaStream_t s, const float* qsh = nullptr);

// Prefill of the latent cache (tcgen05 GEMM x W^d with the append path's
// rounding / quantisation fused): 16-bit weights, r % 256 == 0, E % 64 == 0,
// H2 folded into the weights (not the online mode).
bool prefill_supported(const qsvd_dims& d);
cudaError_t launch_prefill(const qsvd_dims& d, const void* wd, const void* x, int n_rows,
                           const int32_t* dst_rows, void* cache, void* scales, float* c_out,
                           int32_t* status, cudaStream_t s);

// Combine phase.  16-bit weights with d_h % 64 == 0: a merge kernel writes
// the merged latents zm, then the tensor-core GEMV applies W^u_v per head;
// otherwise one kernel merges and applies W^u_v per (head, 128 rows of r).
// Prefill attention (prefill_attn.cu): workspace sections and launcher.
struct PrefillAttnWs {
  float* stage;     // [B max_len][E] float32 rows of the GEMM (Q, then K, then V)
  void* q[2];       // hi, lo parts [B max_len][E], cache type
  void* k[2];
  void* v[2];
  size_t total;     // bytes
};
bool prefill_attention_supported(const qsvd_dims& d);
PrefillAttnWs prefill_attention_ws(const qsvd_dims& d, void* workspace);
cudaError_t launch_prefill_attention(const qsvd_dims& d, const void* wuq, const void* wuk, const void* wuv,
                                     const float* rope_tab, const void* cache, const int32_t* lengths,
                                     const PrefillAttnWs& w, void* out, int32_t* status, float sl2,
                                     cudaStream_t s);

bool combine_uses_gemv(const qsvd_dims& d);
cudaError_t set_score_wait_ns(unsigned long long ns);   // test hook of the split kernel
// Merge + V-up on the tensor-core GEMV.  With d.out_proj the output is
// projected by W_O: CHAIN runs the V-up into `ow` (B x E fp32) and a second
// GEMV by `wo` (E x E); FOLD skips the V-up and runs one GEMV of the merged
// latents (B x H r) by `wo` = F (H r x E).  `ypart` holds that GEMV's KSY
// split-K partials; `ytickets` its ticket counters.
struct OutProj {
  const void* wo;
  float* ow;
  float* ypart;
  int32_t* ytickets;
};
cudaError_t launch_combine_gemv(const qsvd_dims& d, const WsHeader* hdr, const int32_t* sched,
                                const float* pm, const float* pl, const float* pz, const void* wuv,
                                float* zm, float* vpart, int32_t* tickets, int32_t* status, void* out,
                                const OutProj& op, cudaStream_t s);
cudaError_t launch_combine(const qsvd_dims& d, const WsHeader* hdr, const int32_t* sched,
                           const float* pm, const float* pl, const float* pz,
                           const void* wuv, float* opart, int JS, int P, void* out,
                           cudaStream_t s);

// Append.
int append_ksplit(const qsvd_dims& d);
cudaError_t launch_append(const qsvd_dims& d, const void* x, const void* wd,
                          const float* h2q, float h2_scale, const int32_t* pos,
                          void* cache, void* scales, float* c_out, float* cpart,
                          int KS, int32_t* status, cudaStream_t s);

// Prepare.
cudaError_t launch_prepare(const qsvd_dims& d, const void* wd, const void* wuq,
                           const void* wuk, const void* wuv, const float* h2q_host,
                           void* packed, const PackedLayout& L, cudaStream_t s);
// Factors of one singular-value split: W^d = U diag(a), W^u = diag(b) V^T.
cudaError_t launch_split_factors(const qsvd_dims& d, const float* u, const float* vt, const float* a,
                                 const float* b, void* wd, void* wuq, void* wuk, void* wuv,
                                 cudaStream_t s);
// Output-projection section of the packed buffer: W_O copied (CHAIN) or the
// per-head fold F = W^u_{v,h} W_{O,h} (FOLD); W^u_v read from the buffer.
cudaError_t launch_beta_split(const float* sigma, double beta, float* a, float* b, int r, cudaStream_t s);
cudaError_t launch_sq_diff_sum(const float* y, const float* yq, size_t n, double* out, cudaStream_t s);
cudaError_t launch_per_head_fold(const qsvd_dims& d, const void* bv, const void* wo, void* f, cudaStream_t s);
cudaError_t launch_prepare_out_proj(const qsvd_dims& d, const void* wo, void* packed,
                                    const PackedLayout& L, cudaStream_t s);

}  // namespace qsvd

// ------------------------------------------------------------ device helpers

namespace qsvd {
namespace dev {
// This CTA's share of [p, p + bytes) requested into L2 by bulk prefetches
// (16-byte granules, 64 KB per request): a hint for the kernel that reads
// those bytes next, with no effect on any result.  p 16-byte aligned.
__device__ __forceinline__ void l2_prefetch_share(const uint8_t* p, unsigned long long bytes) {
  const unsigned long long ncta = (unsigned long long)gridDim.x * gridDim.y * gridDim.z;
  const unsigned long long cta =
      blockIdx.x + (unsigned long long)gridDim.x * (blockIdx.y + (unsigned long long)gridDim.y * blockIdx.z);
  const unsigned long long end = bytes & ~15ull;
  const unsigned long long share = ((end + ncta - 1) / ncta + 15) & ~15ull;
  unsigned long long lo = cta * share;
  const unsigned long long hi = lo + share < end ? lo + share : end;
  for (; lo < hi; lo += 65536) {
    const unsigned n = unsigned(hi - lo < 65536 ? hi - lo : 65536);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p + lo), "r"(n) : "memory");
  }
}


// See launch_pdl.  A no-op when the kernel was launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

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

// sum_{k < n} p[k * stride] in order k = 0, 1, ..., with the loads issued in
// batches of 8 so that they are in flight together (L2 path, no L1).
__device__ __forceinline__ float sum_strided(const float* p, size_t stride, int n) {
  float s = 0.f;
  int k = 0;
  for (; k + 8 <= n; k += 8) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __ldcg(p + size_t(k + i) * stride);
#pragma unroll
    for (int i = 0; i < 8; ++i) s += v[i];
  }
  for (; k < n; ++k) s += __ldcg(p + size_t(k) * stride);
  return s;
}

// Reduce v[0..N) over the 32 lanes of a warp (N a power of two <= 32) with a
// transposing butterfly: each round a lane keeps the half of its elements
// whose index bit matches its own lane bit and adds the partner's copy of
// that half, so lane L ends with the reduction of element L % N after
// N - 1 + log2(32 / N) shuffles (32 separate reductions would take 5 N).
// v is overwritten.
struct OpAdd { __device__ float operator()(float a, float b) const { return a + b; } };
struct OpMax { __device__ float operator()(float a, float b) const { return fmaxf(a, b); } };
template <int N, typename Op>
__device__ __forceinline__ float warp_reduce_transposed(float (&v)[N], int lane, Op op) {
#pragma unroll
  for (int k = N / 2; k >= 1; k >>= 1) {
    const bool upper = (lane & k) != 0;
#pragma unroll
    for (int j = 0; j < k; ++j) {
      const float send = upper ? v[j] : v[j + k];
      const float keep = upper ? v[j + k] : v[j];
      v[j] = op(keep, __shfl_xor_sync(0xffffffffu, send, k));
    }
  }
  float x = v[0];
#pragma unroll
  for (int k = N; k < 32; k <<= 1) x = op(x, __shfl_xor_sync(0xffffffffu, x, k));
  return x;
}

// Number of tiles of a sequence of n tokens.
__device__ __forceinline__ int tiles_of(int n) { return (n + kTile - 1) / kTile; }

// Clamp a device length into [0, max_len]; flag out-of-range values.
__device__ __forceinline__ int clamp_len(int n, int max_len, int32_t* status) {
  if (n < 0 || n > max_len) {
    if (status) atomicOr(status, QSVD_STATUS_LEN_CLAMPED);
    n = n < 0 ? 0 : max_len;
  }
  return n;
}

// Split c of G covers global tiles [split_begin(c), split_begin(c + 1)).
__device__ __forceinline__ long long split_begin(long long c, long long G, long long T) {
  return (c * T) / G;
}
// The split whose range contains global tile t.
__device__ __forceinline__ long long split_of_tile(long long t, long long G, long long T) {
  return ((t + 1) * G - 1) / T;
}

// Sixteen bytes of a cache row converted to float.  Element index j0 is the
// first of the vector; `scale` is the group scale for int caches.
template <qsvd_dtype CT> struct CacheVec;

template <> struct CacheVec<QSVD_F32> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const uint8_t* row, int j0, float s, float* o) {
    float4 v = *reinterpret_cast<const float4*>(row + size_t(j0) * 4);
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
  }
};
template <> struct CacheVec<QSVD_F16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const uint8_t* row, int j0, float s, float* o) {
    uint4 v = *reinterpret_cast<const uint4*>(row + size_t(j0) * 2);
    const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) { float2 f = __half22float2(h[i]); o[2 * i] = f.x; o[2 * i + 1] = f.y; }
  }
};
template <> struct CacheVec<QSVD_BF16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const uint8_t* row, int j0, float s, float* o) {
    uint4 v = *reinterpret_cast<const uint4*>(row + size_t(j0) * 2);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) { float2 f = __bfloat1622float2(h[i]); o[2 * i] = f.x; o[2 * i + 1] = f.y; }
  }
};
template <> struct CacheVec<QSVD_I8> {
  static constexpr int N = 16;
  __device__ __forceinline__ static void load(const uint8_t* row, int j0, float s, float* o) {
    uint4 v = *reinterpret_cast<const uint4*>(row + size_t(j0));
    const int8_t* c = reinterpret_cast<const int8_t*>(&v);
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = float(c[i]) * s;
  }
};
template <> struct CacheVec<QSVD_I4> {
  static constexpr int N = 32;
  __device__ __forceinline__ static void load(const uint8_t* row, int j0, float s, float* o) {
    uint4 v = *reinterpret_cast<const uint4*>(row + size_t(j0) / 2);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        // nibble i of word k is element 8k + i (low nibble first)
        int q = int((w[k] >> (4 * i)) & 0xFu);
        q = (q ^ 8) - 8;  // sign-extend 4-bit two's complement
        o[8 * k + i] = float(q) * s;
      }
    }
  }
};

}  // namespace dev
}  // namespace qsvd
