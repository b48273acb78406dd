// C-ABI layer: argument validation, layouts, phase dispatch.
#include <atomic>
#include <cstdarg>
#include <cmath>
#include <cstdio>
#include <cstring>

#include "internal.cuh"
#include "wsvd.cuh"

namespace qsvd {

static std::atomic<uint64_t> g_launches{0};
static thread_local char g_err[512] = "";

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
cudaError_t check_launch() { return cudaGetLastError(); }

TensorMapEncode tensor_map_encoder() {
  static TensorMapEncode fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<TensorMapEncode>(p);
    return TensorMapEncode(nullptr);
  }();
  return fn;
}

static qsvd_status fail(qsvd_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

qsvd_status set_error(qsvd_status st, const char* msg) { return fail(st, "%s", msg); }

static qsvd_status cuda_fail(cudaError_t e, const char* where) {
  return fail(QSVD_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

static bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// fp16 group scales are read and written two bytes at a time, fp32 outputs
// four (the decode's fp32 output 16: it is stored as float4)
static bool aligned2(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 1u) == 0; }
static bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Host-checkable constraints shared by all calls.
static qsvd_status validate(const qsvd_dims* d) {
  if (!d) return fail(QSVD_ERR_INVALID_ARG, "dims is NULL");
  if (d->H <= 0 || d->d_h <= 0 || (long long)d->E != (long long)d->H * d->d_h)
    return fail(QSVD_ERR_INVALID_ARG, "E (%d) must equal H (%d) * d_h (%d)", d->E, d->H, d->d_h);
  if (d->E % 64) return fail(QSVD_ERR_INVALID_ARG, "E (%d) must be a multiple of 64", d->E);
  if (d->d_h % 8 || d->d_h > 256)
    return fail(QSVD_ERR_INVALID_ARG, "d_h (%d) must be a multiple of 8, at most 256", d->d_h);
  if (d->r < 32 || d->r % 32 || d->r > 8192)
    return fail(QSVD_ERR_INVALID_ARG, "r (%d) must be a multiple of 32 in [32, 8192]", d->r);
  // several kernels put the sequences on a grid's y or z axis
  if (d->batch < 1 || d->batch > 65535) return fail(QSVD_ERR_INVALID_ARG, "batch must be in [1, 65535]");
  if (d->max_len < 1) return fail(QSVD_ERR_INVALID_ARG, "max_len must be >= 1");
  // cache rows b * max_len + t are tensor-map coordinates and int indices
  if ((long long)d->batch * d->max_len > 0x7FFFFFFFLL)
    return fail(QSVD_ERR_INVALID_ARG, "batch x max_len (%lld) must be below 2^31",
                (long long)d->batch * d->max_len);
  if (d->cache_dtype < QSVD_F32 || d->cache_dtype > QSVD_I4)
    return fail(QSVD_ERR_INVALID_ARG, "unknown cache dtype %d", int(d->cache_dtype));
  if (d->weight_dtype < QSVD_F32 || d->weight_dtype > QSVD_BF16)
    return fail(QSVD_ERR_INVALID_ARG, "weight dtype must be F32, F16 or BF16");
  if (d->out_dtype < QSVD_F32 || d->out_dtype > QSVD_BF16)
    return fail(QSVD_ERR_INVALID_ARG, "out dtype must be F32, F16 or BF16");
  if (cache_is_int(*d)) {
    if (d->group < 32 || d->group > 1024 || d->group % 32 || d->r % d->group)
      return fail(QSVD_ERR_INVALID_ARG,
                  "group (%d) must be a multiple of 32 in [32, 1024] dividing r (%d)",
                  d->group, d->r);
  }
  if (d->rope) {
    if (!(d->rope_base > 0.f)) return fail(QSVD_ERR_INVALID_ARG, "rope_base must be > 0");
    if (d->d_h % 64) return fail(QSVD_ERR_UNSUPPORTED, "rotary mode needs d_h %% 64 == 0");
  }
  if (d->h2) {
    if (d->h2_m < 1 || d->h2_m > 16 || d->r % d->h2_m || !is_pow2(d->r / d->h2_m))
      return fail(QSVD_ERR_INVALID_ARG, "H2 needs r/h2_m a power of two, 1 <= h2_m <= 16");
  }
  if (d->kernel < QSVD_KERNEL_AUTO || d->kernel > QSVD_KERNEL_TCGEN05_CLUSTER)
    return fail(QSVD_ERR_INVALID_ARG, "unknown kernel choice %d", d->kernel);
  if (d->out_proj < QSVD_OUT_PROJ_NONE || d->out_proj > QSVD_OUT_PROJ_FOLD)
    return fail(QSVD_ERR_INVALID_ARG, "unknown out_proj %d", d->out_proj);
  return QSVD_OK;
}

static int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return sms;
}

// Split kernel actually used for these dims: SIMT, TCGEN05_CTA or
// TCGEN05_CLUSTER (the rotary tensor-core path counts as one CTA per split).
// The tensor-core choice prefers one CTA per split: on the LLaVA-7B fp16
// workload it measured 112 us against 515 us for the cluster kernel, whose
// per-tile cross-CTA exchange of partial scores sits on the softmax's path.
static int pick_kernel(const qsvd_dims& d) {
  const bool cl = split_cl_supported(d);
  switch (d.kernel) {
    case QSVD_KERNEL_SIMT:
    case QSVD_KERNEL_TCGEN05_CTA:
    case QSVD_KERNEL_TCGEN05_CLUSTER:
      return d.kernel;
    case QSVD_KERNEL_TCGEN05:
      if (d.rope || split_tc_supported(d)) return QSVD_KERNEL_TCGEN05_CTA;
      return cl ? QSVD_KERNEL_TCGEN05_CLUSTER : QSVD_KERNEL_TCGEN05_CTA;
    default:
      if (d.rope) return rope_tc_supported(d) ? QSVD_KERNEL_TCGEN05_CTA : QSVD_KERNEL_SIMT;
      return split_tc_supported(d) ? QSVD_KERNEL_TCGEN05_CTA : (cl ? QSVD_KERNEL_TCGEN05_CLUSTER : QSVD_KERNEL_SIMT);
  }
}

static qsvd_status resolve_splits(const qsvd_dims& d, int num_splits, int kernel, int* G) {
  const long long max_tiles = (long long)d.batch * ((d.max_len + kTile - 1) / kTile);
  long long g = num_splits;
  if (num_splits < 0) return fail(QSVD_ERR_INVALID_ARG, "num_splits must be >= 0");
  if (g == 0) {
    const int sms = device_sms();
    if (sms <= 0) return fail(QSVD_ERR_CUDA, "no CUDA device to size the split grid");
    if (kernel == QSVD_KERNEL_TCGEN05_CLUSTER) {
      g = split_cl_clusters(d);   // as many clusters as fit at once
      if (g <= 0) return fail(QSVD_ERR_CUDA, "no cluster configuration fits this device");
    } else if (kernel == QSVD_KERNEL_TCGEN05_CTA && !d.rope) {
      g = sms;   // one CTA per SM (persistent over its tile range)
    } else if (kernel == QSVD_KERNEL_TCGEN05_CTA && split_tc_scores_supported(d)) {
      g = sms / split_tc_scores_parts(d);   // ch CTAs per split, one per SM
      if (g < 1) g = 1;
    } else {
      const int hb = split_simt_grid_heads(d);
      g = hb > 0 ? (2LL * sms + hb - 1) / hb : sms;
    }
  }
  if (g > max_tiles) g = max_tiles;
  if (g > kMaxSplits) g = kMaxSplits;
  if (g < 1) g = 1;
  *G = int(g);
  return QSVD_OK;
}

static float score_scale_log2(const qsvd_dims& d) {
  const double tau = d.softmax_scale > 0.f ? double(d.softmax_scale) : 1.0 / std::sqrt(double(d.d_h));
  return float(tau * 1.4426950408889634);
}

}  // namespace qsvd

using namespace qsvd;

extern "C" {

const char* qsvd_status_string(qsvd_status s) {
  switch (s) {
    case QSVD_OK: return "QSVD_OK";
    case QSVD_ERR_INVALID_ARG: return "QSVD_ERR_INVALID_ARG";
    case QSVD_ERR_UNSUPPORTED: return "QSVD_ERR_UNSUPPORTED";
    case QSVD_ERR_WORKSPACE: return "QSVD_ERR_WORKSPACE";
    case QSVD_ERR_CUDA: return "QSVD_ERR_CUDA";
  }
  return "QSVD_UNKNOWN_STATUS";
}

const char* qsvd_last_error(void) { return g_err; }

uint64_t qsvd_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

int qsvd_abi_version(void) { return QSVD_ABI_VERSION; }

qsvd_status qsvd_testing_set_score_wait_ns(unsigned long long ns) {
  const cudaError_t e = set_score_wait_ns(ns);
  if (e != cudaSuccess) return cuda_fail(e, "qsvd_testing_set_score_wait_ns");
  return QSVD_OK;
}

qsvd_status qsvd_prepare_weights(const qsvd_dims* dims, const void* wd, const void* wuq,
                                 const void* wuk, const void* wuv, const float* h2_q,
                                 void* packed, size_t* packed_bytes, void* stream) {
  qsvd_status st = validate(dims);
  if (st != QSVD_OK) return st;
  if (!packed_bytes) return fail(QSVD_ERR_INVALID_ARG, "packed_bytes is NULL");
  const qsvd_dims& d = *dims;
  if (h2_q && (d.h2_m < 1 || d.h2_m > 16 || d.r % d.h2_m || !is_pow2(d.r / d.h2_m)))
    return fail(QSVD_ERR_INVALID_ARG, "H2 needs r/h2_m a power of two, 1 <= h2_m <= 16");
  const PackedLayout L = packed_layout(d);
  if (!packed) { *packed_bytes = L.total; return QSVD_OK; }
  if (d.h2 && !h2_q) return fail(QSVD_ERR_INVALID_ARG, "dims->h2 = 1 needs h2_q");
  if (*packed_bytes < L.total)
    return fail(QSVD_ERR_WORKSPACE, "packed buffer holds %zu bytes, %zu needed", *packed_bytes, L.total);
  if (!wd || !wuq || !wuk || !wuv) return fail(QSVD_ERR_INVALID_ARG, "a weight pointer is NULL");
  if ((reinterpret_cast<uintptr_t>(packed) & 255u) != 0)
    return fail(QSVD_ERR_INVALID_ARG, "packed must be 256-byte aligned");
  *packed_bytes = L.total;
  cudaError_t e = launch_prepare(d, wd, wuq, wuk, wuv, h2_q, packed, L,
                                 static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prepare_weights");
  return QSVD_OK;
}

qsvd_status qsvd_split_factors(const qsvd_dims* dims, const float* u, const float* vt,
                               const float* a, const float* b, void* wd, void* wuq, void* wuk,
                               void* wuv, void* stream) {
  qsvd_status st = validate(dims);
  if (st != QSVD_OK) return st;
  if (!u || !vt || !a || !b || !wd || !wuq || !wuk || !wuv)
    return fail(QSVD_ERR_INVALID_ARG, "a required pointer is NULL");
  cudaError_t e = launch_split_factors(*dims, u, vt, a, b, wd, wuq, wuk, wuv,
                                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "split_factors");
  return QSVD_OK;
}

qsvd_status qsvd_beta_exponents(const float* sigma, int r, double beta, float* a, float* b, void* stream) {
  if (r < 1 || r > 8192) return fail(QSVD_ERR_INVALID_ARG, "r (%d) must be in [1, 8192]", r);
  if (!sigma || !a || !b) return fail(QSVD_ERR_INVALID_ARG, "a required pointer is NULL");
  cudaError_t e = launch_beta_split(sigma, beta, a, b, r, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "beta_exponents");
  return QSVD_OK;
}

qsvd_status qsvd_sq_diff_sum(const float* y, const float* yq, int64_t n, double* out, void* stream) {
  if (n < 0) return fail(QSVD_ERR_INVALID_ARG, "n must be >= 0");
  if (!y || !yq || !out) return fail(QSVD_ERR_INVALID_ARG, "a required pointer is NULL");
  cudaError_t e = launch_sq_diff_sum(y, yq, size_t(n), out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "sq_diff_sum");
  return QSVD_OK;
}

qsvd_status qsvd_prepare_out_proj(const qsvd_dims* dims, const void* wo, void* packed,
                                  size_t packed_bytes, void* stream) {
  qsvd_status st = validate(dims);
  if (st != QSVD_OK) return st;
  const qsvd_dims& d = *dims;
  if (d.out_proj == QSVD_OUT_PROJ_NONE)
    return fail(QSVD_ERR_INVALID_ARG, "dims->out_proj is QSVD_OUT_PROJ_NONE");
  if (!combine_uses_gemv(d))
    return fail(QSVD_ERR_UNSUPPORTED,
                "the output projection needs 16-bit weights, d_h %% 64 == 0, r %% 32 == 0");
  if (!wo || !packed) return fail(QSVD_ERR_INVALID_ARG, "wo/packed is NULL");
  const PackedLayout L = packed_layout(d);
  if (packed_bytes < L.total)
    return fail(QSVD_ERR_WORKSPACE, "packed buffer holds %zu bytes, %zu needed", packed_bytes, L.total);
  if ((reinterpret_cast<uintptr_t>(packed) & 255u) != 0)
    return fail(QSVD_ERR_INVALID_ARG, "packed must be 256-byte aligned");
  cudaError_t e = launch_prepare_out_proj(d, wo, packed, L, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prepare_out_proj");
  return QSVD_OK;
}

qsvd_status qsvd_append_latent(const qsvd_dims* dims, const void* packed, const void* x,
                               const int32_t* pos, void* cache, void* scales, float* c_out,
                               int32_t* status, void* workspace, size_t* workspace_bytes,
                               void* stream) {
  qsvd_status st = validate(dims);
  if (st != QSVD_OK) return st;
  const qsvd_dims& d = *dims;
  if (!workspace_bytes) return fail(QSVD_ERR_INVALID_ARG, "workspace_bytes is NULL");
  const int KS = append_ksplit(d);
  const size_t need = align256(size_t(KS) * d.batch * d.r * 4);
  if (!workspace) { *workspace_bytes = need; return QSVD_OK; }
  if (*workspace_bytes < need)
    return fail(QSVD_ERR_WORKSPACE, "append workspace holds %zu bytes, %zu needed", *workspace_bytes, need);
  if (!packed || !x || !pos || !cache) return fail(QSVD_ERR_INVALID_ARG, "a required pointer is NULL");
  if (cache_is_int(d) && !scales) return fail(QSVD_ERR_INVALID_ARG, "int caches need scales");
  if (!aligned16(x) || !aligned16(cache) || !aligned16(workspace))
    return fail(QSVD_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if ((scales && !aligned2(scales)) || (c_out && !aligned4(c_out)))
    return fail(QSVD_ERR_INVALID_ARG, "scales must be 2-byte and c_out 4-byte aligned");
  const PackedLayout L = packed_layout(d);
  const uint8_t* P = static_cast<const uint8_t*>(packed);
  const float h2_scale = d.h2 ? float(1.0 / std::sqrt(double(d.r / d.h2_m))) : 1.f;
  cudaError_t e = launch_append(d, x, P + L.wd, reinterpret_cast<const float*>(P + L.h2q), h2_scale,
                                pos, cache, scales, c_out, static_cast<float*>(workspace), KS,
                                status, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "append_latent");
  return QSVD_OK;
}

qsvd_status qsvd_prefill_latent(const qsvd_dims* dims, const void* packed, const void* x, int n_rows,
                                const int32_t* dst_rows, void* cache, void* scales, float* c_fp32_debug,
                                int32_t* status, void* stream) {
  qsvd_status st = validate(dims);
  if (st != QSVD_OK) return st;
  const qsvd_dims& d = *dims;
  if (n_rows < 0) return fail(QSVD_ERR_INVALID_ARG, "n_rows must be >= 0");
  if (!prefill_supported(d) || (cache_is_int(d) && d.group != 128))
    return fail(QSVD_ERR_UNSUPPORTED,
                "prefill needs 16-bit weights, r %% 256 == 0, E %% 64 == 0, group 128, H2 folded into the weights");
  if (n_rows == 0) return QSVD_OK;
  if (!packed || !x || !dst_rows || !cache) return fail(QSVD_ERR_INVALID_ARG, "a required pointer is NULL");
  if (cache_is_int(d) && !scales) return fail(QSVD_ERR_INVALID_ARG, "int caches need scales");
  if (scales && !aligned2(scales)) return fail(QSVD_ERR_INVALID_ARG, "scales must be 2-byte aligned");
  if (!aligned16(x) || !aligned16(cache) || (c_fp32_debug && !aligned16(c_fp32_debug)))
    return fail(QSVD_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const PackedLayout L = packed_layout(d);
  const uint8_t* P = static_cast<const uint8_t*>(packed);
  cudaError_t e = launch_prefill(d, P + L.wd, x, n_rows, dst_rows, cache, scales, c_fp32_debug, status,
                                 static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prefill_latent");
  return QSVD_OK;
}

qsvd_status qsvd_prefill_attention(const qsvd_dims* dims, const void* packed, const void* cache,
                                   const int32_t* lengths, void* workspace, size_t* workspace_bytes,
                                   void* out, int32_t* status, void* stream) {
  qsvd_status st = validate(dims);
  if (st != QSVD_OK) return st;
  const qsvd_dims& d = *dims;
  if (!workspace_bytes) return fail(QSVD_ERR_INVALID_ARG, "workspace_bytes is NULL");
  if (!prefill_attention_supported(d))
    return fail(QSVD_ERR_UNSUPPORTED,
                "prefill attention needs d_h == 128, an F16 or BF16 cache of the weight type, "
                "E %% 256 == 0 and r %% 64 == 0");
  const PrefillAttnWs need = prefill_attention_ws(d, nullptr);
  if (!workspace) { *workspace_bytes = need.total; return QSVD_OK; }
  if (*workspace_bytes < need.total)
    return fail(QSVD_ERR_WORKSPACE, "workspace holds %zu bytes, %zu needed", *workspace_bytes, need.total);
  if (!packed || !cache || !lengths || !out || !status)
    return fail(QSVD_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(workspace) || !aligned16(cache) || !aligned16(out))
    return fail(QSVD_ERR_INVALID_ARG, "workspace, cache and out must be 16-byte aligned");
  const PackedLayout L = packed_layout(d);
  const uint8_t* P = static_cast<const uint8_t*>(packed);
  cudaError_t e = launch_prefill_attention(d, P + L.wuq, P + L.wuk, P + L.wuv,
                                           reinterpret_cast<const float*>(P + L.rope), cache, lengths,
                                           prefill_attention_ws(d, workspace), out, status,
                                           score_scale_log2(d), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prefill_attention");
  return QSVD_OK;
}

// Quantised latent on the tensor cores: the int8 query parts [B][3][H][r]
// take the first three quarters of the 16-bit parts' section ([B][2][H][r]
// 16-bit), their per-(sequence, head) scales [B][H] the rest.
static float* quant_query_scales(const qsvd_dims& d, void* qt16) {
  return reinterpret_cast<float*>(static_cast<uint8_t*>(qt16) + size_t(3) * d.batch * d.H * d.r);
}

static qsvd_status decode_impl(const qsvd_dims& d, const void* packed, const float* qin,
                               int qin_is_latent, const void* cache, const void* scales,
                               const int32_t* lengths, int num_splits, void* workspace,
                               size_t* workspace_bytes, void* out, unsigned phases,
                               cudaStream_t s) {
  if (phases == 0) phases = QSVD_PHASE_ALL;
  constexpr unsigned kSub = QSVD_PHASE_SPLIT_SCORES | QSVD_PHASE_SPLIT_ACCUM;
  if (phases & ~(QSVD_PHASE_ALL | kSub)) return fail(QSVD_ERR_INVALID_ARG, "unknown phase bits");
  const int kernel = pick_kernel(d);
  if ((phases & kSub) && !(d.rope && kernel == QSVD_KERNEL_TCGEN05_CTA))
    return fail(QSVD_ERR_INVALID_ARG, "split sub-phases exist in rotary mode on the tensor cores only");
  if (phases & QSVD_PHASE_SPLIT) phases |= kSub;
  const bool split_any = (phases & kSub) != 0;
  if (kernel == QSVD_KERNEL_TCGEN05_CLUSTER && !split_cl_supported(d))
    return fail(QSVD_ERR_UNSUPPORTED,
                "cluster split kernel needs absorbed mode, a 16-bit cache, r = 128 k or 256 k (2 <= k <= 8), H <= 32");
  if (kernel == QSVD_KERNEL_TCGEN05_CTA && !d.rope && !split_tc_supported(d))
    return fail(QSVD_ERR_UNSUPPORTED,
                "tensor-core split kernel needs a 16-bit or int4/int8 (group 128) cache, r %% 128 == 0, H <= 32");
  if (kernel == QSVD_KERNEL_TCGEN05_CTA && d.rope && !rope_tc_supported(d))
    return fail(QSVD_ERR_UNSUPPORTED,
                "tensor-core rotary path needs d_h == 128, r %% 64 == 0, cache and weights both fp16 or both bf16");
  if (kernel == QSVD_KERNEL_SIMT && !d.rope && split_simt_grid_heads(d) == 0)
    return fail(QSVD_ERR_UNSUPPORTED, "rank too large for the CUDA-core split kernel");
  if ((phases & QSVD_PHASE_COMBINE) && d.out_proj != QSVD_OUT_PROJ_NONE && !combine_uses_gemv(d))
    return fail(QSVD_ERR_UNSUPPORTED,
                "the output projection needs 16-bit weights, d_h %% 64 == 0, r %% 32 == 0 and "
                "at most 2047 tiles per sequence");
  int G = 0;
  qsvd_status st = resolve_splits(d, num_splits, kernel, &G);
  if (st != QSVD_OK) return st;
  const WsLayout W = ws_layout(d, G);
  if (!workspace) { *workspace_bytes = W.total; return QSVD_OK; }
  if (*workspace_bytes < W.total)
    return fail(QSVD_ERR_WORKSPACE, "workspace holds %zu bytes, %zu needed", *workspace_bytes, W.total);
  if (!packed || !lengths) return fail(QSVD_ERR_INVALID_ARG, "packed/lengths is NULL");
  if ((phases & QSVD_PHASE_PROLOGUE) && !qin) return fail(QSVD_ERR_INVALID_ARG, "qin is NULL");
  if (split_any && !cache) return fail(QSVD_ERR_INVALID_ARG, "cache is NULL");
  if (split_any && cache_is_int(d) && !scales)
    return fail(QSVD_ERR_INVALID_ARG, "int caches need scales");
  if ((phases & QSVD_PHASE_COMBINE) && !out) return fail(QSVD_ERR_INVALID_ARG, "out is NULL");
  if (!aligned16(workspace) || (cache && !aligned16(cache)) || (qin && !aligned16(qin)))
    return fail(QSVD_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if ((out && !aligned16(out)) || (scales && !aligned2(scales)))
    return fail(QSVD_ERR_INVALID_ARG, "out must be 16-byte and scales 2-byte aligned");

  const PackedLayout L = packed_layout(d);
  const uint8_t* P = static_cast<const uint8_t*>(packed);
  uint8_t* Wb = static_cast<uint8_t*>(workspace);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(Wb + W.hdr);
  int32_t* sched = reinterpret_cast<int32_t*>(Wb + W.sched);
  float* q = reinterpret_cast<float*>(Wb + W.q);
  float* qt32 = reinterpret_cast<float*>(Wb + W.qt32);
  void* qt16 = Wb + W.qt16;
  float* qpart = reinterpret_cast<float*>(Wb + W.qpart);
  float* pm = reinterpret_cast<float*>(Wb + W.pm);
  float* pl = reinterpret_cast<float*>(Wb + W.pl);
  float* pz = reinterpret_cast<float*>(Wb + W.pz);
  float* opart = reinterpret_cast<float*>(Wb + W.opart);
  const float* rope_tab = reinterpret_cast<const float*>(P + L.rope);
  const float sl2 = score_scale_log2(d);
  cudaError_t e;

  if (phases & QSVD_PHASE_PROLOGUE) {
    int32_t* tickets = reinterpret_cast<int32_t*>(Wb + W.tickets);
    if ((e = launch_schedule(d, lengths, G, sched, hdr, kernel, tickets, W.NT, s)) != cudaSuccess)
      return cuda_fail(e, "schedule");
    // q = c_new W^u_q (reduced into the workspace), or the query as given
    const float* qsrc = qin;
    if (qin_is_latent) {
      if ((e = launch_q_partial(d, qin, P + L.wuq, qpart, W.KS, q, tickets, &hdr->status, s)) != cudaSuccess)
        return cuda_fail(e, "query projection");
      qsrc = q;
    }
    // rotary mode keeps the rotated query in the q section (qt32 is unused there)
    if (d.rope)
      e = launch_rope_query(d, qsrc, sched, rope_tab, sl2, qt32, s);
    else
      // only the copy the split kernel reads: fp32 for CUDA cores, 16-bit hi/lo
      // for tensor cores; a quantised latent on the tensor cores takes the
      // absorbed query as three int8 parts and one scale per (sequence, head),
      // both written into the 16-bit parts' section from the fp32 copy
      if (kernel != QSVD_KERNEL_SIMT && cache_is_int(d)) {
        e = launch_absorb(d, qsrc, P + L.wuk, sl2, qt32, nullptr, &hdr->status, s);
        if (e == cudaSuccess)
          e = launch_quant_query(d, qt32, static_cast<int8_t*>(qt16), quant_query_scales(d, qt16), s);
      } else {
        e = launch_absorb(d, qsrc, P + L.wuk, sl2, kernel == QSVD_KERNEL_SIMT ? qt32 : nullptr,
                          kernel == QSVD_KERNEL_SIMT ? nullptr : qt16, &hdr->status, s);
      }
    if (e != cudaSuccess) return cuda_fail(e, "query prologue");
  }
  if (split_any) {
    if (d.rope && kernel == QSVD_KERNEL_TCGEN05_CTA) {
      float* scores = reinterpret_cast<float*>(Wb + W.scores);
      const int sms = device_sms();
      e = cudaSuccess;
      if (phases & QSVD_PHASE_SPLIT_SCORES)
        e = launch_rope_scores(d, cache, P + L.wukT, qt32, rope_tab, sched, sms > 0 ? sms : 1,
                               scores, &hdr->status, s);
      if (e == cudaSuccess && (phases & QSVD_PHASE_SPLIT_ACCUM))
        e = split_tc_scores_supported(d)
                ? launch_split_tc_scores(d, scores, cache, sched, G, pm, pl, pz, &hdr->status, s)
                : launch_split_simt_scores(d, scores, cache, scales, sched, G, pm, pl, pz, s);
    } else if (d.rope) {
      e = launch_split_simt_rope(d, qt32, P + L.wuk, rope_tab, cache, scales, sched, G, pm, pl, pz, s);
    }
    else if (kernel == QSVD_KERNEL_TCGEN05_CLUSTER)
      e = launch_split_cl(d, cache, qt16, sched, G, pm, pl, pz, &hdr->status, s);
    else if (kernel == QSVD_KERNEL_TCGEN05_CTA)
      e = launch_split_tc(d, cache, scales, qt16, sched, G, pm, pl, pz, &hdr->status, s,
                          quant_query_scales(d, qt16));
    else
      e = launch_split_simt_absorbed(d, qt32, cache, scales, sched, G, pm, pl, pz, s);
    if (e != cudaSuccess) return cuda_fail(e, "split phase");
  }
  if (phases & QSVD_PHASE_COMBINE) {
    if (combine_uses_gemv(d)) {
      float* zm = reinterpret_cast<float*>(Wb + W.zm);
      int32_t* tickets = reinterpret_cast<int32_t*>(Wb + W.tickets) + W.NTQ;
      const OutProj op{P + L.wo, reinterpret_cast<float*>(Wb + W.ow), reinterpret_cast<float*>(Wb + W.ypart),
                       tickets + W.NTV};
      e = launch_combine_gemv(d, hdr, sched, pm, pl, pz, P + L.wuv, zm, opart, tickets, &hdr->status,
                              out, op, s);
    } else {
      e = launch_combine(d, hdr, sched, pm, pl, pz, P + L.wuv, opart, W.JS, W.P, out, s);
    }
    if (e != cudaSuccess)
      return cuda_fail(e, "combine phase");
  }
  return QSVD_OK;
}

qsvd_status qsvd_decode_attn(const qsvd_dims* dims, const void* packed, const float* qin,
                             int qin_is_latent, const void* cache, const void* scales,
                             const int32_t* lengths, int num_splits, void* workspace,
                             size_t* workspace_bytes, void* out, unsigned phases, void* stream) {
  qsvd_status st = validate(dims);
  if (st != QSVD_OK) return st;
  if (!workspace_bytes) return fail(QSVD_ERR_INVALID_ARG, "workspace_bytes is NULL");
  return decode_impl(*dims, packed, qin, qin_is_latent, cache, scales, lengths, num_splits,
                     workspace, workspace_bytes, out, phases, static_cast<cudaStream_t>(stream));
}

qsvd_status qsvd_decode_attn_per_head(const qsvd_dims* dims, const void* bk, const void* bv,
                                      const float* q, const void* ck, const void* cv,
                                      const int32_t* lengths, int layout, void* workspace,
                                      size_t* workspace_bytes, void* out, void* stream) {
  qsvd_status st = validate(dims);
  if (st != QSVD_OK) return st;
  const qsvd_dims& d = *dims;
  if (!workspace_bytes) return fail(QSVD_ERR_INVALID_ARG, "workspace_bytes is NULL");
  if (d.rope && !wsvd_rope_supported(d))
    return fail(QSVD_ERR_UNSUPPORTED,
                "per-head latents, rotary mode: d_h == 128, r in {64, 128}, an F16 or BF16 cache "
                "of the weight type");
  if (d.rope && (long long)d.batch * d.H * d.max_len > 0x7FFFFFFFLL)   // head-major rows: 32-bit coordinates
    return fail(QSVD_ERR_UNSUPPORTED, "per-head latents, rotary mode: batch x H x max_len must be below 2^31");
  if (cache_is_int(d)) return fail(QSVD_ERR_UNSUPPORTED, "per-head latents: F32, F16 or BF16 caches");
  if (d.h2 || d.out_proj == QSVD_OUT_PROJ_CHAIN)
    return fail(QSVD_ERR_UNSUPPORTED, "per-head latents: no online H2, no chained output projection");
  if (d.out_proj == QSVD_OUT_PROJ_FOLD && d.weight_dtype == QSVD_F32)
    return fail(QSVD_ERR_UNSUPPORTED, "per-head latents: the folded output projection needs 16-bit weights");
  if (layout != QSVD_PER_HEAD_HEAD_MAJOR && layout != QSVD_PER_HEAD_TOKEN_MAJOR)
    return fail(QSVD_ERR_INVALID_ARG, "unknown per-head latent layout %d", layout);
  const WsvdLayout W = wsvd_layout(d);
  if ((size_t(W.S) + d.r + 4) * 4 > 227 * 1024)
    return fail(QSVD_ERR_UNSUPPORTED, "max_len too large for the per-head merge");
  if (!workspace) { *workspace_bytes = W.total; return QSVD_OK; }
  if (*workspace_bytes < W.total)
    return fail(QSVD_ERR_WORKSPACE, "workspace holds %zu bytes, %zu needed", *workspace_bytes, W.total);
  if (!bk || !bv || !q || !ck || !cv || !lengths || !out)
    return fail(QSVD_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(workspace) || !aligned16(ck) || !aligned16(cv) || !aligned16(q) || !aligned16(out))
    return fail(QSVD_ERR_INVALID_ARG, "workspace, q, ck, cv and out must be 16-byte aligned");
  cudaError_t e = launch_wsvd_decode(d, bk, bv, q, ck, cv, lengths, score_scale_log2(d), workspace, W, out,
                                     layout == QSVD_PER_HEAD_TOKEN_MAJOR, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode_attn_per_head");
  return QSVD_OK;
}

qsvd_status qsvd_prepare_per_head_fold(const qsvd_dims* dims, const void* bv, const void* wo, void* f,
                                       void* stream) {
  qsvd_status st = validate(dims);
  if (st != QSVD_OK) return st;
  const qsvd_dims& d = *dims;
  if (d.weight_dtype != QSVD_F16 && d.weight_dtype != QSVD_BF16)
    return fail(QSVD_ERR_UNSUPPORTED, "the per-head fold needs 16-bit weights");
  if (!bv || !wo || !f) return fail(QSVD_ERR_INVALID_ARG, "a required pointer is NULL");
  cudaError_t e = launch_per_head_fold(d, bv, wo, f, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prepare_per_head_fold");
  return QSVD_OK;
}

qsvd_status qsvd_combine_splits(const qsvd_dims* dims, const void* packed, void* workspace,
                                int num_splits, const int32_t* lengths, void* out,
                                void* stream) {
  qsvd_status st = validate(dims);
  if (st != QSVD_OK) return st;
  if (!packed || !workspace || !lengths || !out)
    return fail(QSVD_ERR_INVALID_ARG, "a required pointer is NULL");
  size_t cap = ~size_t(0);
  return decode_impl(*dims, packed, nullptr, 1, nullptr, nullptr, lengths, num_splits, workspace,
                     &cap, out, QSVD_PHASE_COMBINE, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
