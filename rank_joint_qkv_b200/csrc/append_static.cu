// Allocation-free variant of qsvd_append_latent.
//
// Some callers cannot hand this library a workspace: a serving engine or
// plugin host that owns every device buffer and exposes only the tensors of
// the call, or a deployment with a fixed device-memory budget that forbids
// any allocation once start-up is over.  This entry point needs nothing but
// the call's inputs and outputs: the split-K partials of x W^d live in one
// file-scope device array that every GPU loading the library keeps until the
// process exits.
#include <cmath>
#include <cstdio>
#include <mutex>

#include "internal.cuh"

namespace qsvd {
namespace {

// Scratch for the split-K partials: KS x batch x r floats.
constexpr size_t kStaticScratchFloats = size_t(1) << 20;   // 4 MiB
static __device__ __align__(256) float g_append_scratch[kStaticScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The first
// call on a device looks it up (host code may not use the symbol itself).
cudaError_t scratch_on_current_device(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_append_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace qsvd

using namespace qsvd;

extern "C" qsvd_status qsvd_append_latent_static(const qsvd_dims* dims, const void* packed,
                                                 const void* x, const int32_t* pos,
                                                 void* cache, void* scales, float* c_out,
                                                 int32_t* status, void* stream) {
  if (!dims) return set_error(QSVD_ERR_INVALID_ARG, "dims is NULL");
  const qsvd_dims& d = *dims;
  // Same host-side checks as the workspace entry point, via its size query.
  size_t ws_need = 0;
  qsvd_status st = qsvd_append_latent(dims, nullptr, nullptr, nullptr, nullptr, nullptr,
                                      nullptr, nullptr, nullptr, &ws_need, nullptr);
  if (st != QSVD_OK) return st;
  const int KS = append_ksplit(d);
  const size_t need = size_t(KS) * d.batch * d.r;
  if (need > kStaticScratchFloats) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "qsvd_append_latent_static: ksplit * batch * r = %zu floats exceeds the %zu-float "
             "static scratch (ksplit = ceil(E/512) for 16-bit weights, ceil(E/64) for float32); "
             "use qsvd_append_latent with a workspace", need, kStaticScratchFloats);
    return set_error(QSVD_ERR_WORKSPACE, msg);
  }
  if (!packed || !x || !pos || !cache)
    return set_error(QSVD_ERR_INVALID_ARG, "a required pointer is NULL");
  // The GEMV reads x with 8- and 16-byte vector loads and the finish kernel
  // stores whole rows: the same alignment the workspace entry point demands.
  if (!aligned16(x) || !aligned16(cache))
    return set_error(QSVD_ERR_INVALID_ARG, "x and cache must be 16-byte aligned");
  if ((scales && (reinterpret_cast<uintptr_t>(scales) & 1u)) || (c_out && (reinterpret_cast<uintptr_t>(c_out) & 3u)))
    return set_error(QSVD_ERR_INVALID_ARG, "scales must be 2-byte and c_out 4-byte aligned");
  if (cache_is_int(d) && !scales) return set_error(QSVD_ERR_INVALID_ARG, "int caches need scales");
  float* scratch = nullptr;
  if (scratch_on_current_device(&scratch) != cudaSuccess)
    return set_error(QSVD_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed");
  const PackedLayout L = packed_layout(d);
  const uint8_t* P = static_cast<const uint8_t*>(packed);
  const float h2_scale = d.h2 ? float(1.0 / std::sqrt(double(d.r / d.h2_m))) : 1.f;
  cudaError_t e = launch_append(d, x, P + L.wd, reinterpret_cast<const float*>(P + L.h2q),
                                h2_scale, pos, cache, scales, c_out, scratch, KS, status,
                                static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return set_error(QSVD_ERR_CUDA, cudaGetErrorString(e));
  return QSVD_OK;
}
