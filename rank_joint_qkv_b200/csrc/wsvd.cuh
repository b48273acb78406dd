// Per-head latent (WSVD) decode: layout of its workspace and its launcher.
#pragma once

#include "internal.cuh"

namespace qsvd {

constexpr int kWsvdChunk = 256;   // tokens per split CTA

// Workspace of qsvd_decode_attn_per_head (256-byte aligned sections):
// header (int32 status), qt [B][H][r] fp32 (absorbed query, log2 domain),
// m, l [B][H][S] fp32, z [B][H][S][r] fp32 with S = ceil(max_len / 256).
struct WsvdLayout {
  size_t hdr, qt, m, l, z, total;
  int S;
};

inline WsvdLayout wsvd_layout(const qsvd_dims& d) {
  WsvdLayout w{};
  w.S = (d.max_len + kWsvdChunk - 1) / kWsvdChunk;
  const size_t BH = size_t(d.batch) * d.H;
  size_t o = 0;
  w.hdr = o; o = align256(o + 16);
  w.qt = o;  o = align256(o + BH * d.r * 4);
  w.m = o;   o = align256(o + BH * w.S * 4);
  w.l = o;   o = align256(o + BH * w.S * 4);
  w.z = o;   o = align256(o + BH * w.S * size_t(d.r) * 4);
  w.total = o;
  return w;
}

// Three kernels: absorb (qt = sl2 B_{Kh} q_h), split (per 256-token chunk:
// exact chunk softmax, partial m, l, z), combine (merge the chunks,
// o_h = z_h B_{Vh}).
cudaError_t launch_wsvd_decode(const qsvd_dims& d, const void* bk, const void* bv, const float* q,
                               const void* ck, const void* cv, const int32_t* lengths, float sl2,
                               void* workspace, const WsvdLayout& W, void* out, int token_major,
                               cudaStream_t s);

}  // namespace qsvd
