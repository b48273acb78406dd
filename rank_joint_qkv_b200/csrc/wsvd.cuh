// Per-head latent (WSVD) decode: layout of its workspace and its launcher.
#pragma once

#include "internal.cuh"

namespace qsvd {

constexpr int kWsvdChunk = 256;   // tokens per split CTA

// Workspace of qsvd_decode_attn_per_head (256-byte aligned sections):
// header (int32 status), qt [B][H][r] fp32 (absorbed query, log2 domain),
// m, l [B][H][S] fp32, z [B][H][S][r] fp32 with S = ceil(max_len / 256).
struct WsvdLayout {
  size_t hdr, qt, m, l, z, zm, ypart, tickets, rope, scores, total;
  int S, KSY, NT;   // fold: split-K of the GEMV by F and its ticket counters
};

inline WsvdLayout wsvd_layout(const qsvd_dims& d) {
  WsvdLayout w{};
  w.S = (d.max_len + kWsvdChunk - 1) / kWsvdChunk;
  const size_t BH = size_t(d.batch) * d.H;
  size_t o = 0;
  w.hdr = o; o = align256(o + 16);
  w.qt = o;  o = align256(o + BH * size_t(d.r > d.d_h ? d.r : d.d_h) * 4);   // rotary: q' [B][H][d_h]
  w.m = o;   o = align256(o + BH * w.S * 4);
  w.l = o;   o = align256(o + BH * w.S * 4);
  w.z = o;   o = align256(o + BH * w.S * size_t(d.r) * 4);
  // B_{Vh} folded into W_O: merged latents [B][H r], then one GEMV by F
  const bool fold = d.out_proj == QSVD_OUT_PROJ_FOLD;
  w.KSY = fold ? gemv_ksplit(d.H * d.r, d.weight_dtype) : 0;
  w.NT = fold ? gemv_tickets(d.E, d.batch, d.weight_dtype) : 0;
  w.zm = o;  if (fold) o = align256(o + BH * size_t(d.r) * 4);
  w.ypart = o; if (fold) o = align256(o + size_t(w.KSY) * d.batch * d.E * 4);
  w.tickets = o; if (fold) o = align256(o + size_t(w.NT) * 4);
  // rotary mode: the cos/sin table of every position (fp64 angles) and the
  // scores [B][H][max_len] of the keys rebuilt on the tensor cores
  w.rope = o; if (d.rope) o = align256(o + size_t(d.max_len) * d.d_h * 4);
  w.scores = o; if (d.rope) o = align256(o + BH * size_t(d.max_len) * 4);
  w.total = o;
  return w;
}

// Rotary mode (wsvd_rope.cu): the cos/sin table, the rotated query and the
// scores of keys rebuilt on the tensor cores, into the workspace.
bool wsvd_rope_supported(const qsvd_dims& d);
cudaError_t launch_wsvd_rope_front(const qsvd_dims& d, const void* bk, const float* q, const void* ck,
                                   const int32_t* lengths, float sl2, void* workspace, const WsvdLayout& W,
                                   int token_major, cudaStream_t s);
cudaError_t launch_rope_table(float* tab, int max_len, int d_h, float base, cudaStream_t s);

// Three kernels: absorb (qt = sl2 B_{Kh} q_h), split (per 256-token chunk:
// exact chunk softmax, partial m, l, z), combine (merge the chunks,
// o_h = z_h B_{Vh}).
cudaError_t launch_wsvd_decode(const qsvd_dims& d, const void* bk, const void* bv, const float* q,
                               const void* ck, const void* cv, const int32_t* lengths, float sl2,
                               void* workspace, const WsvdLayout& W, void* out, int token_major,
                               cudaStream_t s);

}  // namespace qsvd
