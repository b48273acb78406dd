// Split phase on the 5th-generation tensor cores, one CTA per split (a
// persistent CTA walks its split's run of tiles): absorbed query with a
// 16-bit or int4/int8 latent, and the rotary mode's two passes (the scores
// kernel k_rope_scores at the end of this file, then this kernel with the
// scores given).
//
// Per 128-token latent tile of one sequence (QSVD digest, Method, Step 1: keys
// and values are never rebuilt when no rotary embedding is applied; WSVD
// digest, Problem: the shared latent must not be re-read once per head):
//
//   S   = C_tile Qt^T        (128 tokens x H heads, K = r)        tcgen05, TMEM
//   P   = 2^(S - m)          (online softmax, log2 domain)        CUDA cores
//   Z^T += C_tile^T P        (r x H in 128-channel chunks, K=128) tcgen05, TMEM
//
// Every head is served from the same staged tile, so HBM sees the latent
// once per step.  The tile is streamed twice through shared memory in
// 128-channel chunks -- once for S (from HBM, together with the matching
// chunk of the absorbed query Qt) and once for Z (re-read from L2 a fraction
// of a tile later) -- because a whole tile (128 x r x 2 bytes) does not fit in
// shared memory.
//
// The two streams are independent pipelines, each with its own ring of
// shared-memory slots, its own TMA producer warp and its own MMA-issuing
// thread: a single thread issues one tcgen05.mma about every 100 cycles
// whatever the shape, and the small-N MMAs of this kernel finish faster than
// that, so two issuers keep the tensor core twice as busy as one.  Each
// 128-channel chunk of the latent (two 64-channel swizzled boxes) arrives in
// one 3D TMA operation, the matching query chunk (two boxes x hi/lo parts) in
// one 4D operation.
//
// Roles (256 threads):
//   warp 0     S producer: latent chunk + query chunk per slot (ragged last
//              tile of a sequence: latent rows past its length are written as
//              zeros by the warp, so a NaN or Inf stored there cannot leak
//              through P = 0)
//   warp 1     TMEM allocation; one thread issues the S MMAs
//   warp 2     Z producer: latent chunk re-read per slot (same ragged rule)
//   warp 3     one thread issues the Z MMAs
//   warps 4-7  softmax over the S accumulator (one TMEM lane = one token),
//              conditional rescale of Z, P written to shared memory, and the
//              per-segment epilogue (partials m, l, z to global memory)
// Quantised latent (384 threads; 512 with 32 padded heads): S runs on the
// integer tensor cores per 128-channel group (int8 codes straight from the
// cache by TMA on warp 0; int4 codes unpacked to bytes by warps 0 and 9) and
// is scaled per token by the softmax; for Z, warp 2 loads each item's raw
// codes into the end of its fp16 slot and warps 8-11 (int4: 8, 10, 11)
// dequantise them in place.  With 32 padded heads a second group of softmax
// warps (12-15) takes heads 16-31.
// Scores given (rotary mode): no S pass; warps 1 and 3 both issue Z MMAs.
//
// Precision: the absorbed query enters the MMA as hi + lo 16-bit parts and,
// for bf16 latents, P does too (two accumulating MMAs); accumulation is fp32.
//
// Online softmax keeps a per-head reference m; P = 2^(s - m) is written with
// m fixed until some score exceeds m + 8, and only then is m raised and the Z
// accumulator rescaled (exactly: the same m is reported with z and l).
//
// Every wait is bounded (2 s of globaltimer); on expiry the kernel records
// QSVD_STATUS_TIMEOUT in the workspace status word, drains its own work in
// flight (bounded), frees its TMEM and returns.
#include <cuda.h>

#include <cstring>

#include "internal.cuh"
#include "tc_common.cuh"

namespace qsvd {
namespace {

constexpr int kThreadsTc = 256;
constexpr int kThreadsTcQ = 384;   // quantised latent: warps 8-11 convert too
// Softmax groups of four warps: two (the second on warps 12-15, heads split
// in halves) for a quantised latent with 32 padded heads, whose per-group
// score reads dominate the softmax; one otherwise.
template <int NP, int QB>
__host__ __device__ constexpr int softmax_groups() { return (QB && NP == 32) ? 2 : 1; }
template <int NP, int QB>
__host__ __device__ constexpr int split_threads() {
  return QB ? kThreadsTcQ + 128 * (softmax_groups<NP, QB>() - 1) : kThreadsTc;
}
constexpr int kBoxBytes = 128 * 128;            // 128 tokens x 64 channels x 2 bytes
constexpr int kMaxSlots = 8;                   // per ring
constexpr int kMaxGroupBufs = 4;               // S accumulators per channel group (quantised latent)
constexpr int kMaxRaw = 8;                     // raw-code slots per stream (quantised latent)
constexpr int kScaleBufs = 3;                  // group-scale tables of tiles in flight (quantised latent)
constexpr float kRescaleLog2 = 8.f;             // P <= 2^8 before a rescale

// Failure injection for tests (qsvd_testing_set_score_wait_ns): when
// non-zero, the softmax warps start their first tile by waiting on a barrier
// that is never released, giving up after this many nanoseconds -- the
// timeout path runs without any fault.  0: no injection.
__device__ unsigned long long g_score_wait_ns = 0;


// Shared-memory carve.  Both rings carry items of 1/(r/64) of a tile.
//   S slot: one 64-channel box of the latent tile (128 tokens x 128 bytes,
//           swizzled) followed by the matching box of the absorbed query, QS
//           parts of NP rows (QS = 2: the query as a rounded 16-bit part plus
//           its 16-bit rounding residual, summed by the MMA into adjacent
//           accumulator columns), laid out [part][row].
//   Z slot: 64 tokens x 128 channels of the latent tile, two 64-channel
//           boxes of 64 rows ([box][row][128 bytes]).
// Small items keep both rings deep for the shared-memory budget, and the
// split of that budget between the rings follows their share of the bytes.
template <int NP, int QS>
__host__ __device__ constexpr int s_slot_bytes() { return kBoxBytes + QS * NP * 128; }
constexpr int kZBoxBytes = 64 * 128;             // 64 tokens x 64 channels x 2 bytes
constexpr int kZSlotBytes = 2 * kZBoxBytes;
// Quantised latent: an S item is one 128-channel group -- the codes as 8-bit
// integers (128 tokens x 128 bytes, K-major, 128-byte swizzle) and the
// query's three int8 parts (3 x NP rows of 128 bytes, part-major).
template <int NP>
__host__ __device__ constexpr int sq_slot_bytes() { return 128 * 128 + 3 * NP * 128; }
// Scores given (SG): no S pass; ring A carries Z items too.
template <int NP, int QS, bool SG, int QB = 0>
__host__ __device__ constexpr int a_slot_bytes() {
  return SG ? kZSlotBytes : (QB ? sq_slot_bytes<NP>() : s_slot_bytes<NP, QS>());
}
template <int NP>
__host__ __device__ constexpr int pbuf_bytes() { return 2 * NP * 128; }   // one P^T part
constexpr int kMiscBytes = 2048;

struct Smem {
  uint8_t* sring;
  uint8_t* zring;
  uint8_t* pbuf;
  uint64_t* s_full;      // [kMaxSlots] S ring: data landed
  uint64_t* s_empty;     // [kMaxSlots] S ring: MMAs done with the slot
  uint64_t* z_full;      // [kMaxSlots]
  uint64_t* z_empty;     // [kMaxSlots]
  uint64_t* acc_full;    // [2] S accumulator of a tile complete
  uint64_t* p_full;      // [2] P of a tile written (S accumulator read)
  uint64_t* z_done;      // [2] Z MMAs of a tile complete
  uint64_t* drain;       // [2] one per MMA issuer
  uint64_t* sg_full;     // [kMaxGroupBufs] quantised latent: S of one channel group complete
  uint64_t* sg_empty;    // [kMaxGroupBufs] ... read by the softmax
  uint8_t* sraw;         // quantised latent: int4 S raw-code ring
  uint8_t* zsc;          // quantised latent: [kScaleBufs][128 tokens][r / 128] fp16 group scales
  uint64_t* sraw_full;   // [kMaxRaw] int4 S raw codes landed
  uint64_t* zraw_full;   // [kMaxSlots] Z raw codes landed in their fp16 slot
  uint64_t* never;       // never released (failure injection)
  uint64_t* zsc_full;    // [kScaleBufs] scale table of a tile written (by the S producer)
  uint64_t* zsc_empty;   // [kScaleBufs] Z MMAs of the table's tile complete
  float* red;            // [4][NP] per-warp partial max / sum
  float* m_run;          // [NP] running reference max per head (log2 domain)
  float* l_run;          // [NP] running sum of P per head
  float* alpha;          // [NP] rescale factor of the current tile
  float* qsig;           // [NP] quantised latent: the query parts' scale per head of the tile
  uint32_t* tmem_holder;
  volatile int* abort_flag;
};

// P buffers: 2 (double buffer) x PS parts (bf16: hi + lo) x pbuf_bytes.
// Quantised latent: raw codes of one Z item (64 rows x 128 channels) are
// QB x 1024 bytes and land at the end of the item's own fp16 slot; of one S
// item (128 rows x 128 channels) int4 only, 8 KB, in a raw ring (int8 S
// items land by TMA in their slot as they are).  One scale table: 128 tokens
// x r / 128 groups of fp16.
__host__ __device__ constexpr int raw_bytes(int qb) { return qb * 1024; }
__host__ __device__ constexpr int raw_s_bytes(int qb) { return qb == 4 ? 128 * 64 : 0; }
__host__ __device__ constexpr int scale_buf_bytes(int r) { return 256 * (r / 128); }

template <int NP, int QS, int PS, bool SG, int QB>
__device__ Smem carve(uint8_t* base, int ns, int nz, int nraw, int r) {
  Smem s;
  s.sring = base;
  s.zring = s.sring + size_t(ns) * a_slot_bytes<NP, QS, SG, QB>();
  s.pbuf = s.zring + size_t(nz) * kZSlotBytes;
  s.sraw = s.pbuf + 2 * PS * pbuf_bytes<NP>();
  s.zsc = s.sraw + size_t(nraw) * raw_s_bytes(QB);
  uint8_t* m = s.zsc + (QB ? kScaleBufs * scale_buf_bytes(r) : 0);
  uint64_t* bars = reinterpret_cast<uint64_t*>(m);
  s.s_full = bars;
  s.s_empty = bars + kMaxSlots;
  s.z_full = bars + 2 * kMaxSlots;
  s.z_empty = bars + 3 * kMaxSlots;
  s.acc_full = bars + 4 * kMaxSlots;
  s.p_full = s.acc_full + 2;
  s.z_done = s.p_full + 2;
  s.drain = s.z_done + 2;
  s.sg_full = s.drain + 2;
  s.sg_empty = s.sg_full + kMaxGroupBufs;
  s.sraw_full = s.sg_empty + kMaxGroupBufs;
  s.zraw_full = s.sraw_full + kMaxRaw;   // 4 kMaxSlots + 8 + 2 kMaxGroupBufs + kMaxRaw + kMaxSlots = 64
  s.never = s.zraw_full + kMaxSlots;     // the 65th
  s.zsc_full = s.never + 1;
  s.zsc_empty = s.zsc_full + kScaleBufs;  // 65 + 2 kScaleBufs = 71 barriers (the barrier area holds 80)
  static_assert(640 + 4 * NP * 4 + 32 + (QB ? 4 : 3) * NP * 4 <= kMiscBytes, "misc region");
  s.red = reinterpret_cast<float*>(m + 640);
  s.tmem_holder = reinterpret_cast<uint32_t*>(m + 640 + 4 * NP * 4);
  s.abort_flag = reinterpret_cast<volatile int*>(m + 640 + 4 * NP * 4 + 16);
  s.m_run = reinterpret_cast<float*>(m + 640 + 4 * NP * 4 + 32);
  s.l_run = s.m_run + NP;
  s.alpha = s.l_run + NP;
  s.qsig = s.alpha + NP;
  return s;
}

// SG with a channel split over `ch` CTAs: 128-channel chunk j belongs to CTA
// part j % ch, and there to the issuer (and ring) (j / ch) % 2.
__device__ __forceinline__ bool sg_owns(int j, int ch, int cpart, int kind) {
  return j % ch == cpart && ((j / ch) & 1) == kind;
}

__device__ __forceinline__ void set_abort(const Smem& s, int32_t* status) {
  *s.abort_flag = 1;
  atomicOr(status, QSVD_STATUS_TIMEOUT);
}


// Zero-filled copy of latent rows into a slot by one warp, in the
// 128-byte-swizzled layout TMA would have produced: `nbox` 64-channel boxes
// of `rows` rows starting at tile row `row_lo`; tile rows >= nv become zeros.
// `src` is the tile's first row at the first box's channel offset.
__device__ __forceinline__ void ragged_rows(uint8_t* d, const uint8_t* src, size_t row_bytes,
                                            int rows, int nbox, int row_lo, int nv, int lane) {
  const int per_box = rows * 8;   // 16-byte vectors per box
  for (int idx = lane; idx < nbox * per_box; idx += 32) {
    const int box = idx / per_box, tt = (idx >> 3) % rows, c = idx & 7;
    const int t = row_lo + tt;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (t < nv) v = *reinterpret_cast<const uint4*>(src + size_t(t) * row_bytes + box * 128 + c * 16);
    *reinterpret_cast<uint4*>(d + box * rows * 128 + tt * 128 + ((c ^ (tt & 7)) << 4)) = v;
  }
  fence_proxy_async();   // generic-proxy stores -> visible to the tensor core
  __syncwarp();
}

// ------------------------------------------------- quantised latent rows
// Symmetric int4 (two's complement nibbles, channel 2j in the low nibble of
// byte j) and int8 codes, turned into exact fp16 integers by offset binary:
// (code + 2^(b-1)) in the mantissa of 1024.0, minus (1024 + 2^(b-1)).

// Eight int4 codes (one 32-bit word) -> four half2 as 32-bit words, channels
// in order (o0 = c0 c1, o1 = c2 c3, o2 = c4 c5, o3 = c6 c7).  Nibbles 0 and 4,
// 1 and 5 (then 2 and 6, 3 and 7 after a byte shift) land in the mantissas of
// a half2 of 1024.0 each (the odd ones 16x too high, scaled back by an exact
// fma); byte permutes restore channel order.
__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
__device__ __forceinline__ void int4x8_to_half(uint32_t w, __half2 s2, uint32_t& o0, uint32_t& o1,
                                               uint32_t& o2, uint32_t& o3) {
  const uint32_t x = w ^ 0x88888888u;   // offset binary: code + 8 in 0..15
  const __half2 b1032 = u2h(0x64086408u), s16 = u2h(0x2C002C00u), b72 = u2h(0xD480D480u);   // 1032, 1/16, -72
  __half2 ha = __hsub2(u2h((x & 0x000F000Fu) | 0x64006400u), b1032);          // c0, c4
  __half2 hb = __hfma2(u2h((x & 0x00F000F0u) | 0x64006400u), s16, b72);       // c1, c5
  __half2 hc = __hsub2(u2h(((x >> 8) & 0x000F000Fu) | 0x64006400u), b1032);   // c2, c6
  __half2 hd = __hfma2(u2h(((x >> 8) & 0x00F000F0u) | 0x64006400u), s16, b72); // c3, c7
  ha = __hmul2(ha, s2);   // times the group scale: one rounding of the exact product
  hb = __hmul2(hb, s2);
  hc = __hmul2(hc, s2);
  hd = __hmul2(hd, s2);
  const uint32_t ua = h2u(ha), ub = h2u(hb), uc = h2u(hc), ud = h2u(hd);
  o0 = __byte_perm(ua, ub, 0x5410);
  o1 = __byte_perm(uc, ud, 0x5410);
  o2 = __byte_perm(ua, ub, 0x7632);
  o3 = __byte_perm(uc, ud, 0x7632);
}
// Four int8 codes (one 32-bit word) -> two half2 words: each byte (offset
// binary) placed under an 0x64 high byte, minus 1024 + 128.
__device__ __forceinline__ void int8x4_to_half(uint32_t w, __half2 s2, uint32_t& o0, uint32_t& o1) {
  const uint32_t x = w ^ 0x80808080u;
  const __half2 bias = u2h(0x64806480u);   // 1152
  __half2 lo = __hsub2(u2h(__byte_perm(x, 0x64646464u, 0x5140)), bias);
  __half2 hi = __hsub2(u2h(__byte_perm(x, 0x64646464u, 0x5342)), bias);
  lo = __hmul2(lo, s2);
  hi = __hmul2(hi, s2);
  o0 = h2u(lo);
  o1 = h2u(hi);
}
// One 16-byte vector of codes -> QB == 4: 32 channels (four 16-byte fp16
// chunks), QB == 8: 16 channels (two chunks), each times the group scale s2
// (one fp16 rounding of the exact product).
template <int QB>
__device__ __forceinline__ void codes_to_half(const uint4& v, __half2 s2, uint4 (&out)[QB == 4 ? 4 : 2]) {
  if (QB == 4) {
    int4x8_to_half(v.x, s2, out[0].x, out[0].y, out[0].z, out[0].w);
    int4x8_to_half(v.y, s2, out[1].x, out[1].y, out[1].z, out[1].w);
    int4x8_to_half(v.z, s2, out[2].x, out[2].y, out[2].z, out[2].w);
    int4x8_to_half(v.w, s2, out[3].x, out[3].y, out[3].z, out[3].w);
  } else {
    int8x4_to_half(v.x, s2, out[0].x, out[0].y);
    int8x4_to_half(v.y, s2, out[0].z, out[0].w);
    int8x4_to_half(v.z, s2, out[1].x, out[1].y);
    int8x4_to_half(v.w, s2, out[1].z, out[1].w);
  }
}

// Explicit shared-space 16-byte accesses (a generic pointer into shared
// memory would be split into narrower generic stores).
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t a, const uint4& v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ __half lds16h(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return __ushort_as_half(v);
}

// Z item of a quantised tile, expanded in place: its raw codes ([64 rows]
// [QB x 16 bytes], at the end of the fp16 slot) become channels 128 j ..
// 128 j + 127 of rows 64 h .. 64 h + 63, dequantised (code x group scale,
// one fp16 rounding of the exact product), two 64-channel boxes of 64 rows,
// 128-byte swizzled.  sct: the tile's scale table [128][ngroups] (zeros for
// rows past the length, which therefore come out as zeros).  Warp-wide, in
// two phases of 32 rows: a phase reads its raw rows into registers before
// its first store, and its stores overwrite only raw rows of this phase or
// the one before (int8: output row x of the second box is raw row x; int4:
// the second box's rows 32-63 are the raw rows).
template <int QB>
__device__ __forceinline__ void convert_z_inplace(uint32_t d, uint32_t sct, int ngroups, int j, int h, int lane) {
  constexpr int RPB = QB * 16;            // raw bytes per row: 64 (int4), 128 (int8)
  constexpr int VPR = RPB / 16;
  constexpr int CPV = QB == 4 ? 4 : 2;
  constexpr int NV = 32 * VPR / 32;       // vectors per lane per phase: 4 (int4), 8 (int8)
  const uint32_t raw = d + uint32_t(kZSlotBytes - 64 * RPB);
#pragma unroll 1
  for (int ph = 0; ph < 2; ++ph) {
    uint4 rv[NV];
    __half sc[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int v = lane + 32 * i, tt = 32 * ph + v / VPR, q = v % VPR;
      rv[i] = lds128(raw + tt * RPB + q * 16);
      sc[i] = lds16h(sct + uint32_t(((64 * h + tt) * ngroups + j) * 2));
    }
    asm volatile("bar.warp.sync 0xffffffff;" ::: "memory");   // the phase's loads before its stores
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int v = lane + 32 * i, tt = 32 * ph + v / VPR, q = v % VPR;
      uint4 out[CPV];
      codes_to_half<QB>(rv[i], __halves2half2(sc[i], sc[i]), out);
      const int ch = q * (CPV * 8);         // first channel of the vector within the 128
      const int box = ch >> 6, c0 = (ch & 63) >> 3;
#pragma unroll
      for (int c = 0; c < CPV; ++c) sts128(d + box * kZBoxBytes + tt * 128 + (((c0 + c) ^ (tt & 7)) << 4), out[c]);
    }
    asm volatile("bar.warp.sync 0xffffffff;" ::: "memory");   // the phase's stores before the next's loads
  }
  fence_proxy_async();   // generic-proxy stores -> visible to the tensor core
  __syncwarp();
}

// Scale table of one tile (quantised latent), written by the S producer when
// it starts the tile: the tile's group scales [128][r / 128] (rows past the
// length as zeros, which the Z items then dequantise to zeros), read by the
// softmax (S) and the converting warps (Z).  A table is reused once the Z
// MMAs of its tile are complete.  Warp-wide; false if the wait expired.
__device__ bool write_scale_table(const Smem& s, const __half* scales, int row, int nv, int r, Ring& sb, int lane) {
  const int NG = r / 128;
  if (!__all_sync(0xffffffffu, mbar_wait(saddr(&s.zsc_empty[sb.slot]), sb.phase ^ 1u))) return false;
  const __half* tsc = scales + size_t(row) * NG;
  __half* tab = reinterpret_cast<__half*>(s.zsc + sb.slot * scale_buf_bytes(r));
  for (int e = lane; e < 128 * NG; e += 32) tab[e] = e < nv * NG ? tsc[e] : __float2half(0.f);
  mbar_arrive(saddr(&s.zsc_full[sb.slot]));   // every lane (count 32), releasing its own stores
  sb.advance();
  return true;
}

// Z stream of a quantised latent, issuing warp: per item, a free fp16 slot,
// then the item's raw codes by TMA into the slot's end, where a converting
// warp expands them in place.  *issued: items issued.
template <int QB>
__device__ bool produce_zq(const Smem& s, const CUtensorMap* tm_raw, const int32_t* sched, int B, int r,
                           int max_len, long long tb, long long te, int n, int nz, int lane, long long* issued) {
  const int NI = r / 64;
  constexpr uint32_t RB = uint32_t(raw_bytes(QB));
  const uint32_t ring0 = saddr(s.zring);
  TileIter it;
  it.init(sched, B, tb, te);
  Ring rg(nz);
  long long k = 0;
  for (int i = 0; i < n; ++i) {
    const int row = it.b * max_len + it.t0();
    for (int u = 0; u < NI; ++u) {
      if (!__all_sync(0xffffffffu, mbar_wait(saddr(&s.z_empty[rg.slot]), rg.phase ^ 1u))) { *issued = k; return false; }
      const uint32_t fb = saddr(&s.zraw_full[rg.slot]);
      if (lane == int(k & 31)) {   // rotating issuing lane
        mbar_expect_tx(fb, RB);
        tma_load_2d(ring0 + uint32_t(rg.slot) * kZSlotBytes + (kZSlotBytes - RB), tm_raw, (u >> 1) * (QB * 16),
                    row + 64 * (u & 1), fb);
      }
      __syncwarp();
      rg.advance();
      ++k;
    }
    it.next();
    if (__any_sync(0xffffffffu, *s.abort_flag)) { *issued = k; return false; }
  }
  *issued = k;
  return true;
}

// Z stream of a quantised latent, converting warps: warp wsub of nsub takes
// the items k == wsub (mod nsub), waits for the tile's scale table (once per
// tile) and the item's raw codes, expands the item in place and hands the
// slot to the Z MMAs.  Issues no copies (nothing to drain after an abort).
template <int QB>
__device__ bool convert_zq(int wsub, int nsub, const Smem& s, int r, int n, int nz, int lane) {
  const int NI = r / 64, NG = r / 128;
  const uint32_t ring0 = saddr(s.zring), sct0 = saddr(s.zsc);
  Ring rg(nz), sb(kScaleBufs);
  int k_sub = 0;
  for (int i = 0; i < n; ++i) {
    bool have = false;
    for (int u = 0; u < NI; ++u) {
      if (k_sub == wsub) {
        if (!have && !__all_sync(0xffffffffu, mbar_wait(saddr(&s.zsc_full[sb.slot]), sb.phase))) return false;
        have = true;
        if (!__all_sync(0xffffffffu, mbar_wait(saddr(&s.zraw_full[rg.slot]), rg.phase))) return false;
        convert_z_inplace<QB>(ring0 + uint32_t(rg.slot) * kZSlotBytes, sct0 + uint32_t(sb.slot * scale_buf_bytes(r)),
                              NG, u >> 1, u & 1, lane);
        if (lane == 0) mbar_arrive(saddr(&s.z_full[rg.slot]));
      }
      if (++k_sub == nsub) k_sub = 0;
      rg.advance();
    }
    sb.advance();
    if (__any_sync(0xffffffffu, *s.abort_flag)) return false;
  }
  return true;
}

// ------------------------------------------- quantised latent, S stream
// The scores pass of a quantised latent runs on the integer tensor cores:
// per 128-channel group g, S_g = C_g Qp_g^T with C_g the codes (int8 as
// stored; int4 unpacked to sign-extended bytes) and Qp_g the absorbed
// query's three int8 parts (rows k NP + h), int32 exact; the softmax warps
// then form s = sigma_h sum_g scale_{t,g} (S_0 + S_1 / 128 + S_2 / 16384)
// with sigma_h the query parts' scale of the head (see k_quant_query).

// Eight int4 codes (one word) -> eight signed bytes in channel order.
__device__ __forceinline__ void unpack_int4x8(uint32_t w, uint32_t& a, uint32_t& b) {
  uint32_t lo = w & 0x0F0F0F0Fu;                 // channels 0, 2, 4, 6 (two's-complement nibbles)
  uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;          // channels 1, 3, 5, 7
  lo |= (lo & 0x08080808u) * 0x1Eu;              // sign-extend each nibble to its byte (0x08 * 0x1E = 0xF0)
  hi |= (hi & 0x08080808u) * 0x1Eu;
  a = __byte_perm(lo, hi, 0x5140);               // channels 0 1 2 3
  b = __byte_perm(lo, hi, 0x7362);               // channels 4 5 6 7
}

// One S item of int4 codes (raw [128 rows][64 bytes]) -> the A operand: 128
// rows of 128 signed bytes, K-major, 128-byte swizzled.  Warp-wide;
// every raw vector of a half is requested before the first store.
__device__ __forceinline__ void unpack_s_group(uint32_t d, uint32_t raw, int lane) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint4 rv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) rv[i] = lds128(raw + uint32_t(lane + 32 * (8 * half + i)) * 16);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int v = lane + 32 * (8 * half + i), t = v >> 2, c0 = 2 * (v & 3);   // row, first 16-byte chunk
      uint32_t o[8];
      unpack_int4x8(rv[i].x, o[0], o[1]);
      unpack_int4x8(rv[i].y, o[2], o[3]);
      unpack_int4x8(rv[i].z, o[4], o[5]);
      unpack_int4x8(rv[i].w, o[6], o[7]);
      sts128(d + t * 128 + ((c0 ^ (t & 7)) << 4), make_uint4(o[0], o[1], o[2], o[3]));
      sts128(d + t * 128 + (((c0 + 1) ^ (t & 7)) << 4), make_uint4(o[4], o[5], o[6], o[7]));
    }
  }
  fence_proxy_async();   // generic-proxy stores -> visible to the tensor core
  __syncwarp();
}

// S stream, int8 codes: one warp; per item the codes (TMA, 128-byte swizzle,
// straight from the cache) and the query parts (TMA) into one slot.  Rows of
// a ragged last tile past the length are read as stored (finite integers;
// the softmax masks them).  *issued: items issued.
template <int NP>
__device__ bool produce_qs8(const Smem& s, const CUtensorMap* tm_a, const CUtensorMap* tm_q, const __half* scales,
                            const int32_t* sched, int B, int r, int max_len, long long tb, long long te, int n,
                            int nslots, int lane, long long* issued) {
  const int NG = r / 128;
  constexpr uint32_t SQ = uint32_t(sq_slot_bytes<NP>());
  const uint32_t ring0 = saddr(s.sring);
  TileIter it;
  it.init(sched, B, tb, te);
  Ring rg(nslots), sb(kScaleBufs);
  long long k = 0;
  for (int i = 0; i < n; ++i) {
    const int row = it.b * max_len + it.t0(), b = it.b;
    if (!write_scale_table(s, scales, row, it.nvalid(), r, sb, lane)) { *issued = k; return false; }
    for (int u = 0; u < NG; ++u) {
      if (!__all_sync(0xffffffffu, mbar_wait(saddr(&s.s_empty[rg.slot]), rg.phase ^ 1u))) { *issued = k; return false; }
      const uint32_t dst = ring0 + uint32_t(rg.slot) * SQ, fb = saddr(&s.s_full[rg.slot]);
      const int ln = int(k & 15) * 2;   // rotating issuing lanes (see produce)
      if (lane == 0) mbar_expect_tx(fb, SQ);
      __syncwarp();
      if (lane == ln) tma_load_2d(dst, tm_a, 128 * u, row, fb);
      if (lane == ln + 1) tma_load_3d(dst + 128 * 128, tm_q, 128 * u, 0, 3 * b, fb);
      __syncwarp();
      rg.advance();
      ++k;
    }
    it.next();
    if (__any_sync(0xffffffffu, *s.abort_flag)) { *issued = k; return false; }
  }
  *issued = k;
  return true;
}

// S stream, int4 codes: nsub warps share the items (item k to warp k % nsub);
// raw codes by TMA into a ring of nraw slots (a multiple of nsub, so a slot is
// always refilled by the warp that drained it) issued nraw items ahead,
// unpacked into the slot; the query parts by TMA.  The slot completes on the
// query's bytes and the warp's arrive.
template <int NP>
__device__ bool produce_qs4(int wsub, int nsub, const Smem& s, const CUtensorMap* tm_raw, const CUtensorMap* tm_q,
                            const __half* scales, const int32_t* sched, int B, int r, int max_len, long long tb,
                            long long te, int n, int nslots, int nraw, int lane, long long* last_item,
                            long long* last_raw) {
  const int NG = r / 128;
  constexpr uint32_t SQ = uint32_t(sq_slot_bytes<NP>());
  constexpr uint32_t RB = uint32_t(raw_s_bytes(4));
  const uint32_t ring0 = saddr(s.sring), raw0 = saddr(s.sraw);
  const int total = n * NG;
  *last_item = -1;
  *last_raw = -1;
  TileIter ia;
  ia.init(sched, B, tb, te);
  int ia_i = 0, ua = 0, ki = 0, ki_sub = 0, own = 0;
  Ring ri(nraw);
  auto issue_next = [&]() {
    if (ki_sub == wsub) {
      const uint32_t fb = saddr(&s.sraw_full[ri.slot]);
      const int row = ia.b * max_len + ia.t0();
      if (lane == (own & 31)) {   // rotating issuing lane
        mbar_expect_tx(fb, RB);
        tma_load_2d(raw0 + ri.slot * RB, tm_raw, ua * 64, row, fb);
      }
      ++own;
      *last_raw = ki;
    }
    ++ki;
    if (++ki_sub == nsub) ki_sub = 0;
    ri.advance();
    if (++ua == NG) {
      ua = 0;
      if (++ia_i < n) ia.next();
    }
  };
  for (int x = 0; x < total && x < nraw; ++x) issue_next();
  TileIter it;
  it.init(sched, B, tb, te);
  int k = 0, k_sub = 0;
  Ring rr(nraw), rs(nslots), sb(kScaleBufs);
  for (int i = 0; i < n; ++i) {
    const int b = it.b;
    if (wsub == 0 && !write_scale_table(s, scales, b * max_len + it.t0(), it.nvalid(), r, sb, lane)) return false;
    for (int u = 0; u < NG; ++u) {
      if (k_sub == wsub) {
        if (!__all_sync(0xffffffffu, mbar_wait(saddr(&s.sraw_full[rr.slot]), rr.phase)) ||
            !__all_sync(0xffffffffu, mbar_wait(saddr(&s.s_empty[rs.slot]), rs.phase ^ 1u)))
          return false;   // warp-uniform
        const uint32_t dst = ring0 + uint32_t(rs.slot) * SQ, fb = saddr(&s.s_full[rs.slot]);
        if (lane == 0) {
          mbar_expect_tx(fb, uint32_t(3 * NP * 128));
          tma_load_3d(dst + 128 * 128, tm_q, 128 * u, 0, 3 * b, fb);
        }
        unpack_s_group(dst, raw0 + uint32_t(rr.slot) * RB, lane);
        if (lane == 0) mbar_arrive(fb);
        *last_item = k;
        for (int x = 0; x < nsub && ki < total; ++x) issue_next();
        __syncwarp();
      }
      ++k;
      if (++k_sub == nsub) k_sub = 0;
      rr.advance();
      rs.advance();
    }
    it.next();
    if (__any_sync(0xffffffffu, *s.abort_flag)) return false;
  }
  return true;
}

// After an abort (int4 S unpacking warps): wait (bounded) for the copies
// this warp may have in flight -- the last raw load into each of its raw
// slots, the query boxes of its last S items -- so that none lands after the
// CTA has left.
__device__ void drain_q(int wsub, int nsub, const Smem& s, int nslots, int nraw, long long last_item,
                        long long last_raw) {
  for (int slot = wsub; slot < nraw; slot += nsub) {
    if (last_raw < slot) continue;
    const long long kk = slot + (last_raw - slot) / nraw * nraw;   // last item issued into the slot
    mbar_wait(saddr(&s.sraw_full[slot]), uint32_t(kk / nraw) & 1u);
  }
  for (long long kk = last_item; kk >= 0 && kk > last_item - nslots; kk -= nsub)
    mbar_wait(saddr(&s.s_full[int(kk % nslots)]), uint32_t(kk / nslots) & 1u);
}

// Producer of one ring (warp-wide).  kind 0: S ring (latent box from HBM,
// kept in L2 for the Z re-read, plus the query box); kind 1: Z ring (latent
// re-read, dropped from L2 after).  Item u of a tile: S -> channel box u;
// Z -> channels [128 (u / 2), +128) x tokens [64 (u % 2), +64).  SG (scores
// given): both rings carry Z items, ring `kind` the chunks sg_owns gives it,
// read once (dropped from L2 after).  Returns false on a wait that expired
// or an abort.
template <int NP, int QS, bool SG>
__device__ bool produce(int kind, const Smem& s, const CUtensorMap* tm_cs, const CUtensorMap* tm_cz,
                        const CUtensorMap* tm_q, const uint8_t* cache, const int32_t* sched, int B,
                        int r, int max_len, long long tb, long long te, int n, int nslots, int lane,
                        long long* issued, int ch, int cpart) {
  const int NI = r / 64;
  const size_t row_bytes = size_t(r) * 2;
  const bool zk = SG || kind == 1;   // this ring carries Z items
  uint8_t* ring = kind == 0 ? s.sring : s.zring;
  const uint32_t slot_bytes = zk ? uint32_t(kZSlotBytes) : uint32_t(s_slot_bytes<NP, QS>());
  uint64_t* full = kind == 0 ? s.s_full : s.z_full;
  uint64_t* empty = kind == 0 ? s.s_empty : s.z_empty;
  const uint64_t policy = zk ? policy_evict_first() : policy_evict_last();
  const uint32_t ring0 = saddr(ring);
  TileIter it;
  it.init(sched, B, tb, te);
  Ring rg(nslots);
  long long k = 0;
  for (int i = 0; i < n; ++i) {
    const int nv = it.nvalid(), b = it.b, t0 = it.t0();
    const int row = b * max_len + t0;
    const uint8_t* tile = cache + size_t(row) * row_bytes;
    for (int u = 0; u < NI; ++u) {
      if (SG && !sg_owns(u >> 1, ch, cpart, kind)) continue;   // another ring's (or CTA's) chunk
      if (!__all_sync(0xffffffffu, mbar_wait(saddr(&empty[rg.slot]), rg.phase ^ 1u))) {   // warp-uniform
        *issued = k;
        return false;
      }
      const uint32_t dst = ring0 + uint32_t(rg.slot) * slot_bytes;
      const uint32_t fb = saddr(&full[rg.slot]);
      const int lo = zk ? 64 * (u & 1) : 0;               // first tile row of the item
      const int hi = zk ? lo + 64 : kTile;
      if (nv >= hi) {
        if (lane == 0) mbar_expect_tx(fb, slot_bytes);
        __syncwarp();
        // TMA operations of one thread are processed one after another, so the
        // issuing lanes rotate between items and the item's two operations
        // go out from different lanes
        const int ln = int(k & 15) * 2;
        if (!zk) {
          if (lane == ln) tma_load_2d_hint(dst, tm_cs, 64 * u, row, fb, policy);
          if (lane == ln + 1) tma_load_4d(dst + kBoxBytes, tm_q, 0, 0, QS * b, u, fb);
        } else if (lane == ln) {
          tma_load_3d_hint(dst, tm_cz, 0, row + lo, 2 * (u >> 1), fb, policy);
        }
      } else {
        // last tile of a sequence: rows past its length are written as zeros
        uint8_t* d = ring + size_t(rg.slot) * slot_bytes;
        if (!zk) ragged_rows(d, tile + 128 * u, row_bytes, kTile, 1, 0, nv, lane);
        else ragged_rows(d, tile + 256 * (u >> 1), row_bytes, 64, 2, lo, nv, lane);
        if (lane == 0) {
          if (!zk) {
            mbar_expect_tx(fb, uint32_t(QS * NP * 128));
            tma_load_4d(dst + kBoxBytes, tm_q, 0, 0, QS * b, u, fb);
          } else {
            mbar_arrive(fb);
          }
        }
      }
      __syncwarp();
      rg.advance();
      ++k;
    }
    it.next();
    if (__any_sync(0xffffffffu, *s.abort_flag)) { *issued = k; return false; }
  }
  *issued = k;
  return true;
}

// Wait (bounded) until the last `min(k, nslots)` loads of a ring have landed,
// so that no copy is in flight when the CTA exits.
__device__ void drain_ring(uint64_t* full, long long k, int nslots) {
  for (long long kk = (k > nslots ? k - nslots : 0); kk < k; ++kk)
    mbar_wait(saddr(&full[int(kk % nslots)]), uint32_t(kk / nslots) & 1u);
}

// ------------------------------------------------------------------ kernel

// QB = 0: 16-bit latent; QB = 4 / 8: int4 / int8 codes with fp16 scales per
// group of 128 channels (S per group into a ring of nsg TMEM buffers, the
// scales applied per token by the softmax; Z from the dequantised latent).
// SG: scores given ([B][H][max_len] fp32, log2 domain: the rotary mode's
// scores kernel), no S pass; warps 1 and 3 both issue Z MMAs, each for
// alternate 128-channel chunks, fed by its own ring.  When the Z accumulator
// of all chunks does not fit TMEM, `ch` CTAs share one tile range (split g =
// blockIdx.x / ch), each owning every ch-th chunk; all of them run the same
// softmax on the same scores and part 0 writes m and l.
template <int NP, bool BF16, int QS, int PS, int QB, bool SG>
__global__ void __launch_bounds__(split_threads<NP, QB>(), 1)
k_split_tc(const __grid_constant__ CUtensorMap tm_cs, const __grid_constant__ CUtensorMap tm_cz,
           const __grid_constant__ CUtensorMap tm_q,
           const uint8_t* __restrict__ cache, const __half* __restrict__ scales,
           const float* __restrict__ scores, const int32_t* __restrict__ sched,
           float* __restrict__ pm, float* __restrict__ pl, float* __restrict__ pz,
           int32_t* __restrict__ status, int B, int H, int r, int max_len, int G, int ns, int nz,
           int nsg, int nraw, int ch, const float* __restrict__ qsh) {
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  static_assert(!(SG && QB), "scores given: 16-bit latent only");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const Smem s = carve<NP, QS, PS, SG, QB>(base, ns, nz, nraw, r);
  // S accumulator columns per buffer: hi and lo query parts (16-bit), or the
  // three int8 query parts' int32 sums of one group (quantised)
  constexpr int SW = QB ? 3 * NP : QS * NP;
  constexpr int WG = softmax_groups<NP, QB>(), HW = NP / WG;   // softmax groups, heads per group
  const int ZC0 = SG ? 0 : (QB ? nsg : 2) * SW;   // first Z column
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NI = r / 64;                      // ring items per tile
  const int NC = r / 128;                     // 128-channel Z accumulator chunks
  const int g = SG ? int(blockIdx.x) / ch : int(blockIdx.x);       // split
  const int cpart = SG ? int(blockIdx.x) % ch : 0;                 // channel part
  const int NCL = SG ? (NC - cpart + ch - 1) / ch : NC;            // chunks held in TMEM
  const long long T = sched[B];
  const long long tb = dev::split_begin(g, G, T);
  const long long te = dev::split_begin(g + 1, G, T);
  if (tb >= te) return;   // uniform across the CTA, before any barrier or TMEM use
  const int n = int(te - tb);

  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(saddr(&s.s_full[i]), QB == 4 ? 2 : 1);   // int4: query TMA + unpacked codes
      mbar_init(saddr(&s.s_empty[i]), 1);
    }
    for (int i = 0; i < kMaxGroupBufs; ++i) {
      mbar_init(saddr(&s.sg_full[i]), 1);
      mbar_init(saddr(&s.sg_empty[i]), 4 * WG);   // one arrive per softmax warp
    }
    for (int i = 0; i < kMaxRaw; ++i) mbar_init(saddr(&s.sraw_full[i]), 1);
    for (int i = 0; i < kMaxSlots; ++i) mbar_init(saddr(&s.zraw_full[i]), 1);
    mbar_init(saddr(s.never), 1);
    for (int i = 0; i < kScaleBufs; ++i) {
      mbar_init(saddr(&s.zsc_full[i]), 32);   // the issuing warp's lanes
      mbar_init(saddr(&s.zsc_empty[i]), 1);
    }
    for (int i = 0; i < nz; ++i) {
      mbar_init(saddr(&s.z_full[i]), 1);
      mbar_init(saddr(&s.z_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(saddr(&s.acc_full[i]), 1);
      mbar_init(saddr(&s.p_full[i]), WG);   // one arrive per softmax group
      mbar_init(saddr(&s.z_done[i]), SG ? 2 : 1);   // SG: one commit per Z issuer
      mbar_init(saddr(&s.drain[i]), 1);
    }
    *s.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     saddr(s.tmem_holder))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s.tmem_holder;

  if (warp == 0 || warp == 2 || (QB && warp >= 8 && warp < 12)) {
    // ----------------------------------------------------------- producers
    bool ok = true;
    long long issued = 0, raw_issued = 0;
    if constexpr (QB != 0) {
      // quantised latent.  S: warp 0 loads int8 codes by TMA; int4 raw codes
      // are unpacked by warps 0 and 9.  Z: warp 2 issues the raw codes and
      // the tiles' scale tables, warps 8-11 (int4: 8, 10, 11) expand them
      // (warp w issues on scheduler w % 4)
      const bool zconv = warp >= 8 && !(QB == 4 && warp == 9);
      if (warp == 2) {
        ok = produce_zq<QB>(s, &tm_cz, sched, B, r, max_len, tb, te, n, nz, lane, &issued);
        if (!ok && lane == 0) {
          set_abort(s, status);
          drain_ring(s.zraw_full, issued, nz);
        }
      } else if (zconv) {
        const int wsub = QB == 8 ? warp - 8 : (warp == 8 ? 0 : warp - 9);
        ok = convert_zq<QB>(wsub, QB == 8 ? 4 : 3, s, r, n, nz, lane);
        if (!ok && lane == 0) set_abort(s, status);
      } else if (QB == 4) {   // warps 0 and 9
        const int wsub = warp == 0 ? 0 : 1;
        ok = produce_qs4<NP>(wsub, 2, s, &tm_cs, &tm_q, scales, sched, B, r, max_len, tb, te, n, ns, nraw, lane,
                             &issued, &raw_issued);
        if (!ok && lane == 0) {
          set_abort(s, status);
          drain_q(wsub, 2, s, ns, nraw, issued, raw_issued);
        }
      } else {   // int8, warp 0: no conversion
        ok = produce_qs8<NP>(s, &tm_cs, &tm_q, scales, sched, B, r, max_len, tb, te, n, ns, lane, &issued);
        if (!ok && lane == 0) {
          set_abort(s, status);
          drain_ring(s.s_full, issued, ns);
        }
      }
    } else {
      const int kind = warp == 0 ? 0 : 1;
      const int nslots = kind == 0 ? ns : nz;
      ok = produce<NP, QS, SG>(kind, s, &tm_cs, &tm_cz, &tm_q, cache, sched, B, r, max_len, tb, te,
                               n, nslots, lane, &issued, ch, cpart);
      if (!ok && lane == 0) {
        set_abort(s, status);
        drain_ring(kind == 0 ? s.s_full : s.z_full, issued, nslots);
      }
    }
    (void)raw_issued;
    __syncwarp();
  } else if (warp == 1 && !SG) {
    // ----------------------------------------------------------- S MMAs
    if (QB && lane == 0) {
      // quantised latent: one S item per 128-channel group, integer MMAs
      // (M 128 tokens, N 3 NP query-part rows, K 32 bytes) accumulated onto
      // a ring of nsg int32 group buffers that the softmax reads and refills
      // with the bias 0x4B400000 (the bits of 1.5 x 2^23): a finished buffer
      // holds the float 1.5 x 2^23 + S exactly (|S| < 2^22)
      constexpr uint32_t id_q = idesc_i8(128, SW, true);   // signed codes x signed query parts
      const uint64_t da0 = sdesc(saddr(s.sring), 16, 1024);   // K-major, 128B swizzle
      constexpr int SQ = sq_slot_bytes<NP>();
      Ring rg(ns);
      Ring gr(nsg);
      bool ok = true;
      for (int i = 0; i < n && ok; ++i) {
        for (int u = 0; u < NC; ++u) {
          // the buffer is released (first: initialised) biased by the softmax
          if (!mbar_wait(saddr(&s.sg_empty[gr.slot]), gr.phase)) { ok = false; break; }
          if (!mbar_wait(saddr(&s.s_full[rg.slot]), rg.phase)) { ok = false; break; }
          tc_fence_after();
          const uint64_t sa = da0 + uint64_t((rg.slot * SQ) >> 4);
          const uint32_t d = tmem + uint32_t(gr.slot * SW);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)   // K = 32 channels (bytes) per MMA
            tc_mma_i8(d, sa + uint64_t((kk * 32) >> 4), sa + uint64_t((128 * 128 + kk * 32) >> 4), id_q, 1u);
          tc_commit(saddr(&s.s_empty[rg.slot]));
          rg.advance();
          tc_commit(saddr(&s.sg_full[gr.slot]));
          gr.advance();
        }
        if (*s.abort_flag) ok = false;
      }
      if (!ok) set_abort(s, status);
      tc_commit(saddr(&s.drain[0]));
      mbar_wait(saddr(&s.drain[0]), 0);
    } else if (lane == 0) {
      constexpr uint32_t id_s = idesc_f16(128, SW, BF16, false, false);
      const uint64_t da0 = sdesc(saddr(s.sring), 16, 1024);   // K-major, 128B swizzle
      Ring rg(ns);
      Ring gr(1);
      bool ok = true;
      for (int i = 0; i < n && ok; ++i) {
        // the accumulator buffer of tile i was last read by the softmax of tile i - 2
        if (!QB && i >= 2 && !mbar_wait(saddr(&s.p_full[i & 1]), uint32_t((i - 2) >> 1) & 1u)) { ok = false; break; }
        uint32_t d = tmem + uint32_t((i & 1) * SW);
        for (int u = 0; u < NI; ++u) {
          if (QB && (u & 1) == 0) {
            // a group (128 channels, two boxes) starts: its buffer must be free
            if (!mbar_wait(saddr(&s.sg_empty[gr.slot]), gr.phase ^ 1u)) { ok = false; break; }
            d = tmem + uint32_t(gr.slot * SW);
          }
          if (!mbar_wait(saddr(&s.s_full[rg.slot]), rg.phase)) { ok = false; break; }
          tc_fence_after();
          // descriptor address field is in 16-byte units
          const uint64_t sa = da0 + uint64_t((rg.slot * s_slot_bytes<NP, QS>()) >> 4);
          const int first = QB ? (u & 1) : u;   // accumulate from the group's (or tile's) first box on
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {   // K = 16 channels per MMA
            const uint64_t a = sa + uint64_t((kk * 32) >> 4);
            const uint64_t bd = sa + uint64_t((kBoxBytes + kk * 32) >> 4);
            tc_mma(d, a, bd, id_s, (first | kk) != 0);
          }
          tc_commit(saddr(&s.s_empty[rg.slot]));
          rg.advance();
          if (QB && (u & 1) == 1) {
            tc_commit(saddr(&s.sg_full[gr.slot]));
            gr.advance();
          }
        }
        if (!ok) break;
        if (!QB) tc_commit(saddr(&s.acc_full[i & 1]));
        if (*s.abort_flag) ok = false;
      }
      if (!ok) set_abort(s, status);
      tc_commit(saddr(&s.drain[0]));
      mbar_wait(saddr(&s.drain[0]), 0);
    }
    __syncwarp();
  } else if (warp == 3 || (SG && warp == 1)) {
    // ----------------------------------------------------------- Z MMAs
    if (lane == 0) {
      const int kind = warp >> 1;   // SG: ring and chunk parity of this issuer
      const bool ra = SG && kind == 0;
      uint64_t* zfull = ra ? s.s_full : s.z_full;
      uint64_t* zempty = ra ? s.s_empty : s.z_empty;
      constexpr uint32_t id_z = idesc_f16(128, NP, BF16, true, false);
      const uint64_t za0 = sdesc(saddr(ra ? s.sring : s.zring), kZBoxBytes, 1024);  // MN-major C^T
      const uint64_t pb0 = sdesc(saddr(s.pbuf), 16, 1024);                          // P^T, K-major
      TileIter it;
      it.init(sched, B, tb, te);
      Ring rg(ra ? ns : nz);
      int sbi = 0;   // quantised latent: scale table of the tile
      bool ok = true;
      for (int i = 0; i < n && ok; ++i) {
        const bool first = it.first(tb);
        if (!mbar_wait(saddr(&s.p_full[i & 1]), uint32_t(i >> 1) & 1u)) { ok = false; break; }
        const uint64_t pb = pb0 + uint64_t(((i & 1) * PS * pbuf_bytes<NP>()) >> 4);
        for (int u = 0; u < NI; ++u) {
          const int j = u >> 1, h = u & 1;   // 128-channel chunk, 64-token half
          if (SG && !sg_owns(j, ch, cpart, kind)) continue;
          if (!mbar_wait(saddr(&zfull[rg.slot]), rg.phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + uint32_t(ZC0 + (SG ? j / ch : j) * NP);
          const uint64_t za = za0 + uint64_t((rg.slot * kZSlotBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {   // K = 16 tokens per MMA
            const uint64_t a = za + uint64_t((kk * 16 * 128) >> 4);
#pragma unroll
            for (int part = 0; part < PS; ++part) {   // P = P_hi (+ P_lo for bf16)
              const uint64_t bd = pb + uint64_t((part * pbuf_bytes<NP>() + h * NP * 128 + kk * 32) >> 4);
              tc_mma(d, a, bd, id_z, (first && h == 0 && kk == 0 && part == 0) ? 0u : 1u);
            }
          }
          tc_commit(saddr(&zempty[rg.slot]));
          rg.advance();
        }
        if (!ok) break;
        tc_commit(saddr(&s.z_done[i & 1]));
        if (QB) {   // the tile's scale table is free once its Z MMAs are complete
          tc_commit(saddr(&s.zsc_empty[sbi]));
          if (++sbi == kScaleBufs) sbi = 0;
        }
        it.next();
        if (*s.abort_flag) ok = false;
      }
      if (!ok) set_abort(s, status);
      tc_commit(saddr(&s.drain[kind]));
      mbar_wait(saddr(&s.drain[kind]), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ softmax and epilogue
    // WG groups of four warps (warps 4-7, and 12-15 when WG = 2) each own
    // HW = NP / WG heads, hb .. hb + HW - 1: their score columns, running max
    // and sum, P rows, Z columns and partials; a group synchronises on its
    // own named barrier (1 + wg)
    const int q = warp & 3;
    const int t = 32 * q + lane;              // token row in the tile == TMEM lane
    const int wg = warp >= 12 ? 1 : 0, hb = wg * HW, bid = 1 + wg;
    const uint32_t lane_off = uint32_t(32 * q) << 16;
    const uint64_t inject_ns = g_score_wait_ns;
    // m and l per head live in shared memory (identical for the group's four
    // warps); thread t < HW owns head hb + t's entries
    TileIter it;
    it.init(sched, B, tb, te);
    Ring sgr(QB ? nsg : 1);   // quantised latent: the per-group S buffers
    Ring scb(kScaleBufs);     // ... and the tiles' scale tables
    constexpr uint32_t kBias = 0x4B400000u;   // the bits of 1.5 x 2^23
    if (QB) {   // the group buffers start biased (each warp its own 32 TMEM lanes)
      for (int gb = 0; gb < nsg; ++gb)
#pragma unroll
        for (int c = 0; c < 3 * HW / 16; ++c)
          tmem_fill16(tmem + lane_off + uint32_t(gb * SW + (c / (HW / 16)) * NP + hb + 16 * (c % (HW / 16))), kBias);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0)
        for (int gb = 0; gb < nsg; ++gb) mbar_arrive(saddr(&s.sg_empty[gb]));
    }
    for (int i = 0; i < n; ++i) {
      const int pb = i & 1;
      const bool first = it.first(tb), last = it.last();
      const int nv = it.nvalid();
      int fail = 0;
      if (inject_ns && i == 0 && group_or(!mbar_wait_ns(saddr(s.never), 0, inject_ns), bid)) {
        if (t == 0) set_abort(s, status);
        break;
      }
      float sv[HW];
      if (QB) {
        // s_t = sigma_h sum_g scale_{t,g} (S0 + S1 / 128 + S2 / 16384), S_k
        // the exact int32 sums of one group buffer (columns k NP + h) and
        // sigma_h the query parts' scale of this (sequence, head), staged in
        // shared memory here and read after the barrier that ends the group loop
        if (t < HW) s.qsig[hb + t] = hb + t < H ? __ldg(qsh + size_t(it.b) * H + hb + t) : 0.f;
#pragma unroll
        for (int h = 0; h < HW; ++h) sv[h] = 0.f;
        // the groups run without CTA-level barriers: each warp waits for a
        // buffer itself and releases it with its own arrive; a failed wait
        // stops that warp's loop and the four agree after it
        fail = !__all_sync(0xffffffffu, mbar_wait(saddr(&s.zsc_full[scb.slot]), scb.phase));   // scale table
        const uint32_t tsc = saddr(s.zsc) + uint32_t(scb.slot * scale_buf_bytes(r) + t * NC * 2);
        scb.advance();
        for (int grp = 0; grp < NC && !fail; ++grp) {
          const float sg = __half2float(lds16h(tsc + uint32_t(grp * 2)));   // 0 past the length
          fail = !__all_sync(0xffffffffu, mbar_wait(saddr(&s.sg_full[sgr.slot]), sgr.phase));   // warp-uniform
          if (fail) break;
          tc_fence_after();
          const uint32_t tg = tmem + lane_off + uint32_t(sgr.slot * SW);
#pragma unroll
          for (int c = 0; c < HW / 16; ++c) {
            float a0[16], a1[16], a2[16];
            tmem_ld16(tg + uint32_t(hb + 16 * c), a0);
            tmem_ld16(tg + uint32_t(NP + hb + 16 * c), a1);
            tmem_ld16(tg + uint32_t(2 * NP + hb + 16 * c), a2);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int h = 16 * c + e;
              // a_k = 1.5 x 2^23 + S_k as floats (exact); subtracting the
              // three biases (1.5 x 2^23 (1 + 2^-7 + 2^-14)) from a_0 is exact
              // and leaves S0 + S1 / 128 + S2 / 16384 after the two fmas
              const float g0 = a0[e] - 12681984.f;
              sv[h] = fmaf(sg, fmaf(a2[e], 1.f / 16384.f, fmaf(a1[e], 1.f / 128.f, g0)), sv[h]);
            }
          }
          // refill the buffer with the bias for its next group
#pragma unroll
          for (int c = 0; c < 3 * HW / 16; ++c)
            tmem_fill16(tg + uint32_t((c / (HW / 16)) * NP + hb + 16 * (c % (HW / 16))), kBias);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(saddr(&s.sg_empty[sgr.slot]));
          sgr.advance();
        }
        if (group_or(fail, bid)) { if (t == 0) set_abort(s, status); break; }   // also orders the qsig stores
#pragma unroll
        for (int h = 0; h < HW; ++h) sv[h] *= s.qsig[hb + h];
      } else if (SG) {
        // head h's scores of this tile: 128 consecutive floats per warp-row
        const float* sc = scores + size_t(it.b) * H * max_len + it.t0() + t;
        const bool ok = t < nv;
#pragma unroll
        for (int h = 0; h < HW; ++h) sv[h] = (ok && hb + h < H) ? __ldg(sc + size_t(hb + h) * max_len) : -INFINITY;
      } else {
        fail = !mbar_wait(saddr(&s.acc_full[pb]), uint32_t(i >> 1) & 1u);
        if (group_or(fail, bid)) { if (t == 0) set_abort(s, status); break; }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < HW / 16; ++c) tmem_ld16(tmem + lane_off + uint32_t(pb * SW + hb + 16 * c), sv + 16 * c);
        if (QS == 2) {   // S = C (q_hi + q_lo)
          float lo[HW];
#pragma unroll
          for (int c = 0; c < HW / 16; ++c)
            tmem_ld16(tmem + lane_off + uint32_t(pb * SW + NP + hb + 16 * c), lo + 16 * c);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < HW; ++h) sv[h] += lo[h];
        }
        tmem_wait_ld();
      }
      const bool valid = t < nv;
      int need = first;   // a segment starts: m and l are set below
#pragma unroll
      for (int h = 0; h < HW; ++h) {
        if (!valid) sv[h] = -INFINITY;
        need |= sv[h] > s.m_run[hb + h] + kRescaleLog2;
      }
      if (group_or(need, bid)) {
        // exact tile max per head over the 128 rows
        {
          float tmp[HW];
#pragma unroll
          for (int h = 0; h < HW; ++h) tmp[h] = sv[h];
          reduce_heads<HW>(tmp, s.red + q * NP + hb, lane, dev::OpMax());
        }
        group_sync(bid);
        if (t < HW) {
          const int h = hb + t;
          const float mt = fmaxf(fmaxf(s.red[h], s.red[NP + h]), fmaxf(s.red[2 * NP + h], s.red[3 * NP + h]));
          const float mo = first ? -INFINITY : s.m_run[h];
          const float mn = fmaxf(mo, mt);
          const float a = exp2f(mo - mn);
          s.alpha[h] = a;
          s.m_run[h] = mn;
          s.l_run[h] = first ? 0.f : s.l_run[h] * a;
        }
        group_sync(bid);
        if (!first) {
          // Z of the previous tile must be complete before it is rescaled
          fail = !mbar_wait(saddr(&s.z_done[(i - 1) & 1]), uint32_t((i - 1) >> 1) & 1u);
          if (group_or(fail, bid)) { if (t == 0) set_abort(s, status); break; }
          tc_fence_after();
          for (int c = 0; c < NCL; ++c) {
#pragma unroll
            for (int h16 = 0; h16 < HW / 16; ++h16) {
              float z[16];
              const uint32_t ta = tmem + lane_off + uint32_t(ZC0 + c * NP + hb + 16 * h16);
              tmem_ld16(ta, z);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) z[e] *= s.alpha[hb + 16 * h16 + e];
              tmem_st16(ta, z);
            }
          }
          tmem_wait_st();
        }
      }
      // P = 2^(s - m) as the B operand of the Z MMA: P^T, K-major, 128B swizzle
      if (i >= 2) {
        fail = !mbar_wait(saddr(&s.z_done[pb]), uint32_t((i - 2) >> 1) & 1u);
        if (group_or(fail, bid)) { if (t == 0) set_abort(s, status); break; }
      }
      uint8_t* pbase = s.pbuf + pb * PS * pbuf_bytes<NP>() + (t >> 6) * NP * 128;
      const int chunk = (t & 63) >> 3, within = (t & 7) * 2;
      float mr[HW];   // m into registers first: the P stores below would order each reload
#pragma unroll
      for (int h4 = 0; h4 < HW / 4; ++h4) {
        const float4 v = reinterpret_cast<const float4*>(s.m_run + hb)[h4];
        mr[4 * h4] = v.x;
        mr[4 * h4 + 1] = v.y;
        mr[4 * h4 + 2] = v.z;
        mr[4 * h4 + 3] = v.w;
      }
#pragma unroll
      for (int h = 0; h < HW; ++h) {
        const float p = valid ? exp2f(sv[h] - mr[h]) : 0.f;
        sv[h] = p;
        uint8_t* dst = pbase + (hb + h) * 128 + ((chunk ^ ((hb + h) & 7)) << 4) + within;
        if (PS == 2) {
          const __nv_bfloat16 hi = __float2bfloat16_rn(p);
          *reinterpret_cast<__nv_bfloat16*>(dst) = hi;
          *reinterpret_cast<__nv_bfloat16*>(dst + pbuf_bytes<NP>()) =
              __float2bfloat16_rn(p - __bfloat162float(hi));
        } else {
          *reinterpret_cast<__half*>(dst) = __float2half_rn(p);
        }
      }
      fence_proxy_async();
      tc_fence_before();
      group_sync(bid);
      if (t == 0) mbar_arrive(saddr(&s.p_full[pb]));   // one arrive per group
      // l += this tile's P summed over its 128 tokens (after the hand-off)
      reduce_heads<HW>(sv, s.red + q * NP + hb, lane, dev::OpAdd());
      group_sync(bid);
      if (t < HW) {
        const int h = hb + t;
        s.l_run[h] += (s.red[h] + s.red[NP + h]) + (s.red[2 * NP + h] + s.red[3 * NP + h]);
      }
      if (last) {
        fail = !mbar_wait(saddr(&s.z_done[pb]), uint32_t(i >> 1) & 1u);
        if (group_or(fail, bid)) { if (t == 0) set_abort(s, status); break; }
        tc_fence_after();
        const size_t slot = size_t(g) + it.b;
        // z^T chunk c: TMEM lane = channel 128 c + t, column = head, taken
        // EW head columns at a time (registers); the load of chunk c + 1 is
        // in flight while chunk c is stored
        constexpr int EW = HW % 32 == 0 ? 32 : 16;
        float* zrow = pz + slot * size_t(H) * r + t;
#pragma unroll 1
        for (int hg = 0; hg < HW / EW; ++hg) {
          float zc[EW], zn[EW];
          const int h0 = hb + hg * EW;   // first head of the group of columns
          const uint32_t tcol = tmem + lane_off + uint32_t(ZC0 + h0);
#pragma unroll
          for (int e16 = 0; e16 < EW / 16; ++e16) tmem_ld16(tcol + uint32_t(16 * e16), zc + 16 * e16);
          tmem_wait_ld();
          for (int c = 0; c < NCL; ++c) {
            if (c + 1 < NCL) {
#pragma unroll
              for (int e16 = 0; e16 < EW / 16; ++e16)
                tmem_ld16(tcol + uint32_t((c + 1) * NP + 16 * e16), zn + 16 * e16);
            }
            // row pointer stepped by r: no per-store index arithmetic
            float* zp = zrow + size_t(h0) * r + 128 * (SG ? c * ch + cpart : c);
#pragma unroll
            for (int e = 0; e < EW; ++e) {
              if (h0 + e < H) *zp = zc[e];
              zp += r;
            }
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < EW; ++e) zc[e] = zn[e];
          }
        }
        if (cpart == 0 && t < HW && hb + t < H) {   // the thread that owns head hb + t's m and l
          pl[slot * H + hb + t] = s.l_run[hb + t];
          pm[slot * H + hb + t] = s.m_run[hb + t];
        }
      }
      it.next();
      if (group_or(*s.abort_flag, bid)) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ---------------------------------------------------------------------------
// Rotary scores on the tensor cores (rotary mode, d_h = 128).
//
//   K_h = C_tile W^u_{k,h}      (128 tokens x 128, K = r)   tcgen05, two heads
//                                                            per MMA (N = 256)
//   s_{t,h} = (R(t) K_{h,t}) . q'_h                          CUDA cores
//
// where q'_h is the query already rotated to its position and scaled by
// tau log2(e) (the prologue's rotary query).  Keys are rebuilt from the
// shared latent as the QSVD digest's rotary reading requires (Method, Step
// 1); the scores go to the workspace, [B][H][max_len] fp32, and the split
// kernel that follows takes them instead of computing C . q~.
//
// Per CTA: the flattened tile range of the split schedule.  Per tile and head
// pair the producer streams (latent box, W^u_k^T box) pairs through a ring,
// one thread issues the MMAs into one of two TMEM buffers (256 columns each),
// and four epilogue warps (one TMEM lane per token) apply the rotation with
// the token's cos/sin row, staged once per tile in shared memory, and take the
// dot products.  Every wait is bounded as in k_split_tc.
// ---------------------------------------------------------------------------
constexpr int kRopeSlotBytes = kBoxBytes + 256 * 128;   // latent box + 256 rows of W^u_k^T
constexpr int kRopeTabPitch = 65;                        // floats per token row (bank-conflict free)

template <bool BF16>
__global__ void __launch_bounds__(192, 1)
k_rope_scores(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_w,
              const float* __restrict__ qrot, const float* __restrict__ rope_tab,
              const int32_t* __restrict__ sched, float* __restrict__ scores, int32_t* __restrict__ status,
              int B, int H, int E, int r, int max_len, int G, int ns) {
  dev::pdl_wait();   // see launch_pdl
  dev::pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = base;
  float* tab_c = reinterpret_cast<float*>(ring + size_t(ns) * kRopeSlotBytes);   // [128][65] cos
  float* tab_s = tab_c + 128 * kRopeTabPitch;                                       // [128][65] sin
  uint64_t* bars = reinterpret_cast<uint64_t*>(tab_s + 128 * kRopeTabPitch);
  uint64_t* full = bars;                  // [kMaxSlots]
  uint64_t* empty = bars + kMaxSlots;     // [kMaxSlots]
  uint64_t* kfull = bars + 2 * kMaxSlots; // [2]
  uint64_t* kempty = kfull + 2;           // [2]
  uint64_t* drain = kempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NI = r / 64, NPAIR = (H + 1) / 2;
  const long long T = sched[B];
  const long long tb = dev::split_begin(blockIdx.x, G, T);
  const long long te = dev::split_begin(blockIdx.x + 1, G, T);
  if (tb >= te) return;   // uniform across the CTA, before any barrier or TMEM use
  const int n = int(te - tb);

  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(saddr(&full[i]), 1);
      mbar_init(saddr(&empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(saddr(&kfull[i]), 1);
      mbar_init(saddr(&kempty[i]), 1);
    }
    mbar_init(saddr(drain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     saddr(tmem_holder))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t ring0 = saddr(ring);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    TileIter it;
    it.init(sched, B, tb, te);
    Ring rg(ns);
    long long k = 0;
    bool ok = true;
    for (int i = 0; i < n && ok; ++i) {
      const int row = it.b * max_len + it.t0();   // rows past the length give keys nobody reads
      for (int p = 0; p < NPAIR && ok; ++p)
        for (int u = 0; u < NI; ++u) {
          if (!__all_sync(0xffffffffu, mbar_wait(saddr(&empty[rg.slot]), rg.phase ^ 1u))) { ok = false; break; }
          const uint32_t dst = ring0 + uint32_t(rg.slot) * kRopeSlotBytes;
          const uint32_t fb = saddr(&full[rg.slot]);
          if (lane == 0) mbar_expect_tx(fb, uint32_t(kRopeSlotBytes));
          __syncwarp();
          const int ln = int(k & 15) * 2;   // rotating issuing lanes
          if (lane == ln) tma_load_2d(dst, &tm_c, 64 * u, row, fb);
          if (lane == ln + 1) tma_load_2d(dst + kBoxBytes, &tm_w, 64 * u, 256 * p, fb);   // rows >= E are zeros
          __syncwarp();
          rg.advance();
          ++k;
        }
      it.next();
      if (__any_sync(0xffffffffu, *abort_flag)) ok = false;
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      atomicOr(status, QSVD_STATUS_TIMEOUT);
      drain_ring(full, k, ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t id = idesc_f16(128, 256, BF16, false, false);
      const uint64_t da0 = sdesc(ring0, 16, 1024);   // K-major, 128B swizzle
      Ring rg(ns);
      long long pc = 0;   // head pairs issued
      bool ok = true;
      for (int i = 0; i < n && ok; ++i)
        for (int p = 0; p < NPAIR && ok; ++p, ++pc) {
          const int kb = int(pc & 1);
          if (pc >= 2 && !mbar_wait(saddr(&kempty[kb]), uint32_t((pc - 2) >> 1) & 1u)) { ok = false; break; }
          const uint32_t d = tmem + uint32_t(kb * 256);
          for (int u = 0; u < NI; ++u) {
            if (!mbar_wait(saddr(&full[rg.slot]), rg.phase)) { ok = false; break; }
            tc_fence_after();
            const uint64_t sa = da0 + uint64_t((rg.slot * kRopeSlotBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)   // K = 16 channels per MMA
              tc_mma(d, sa + uint64_t((kk * 32) >> 4), sa + uint64_t((kBoxBytes + kk * 32) >> 4), id,
                     (u | kk) != 0);
            tc_commit(saddr(&empty[rg.slot]));
            rg.advance();
          }
          if (!ok) break;
          tc_commit(saddr(&kfull[kb]));
          if (*abort_flag) ok = false;
        }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(status, QSVD_STATUS_TIMEOUT);
      }
      tc_commit(saddr(drain));
      mbar_wait(saddr(drain), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ rotation and scores
    const int q = warp & 3;
    const int t = 32 * q + lane;              // token row in the tile == TMEM lane
    const uint32_t lane_off = uint32_t(32 * q) << 16;
    float* tc = tab_c + t * kRopeTabPitch;    // this token's cos / sin row (private)
    float* ts = tab_s + t * kRopeTabPitch;
    TileIter it;
    it.init(sched, B, tb, te);
    long long pc = 0;
    for (int i = 0; i < n; ++i) {
      const int nv = it.nvalid(), b = it.b, t0 = it.t0();
      if (t < nv) {   // the row of position t0 + t: 64 (cos, sin) pairs
        const float4* src = reinterpret_cast<const float4*>(rope_tab + size_t(t0 + t) * 128);
#pragma unroll 8
        for (int v = 0; v < 32; ++v) {
          const float4 x = __ldg(src + v);
          tc[2 * v] = x.x; ts[2 * v] = x.y; tc[2 * v + 1] = x.z; ts[2 * v + 1] = x.w;
        }
      }
      const float* qb = qrot + size_t(b) * E;
      int fail = 0;
      for (int p = 0; p < NPAIR; ++p, ++pc) {
        const int kb = int(pc & 1);
        fail = group_or(!mbar_wait(saddr(&kfull[kb]), uint32_t(pc >> 1) & 1u));   // uniform
        if (fail) break;
        tc_fence_after();
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          const int h = 2 * p + hh;
          if (h >= H) break;
          const float* qh = qb + h * 128;
          const uint32_t ta = tmem + lane_off + uint32_t(kb * 256 + hh * 128);
          float s = 0.f;
#pragma unroll 1
          for (int i0 = 0; i0 < 64; i0 += 16) {
            float klo[16], khi[16];
            tmem_ld16(ta + uint32_t(i0), klo);
            tmem_ld16(ta + uint32_t(64 + i0), khi);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int j = i0 + e;
              const float c = tc[j], sn = ts[j];
              s = fmaf(__ldg(qh + j), fmaf(klo[e], c, -khi[e] * sn), s);
              s = fmaf(__ldg(qh + 64 + j), fmaf(khi[e], c, klo[e] * sn), s);
            }
          }
          if (t < nv) scores[(size_t(b) * H + h) * max_len + t0 + t] = s;
        }
        tc_fence_before();
        group_sync();
        if (t == 0) mbar_arrive(saddr(&kempty[kb]));
      }
      if (fail) {
        if (t == 0) { *abort_flag = 1; atomicOr(status, QSVD_STATUS_TIMEOUT); }
        break;
      }
      it.next();
      if (group_or(*abort_flag)) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ------------------------------------------------------------------- host

constexpr int kSmemLimit = 232448;   // opt-in dynamic shared memory per block on sm_100

// Slots per ring.  The S ring holds about 96 KB, the Z ring the rest of the
// shared memory.  On the LLaVA-7B-shaped layer (fp16 latent, r = 1536, 32
// heads) 4 S + 7 Z slots took 102.7 us, 4 + 6 104.5, 3 + 8 105.0, 3 + 7
// 105.7, 5 + 5 111.1, 5 + 4 125.5, 6 + 4 128.8: the Z stream (re-reads from
// L2) is the more sensitive of the two.
constexpr int kRingTargetBytes = 96 * 1024;
template <int NP, int QS, int PS>
void ring_slots(int* ns, int* nz) {
  const int avail = kSmemLimit - 1024 - kMiscBytes - 2 * PS * pbuf_bytes<NP>();
  const int sb = s_slot_bytes<NP, QS>();
  int s = kRingTargetBytes / sb;
  if (s > kMaxSlots) s = kMaxSlots;
  const int zbytes = avail - s * sb;
  int z = zbytes / kZSlotBytes;
  if (z > kMaxSlots) z = kMaxSlots;
  *ns = s;
  *nz = z;
}

template <int NP, bool BF16, int QB, bool SG = false>
cudaError_t launch_t(const qsvd_dims& d, const void* cache, const void* scales, const void* qt16,
                     const float* scores, const int32_t* sched, int G, float* pm, float* pl,
                     float* pz, int32_t* status, cudaStream_t s, int ch = 1, const float* qsh = nullptr) {
  TensorMapEncode enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  constexpr int QS = 2;              // absorbed query as hi + lo 16-bit parts
  constexpr int PS = BF16 ? 2 : 1;   // P as hi + lo parts for bf16 (8-bit mantissa)
  const CUtensorMapDataType dt = BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t rows = cuuint64_t(d.batch) * d.max_len;
  CUtensorMap tcs, tcz, tq;
  memset(&tcs, 0, sizeof(tcs));
  memset(&tcz, 0, sizeof(tcz));
  memset(&tq, 0, sizeof(tq));
  if (QB) {
    // quantised latent: code rows [B * max_len][r QB / 8] bytes.  S items are
    // 128-channel groups of 128 rows: int8 codes straight into the MMA's
    // layout (box {128 bytes, 128 rows}, 128-byte swizzle), int4 raw (box
    // {64 bytes, 128 rows}, unswizzled: the warps unpack them).  Z items: box
    // {QB x 16 bytes, 64 rows} (128 channels), unswizzled (converted).
    const cuuint64_t rb = cuuint64_t(d.r) * QB / 8;
    const cuuint64_t dims[2] = {rb, rows};
    const cuuint64_t strides[1] = {rb};
    const cuuint32_t es[2] = {1, 1};
    const cuuint32_t bs[2] = {cuuint32_t(QB * 16), 128}, bz[2] = {cuuint32_t(QB * 16), 64};
    if (enc(&tcs, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(cache), dims, strides, bs, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, QB == 8 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        enc(&tcz, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(cache), dims, strides, bz, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (!QB && !SG) {
    // S items: latent rows [B * max_len][r], one box {64 channels, 128 rows}
    const cuuint64_t dims[2] = {cuuint64_t(d.r), rows};
    const cuuint64_t strides[1] = {cuuint64_t(d.r) * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&tcs, dt, 2, const_cast<void*>(cache), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (!QB) {
    // Z items: the same rows seen as {64 channels, row, 64-channel box}; one
    // box {64, 64, 2} is 64 tokens x 128 channels, smem [box][row][64]
    const cuuint64_t dims[3] = {64, rows, cuuint64_t(d.r / 64)};
    const cuuint64_t strides[2] = {cuuint64_t(d.r) * 2, 128};
    const cuuint32_t box[3] = {64, 64, 2};
    const cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tcz, dt, 3, const_cast<void*>(cache), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (QB) {
    // int8 query parts [B][3][H][r]: {128 channels, head, sequence x part};
    // one box {128, NP, 3} lands as smem [part][head][128 bytes] (rows
    // k NP + h), 128-byte swizzle.  Heads H..NP-1 arrive as zeros.
    const cuuint64_t dims[3] = {cuuint64_t(d.r), cuuint64_t(d.H), cuuint64_t(d.batch) * 3};
    const cuuint64_t strides[2] = {cuuint64_t(d.r), cuuint64_t(d.H) * d.r};
    const cuuint32_t box[3] = {128, cuuint32_t(NP), 3};
    const cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(qt16), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else if (!SG) {
    // query parts: qt16 holds [B][QS][H][r] (hi, then the rounding residual),
    // seen as {64 channels, head, sequence * part, 64-channel box}; one box
    // {64, NP, QS, 1} lands as smem [part][head][64].  Heads H..NP-1 are
    // outside the map and arrive as zeros.
    const cuuint64_t dims[4] = {64, cuuint64_t(d.H), cuuint64_t(d.batch) * QS, cuuint64_t(d.r / 64)};
    const cuuint64_t strides[3] = {cuuint64_t(d.r) * 2, cuuint64_t(d.H) * d.r * 2, 128};
    const cuuint32_t box[4] = {64, cuuint32_t(NP), QS, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    if (enc(&tq, dt, 4, const_cast<void*>(qt16), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  int ns = 0, nz = 0, nraw = 0;
  ring_slots<NP, QS, PS>(&ns, &nz);
  if constexpr (QB != 0) {
    // quantised latent: S slots of codes + query parts (int8 by TMA; int4
    // unpacked from a raw ring of 4 slots, a multiple of its two warps); the
    // fp16 Z slots take the rest -- each converting warp holds one while it
    // expands it, the MMAs read the ones before
    nraw = QB == 4 ? 4 : 0;
    const int avail = kSmemLimit - 1024 - kMiscBytes - 2 * PS * pbuf_bytes<NP>() -
                      kScaleBufs * scale_buf_bytes(d.r) - nraw * raw_s_bytes(QB);
    // int4: two S slots (its S stream waits on the two unpacking warps, not on
    // slots; the Z ring gets the memory: 369 against 382 us at LLaVA-7B int4);
    // int8: three (210 against 224 us), two only where three leave < 5 Z slots
    for (ns = QB == 4 ? 2 : 3; ns >= 2; --ns) {
      nz = (avail - ns * sq_slot_bytes<NP>()) / kZSlotBytes;
      if (nz >= 5) break;
    }
    if (ns < 2) ns = 2;
    if (nz > kMaxSlots) nz = kMaxSlots;
    if (nz < 4) return cudaErrorInvalidConfiguration;
  }
  if constexpr (SG) {
    // no S items: both rings carry Z items and share the budget
    const int avail = kSmemLimit - 1024 - kMiscBytes - 2 * PS * pbuf_bytes<NP>();
    ns = nz = avail / kZSlotBytes / 2;
    if (ns > kMaxSlots) ns = nz = kMaxSlots;
  }
  if (ns < 2 || nz < 2) return cudaErrorInvalidConfiguration;
  // quantised latent: per-group int32 S buffers (3 NP columns) in the TMEM
  // left beside Z
  int nsg = (512 - (d.r / 128) * NP) / (3 * NP);
  if (nsg > kMaxGroupBufs) nsg = kMaxGroupBufs;
  if (QB && nsg < 1) return cudaErrorInvalidConfiguration;
  const size_t smem = 1024 + size_t(ns) * a_slot_bytes<NP, QS, SG, QB>() + size_t(nz) * kZSlotBytes +
                      2 * PS * pbuf_bytes<NP>() +
                      (QB ? size_t(nraw) * raw_s_bytes(QB) + kScaleBufs * scale_buf_bytes(d.r) : 0) + kMiscBytes;
  auto kern = k_split_tc<NP, BF16, QS, PS, QB, SG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  {
    const cudaError_t le = launch_pdl(kern, dim3(G * ch), dim3(split_threads<NP, QB>()), smem, s,
                                     tcs, tcz, tq, static_cast<const uint8_t*>(cache), static_cast<const __half*>(scales), scores, sched, pm, pl, pz, status, d.batch, d.H, d.r, d.max_len, G, ns, nz, nsg, nraw, ch, qsh);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return check_launch();
}

template <bool BF16>
cudaError_t rope_scores_t(const qsvd_dims& d, const void* cache, const void* wukT, const float* qrot,
                          const float* rope_tab, const int32_t* sched, int G, float* scores,
                          int32_t* status, cudaStream_t s) {
  TensorMapEncode enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const CUtensorMapDataType dt = BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap tc, tw;
  {
    const cuuint64_t dims[2] = {cuuint64_t(d.r), cuuint64_t(d.batch) * d.max_len};
    const cuuint64_t strides[1] = {cuuint64_t(d.r) * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&tc, dt, 2, const_cast<void*>(cache), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // W^u_k^T [E][r]: one box is 256 rows (two heads' d_h) x 64 channels
    const cuuint64_t dims[2] = {cuuint64_t(d.r), cuuint64_t(d.E)};
    const cuuint64_t strides[1] = {cuuint64_t(d.r) * 2};
    const cuuint32_t box[2] = {64, 256};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&tw, dt, 2, const_cast<void*>(wukT), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  constexpr int ns = 3;
  const size_t smem = 1024 + size_t(ns) * kRopeSlotBytes + 2 * 128 * kRopeTabPitch * 4 +
                      (2 * kMaxSlots + 5) * 8 + 16;
  auto kern = k_rope_scores<BF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  {
    const cudaError_t le = launch_pdl(kern, dim3(G), dim3(192), smem, s,
                                     tc, tw, qrot, rope_tab, sched, scores, status, d.batch, d.H, d.E, d.r, d.max_len, G, ns);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return check_launch();
}

}  // namespace

int split_tc_heads_padded(const qsvd_dims& d) { return d.H <= 16 ? 16 : (d.H <= 32 ? 32 : 0); }

bool split_tc_supported(const qsvd_dims& d) {
  if (d.rope) return false;
  const bool q = d.cache_dtype == QSVD_I4 || d.cache_dtype == QSVD_I8;
  if (d.cache_dtype != QSVD_F16 && d.cache_dtype != QSVD_BF16 && !q) return false;
  if (q && d.group != 128) return false;   // one scale group = one 128-channel Z chunk
  if (d.r % 128) return false;
  const int np = split_tc_heads_padded(d);
  if (np == 0) return false;
  if (!q && (2 * 2 + d.r / 128) * np > 512) return false;   // two S buffers of 2 np + Z
  if (q && (3 + d.r / 128) * np > 512) return false;        // one int32 group buffer of 3 np + Z
  // quantised: the int8 query parts come from the tensor-core absorb kernel
  if (q && ((d.weight_dtype != QSVD_F16 && d.weight_dtype != QSVD_BF16) || d.d_h % 64 || d.d_h > 256)) return false;
  return true;
}

cudaError_t launch_split_tc(const qsvd_dims& d, const void* cache, const void* scales, const void* qt16,
                            const int32_t* sched, int G, float* pm, float* pl, float* pz,
                            int32_t* status, cudaStream_t s, const float* qsh) {
  const int np = split_tc_heads_padded(d);
  const float* ns = nullptr;
  switch (d.cache_dtype) {
    case QSVD_BF16:
      return np == 16 ? launch_t<16, true, 0>(d, cache, scales, qt16, ns, sched, G, pm, pl, pz, status, s)
                      : launch_t<32, true, 0>(d, cache, scales, qt16, ns, sched, G, pm, pl, pz, status, s);
    case QSVD_I4:
      return np == 16 ? launch_t<16, false, 4>(d, cache, scales, qt16, ns, sched, G, pm, pl, pz, status, s, 1, qsh)
                      : launch_t<32, false, 4>(d, cache, scales, qt16, ns, sched, G, pm, pl, pz, status, s, 1, qsh);
    case QSVD_I8:
      return np == 16 ? launch_t<16, false, 8>(d, cache, scales, qt16, ns, sched, G, pm, pl, pz, status, s, 1, qsh)
                      : launch_t<32, false, 8>(d, cache, scales, qt16, ns, sched, G, pm, pl, pz, status, s, 1, qsh);
    default:
      return np == 16 ? launch_t<16, false, 0>(d, cache, scales, qt16, ns, sched, G, pm, pl, pz, status, s)
                      : launch_t<32, false, 0>(d, cache, scales, qt16, ns, sched, G, pm, pl, pz, status, s);
  }
}

// Scores given: heads padded to 16, 32 or 48 (softmax registers), and the
// Z accumulator of the 128-channel chunks a CTA holds within TMEM's 512
// columns -- shared over ch CTAs when all chunks do not fit.
static int sg_heads_padded(const qsvd_dims& d) {
  return d.H <= 16 ? 16 : (d.H <= 32 ? 32 : (d.H <= 48 ? 48 : 0));
}

int split_tc_scores_parts(const qsvd_dims& d) {
  const int np = sg_heads_padded(d), nc = d.r / 128;
  if (np == 0 || nc == 0) return 0;
  int ch = 1;
  while ((nc + ch - 1) / ch * np > 512) ++ch;
  return ch <= 8 ? ch : 0;
}

bool split_tc_scores_supported(const qsvd_dims& d) {
  if (d.cache_dtype != QSVD_F16 && d.cache_dtype != QSVD_BF16) return false;
  if (d.r % 128) return false;
  return split_tc_scores_parts(d) != 0;
}

cudaError_t launch_split_tc_scores(const qsvd_dims& d, const float* scores, const void* cache,
                                   const int32_t* sched, int G, float* pm, float* pl, float* pz,
                                   int32_t* status, cudaStream_t s) {
  const int np = sg_heads_padded(d), ch = split_tc_scores_parts(d);
  if (ch == 0) return cudaErrorInvalidConfiguration;
#define QSVD_SG(NP, BF)                                                                         \
  launch_t<NP, BF, 0, true>(d, cache, nullptr, nullptr, scores, sched, G, pm, pl, pz, status, s, ch)
  if (d.cache_dtype == QSVD_BF16)
    return np == 16 ? QSVD_SG(16, true) : np == 32 ? QSVD_SG(32, true) : QSVD_SG(48, true);
  return np == 16 ? QSVD_SG(16, false) : np == 32 ? QSVD_SG(32, false) : QSVD_SG(48, false);
#undef QSVD_SG
}

cudaError_t set_score_wait_ns(unsigned long long ns) {
  return cudaMemcpyToSymbol(g_score_wait_ns, &ns, sizeof(ns));
}

bool rope_tc_supported(const qsvd_dims& d) {
  return d.rope && d.d_h == 128 && d.r % 64 == 0 && d.cache_dtype == d.weight_dtype &&
         (d.cache_dtype == QSVD_F16 || d.cache_dtype == QSVD_BF16);
}

cudaError_t launch_rope_scores(const qsvd_dims& d, const void* cache, const void* wukT,
                               const float* qrot, const float* rope_tab, const int32_t* sched,
                               int G, float* scores, int32_t* status, cudaStream_t s) {
  return d.cache_dtype == QSVD_BF16
             ? rope_scores_t<true>(d, cache, wukT, qrot, rope_tab, sched, G, scores, status, s)
             : rope_scores_t<false>(d, cache, wukT, qrot, rope_tab, sched, G, scores, status, s);
}

}  // namespace qsvd
