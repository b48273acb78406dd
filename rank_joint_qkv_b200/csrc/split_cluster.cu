// Split phase on the tensor cores with the latent channels spread over a
// thread-block cluster: absorbed query, 16-bit latent.
//
// A cluster of CS CTAs (one per SM) works on one split's tile range.  CTA k
// of the cluster owns channels [k RC, (k + 1) RC) of every latent row, so a
// 128-token tile enters the cluster once, each CTA staging only its RC
// channels, and the staged slice stays in shared memory from the score MMAs
// to the latent accumulation (QSVD digest, Method, Step 1: scores and the
// latent sum from one shared latent cache; WSVD digest, Problem: the latent
// must not be re-read).  The matching RC channels of the absorbed query stay
// resident for the whole sequence.
//
//   S_k = C[:, slice k] Qt[slice k]^T   per CTA, tcgen05 into TMEM
//   S   = S_0 + S_1 + ... + S_{CS-1}    every CTA sums the CS partials,
//                                       read from the peers' shared memory
//                                       (distributed shared memory), in
//                                       rank order: all CTAs hold the same
//                                       bits of S, hence the same softmax
//   P   = 2^(S - m)                     online softmax, as k_split_tc
//   Z_k^T += C[:, slice k]^T P          per CTA, tcgen05, own channels
//
// Roles (256 threads):
//   warp 0     producer: the query slice (TMA, once per sequence) and the
//              tile slices (TMA; ragged last tile zero-filled by the warp)
//   warp 1     TMEM allocation; one thread issues the S MMAs
//   warp 3     one thread issues the Z MMAs, then frees the tile slot
//   warps 4-7  S partial out of TMEM into the exchange buffer, the cluster
//              sum, softmax, P, the per-segment epilogue
//
// Cross-CTA hand-offs are mbarriers: a CTA announces its partial with one
// remote arrive (release, cluster scope) on every peer's `x_full`, and
// frees the peers' buffers with one remote arrive on every `x_empty` after
// reading them.  Every wait is bounded (2 s of globaltimer); on expiry the
// kernel records QSVD_STATUS_TIMEOUT, stops, and meets the rest of its
// cluster at a final cluster barrier before freeing TMEM, so that no CTA
// leaves while a peer may still read its shared memory.  Every path to that
// barrier is bounded.
#include <cuda.h>

#include <cstring>

#include "internal.cuh"
#include "tc_common.cuh"

namespace qsvd {
namespace {

constexpr int kThreadsCl = 256;
constexpr int kClBox = 128 * 128;              // 128 tokens x 64 channels x 2 bytes
constexpr float kRescaleLog2Cl = 8.f;          // P <= 2^8 before a rescale
constexpr int kClMisc = 2048;

// ------------------------------------------------------ cluster helpers

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait on a barrier that peers arrive on (acquire at cluster scope).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity) {
  if (mbar_try_cluster(bar, parity)) return true;
  const uint64_t t0 = gtimer();
  while (!mbar_try_cluster(bar, parity)) {
    if (gtimer() - t0 > kWaitNs) return false;
  }
  return true;
}
__device__ __forceinline__ void fence_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }
__device__ __forceinline__ float4 ld_cluster_v4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, float4 v) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w)
               : "memory");
}
// All threads of all CTAs of the cluster (release / acquire).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// ------------------------------------------------------- shared memory
//
//   ring   NT tile slots, each the CTA's RC channels of one 128-token tile:
//          RC / 64 boxes of [128 rows][64 channels], 128-byte swizzle
//   qbuf   the CTA's query slice: per 64-channel box [part][NP rows][64],
//          QS = 2 parts (rounded 16-bit query + its rounding residual)
//   xbuf   two exchange buffers of the S partial, [NP / 4][128 tokens][4]
//          floats (16-byte vectors: conflict-free for token-per-thread)
//   pbuf   two P^T buffers, PS parts each, [half][NP rows][64 tokens]
template <int NP, int RC>
struct ClSizes {
  static constexpr int NBX = RC / 64;                  // boxes per tile slot
  static constexpr int kSlot = NBX * kClBox;
  static constexpr int kQBox = 2 * NP * 128;           // QS = 2
  static constexpr int kQBuf = NBX * kQBox;
  static constexpr int kXBuf = NP * 128 * 4;
  static constexpr int kPPart = 2 * NP * 128;
};

struct ClSmem {
  uint8_t* ring;
  uint8_t* qbuf;
  uint8_t* xbuf;       // [2]
  uint8_t* pbuf;       // [2][PS]
  uint64_t* t_full;    // [kClMaxSlots]
  uint64_t* t_empty;   // [kClMaxSlots]
  uint64_t* q_full;
  uint64_t* q_free;
  uint64_t* acc_full;  // [2]
  uint64_t* p_full;    // [2]
  uint64_t* z_done;    // [2]
  uint64_t* x_full;    // [2] partials of all CS CTAs written
  uint64_t* x_empty;   // [2] this CTA's partial read by all CS CTAs
  uint64_t* drain;     // [2]
  float* red;          // [4][NP]
  float* m_run;        // [NP]
  float* l_run;        // [NP]
  float* alpha;        // [NP]
  uint32_t* tmem_holder;
  volatile int* abort_flag;
};
constexpr int kClMaxSlots = 4;

template <int NP, int RC, int PS>
__device__ ClSmem cl_carve(uint8_t* base, int nt) {
  using Z = ClSizes<NP, RC>;
  ClSmem s;
  s.ring = base;
  s.qbuf = s.ring + size_t(nt) * Z::kSlot;
  s.xbuf = s.qbuf + Z::kQBuf;
  s.pbuf = s.xbuf + 2 * Z::kXBuf;
  uint8_t* m = s.pbuf + 2 * PS * Z::kPPart;
  uint64_t* bars = reinterpret_cast<uint64_t*>(m);
  s.t_full = bars;
  s.t_empty = bars + kClMaxSlots;
  s.q_full = bars + 2 * kClMaxSlots;
  s.q_free = s.q_full + 1;
  s.acc_full = s.q_free + 1;
  s.p_full = s.acc_full + 2;
  s.z_done = s.p_full + 2;
  s.x_full = s.z_done + 2;
  s.x_empty = s.x_full + 2;
  s.drain = s.x_empty + 2;   // 2 kClMaxSlots + 14 barriers = 176 bytes
  static_assert(256 + 4 * NP * 4 + 3 * NP * 4 + 32 <= kClMisc, "misc region");
  s.red = reinterpret_cast<float*>(m + 256);
  s.m_run = s.red + 4 * NP;
  s.l_run = s.m_run + NP;
  s.alpha = s.l_run + NP;
  s.tmem_holder = reinterpret_cast<uint32_t*>(s.alpha + NP);
  s.abort_flag = reinterpret_cast<volatile int*>(s.tmem_holder + 4);
  return s;
}

__device__ __forceinline__ void cl_abort(const ClSmem& s, int32_t* status) {
  *s.abort_flag = 1;
  atomicOr(status, QSVD_STATUS_TIMEOUT);
}

// Zero-filled copy of a ragged tile slice into a slot (one warp), in the
// layout TMA produces: nbox boxes of [128 rows][128 bytes], 128-byte swizzle;
// rows >= nv become zeros.  src is the tile's first row at the slice start.
__device__ __forceinline__ void cl_ragged(uint8_t* d, const uint8_t* src, size_t row_bytes, int nbox,
                                          int nv, int lane) {
  const int per_box = kTile * 8;   // 16-byte vectors per box
  for (int idx = lane; idx < nbox * per_box; idx += 32) {
    const int box = idx / per_box, t = (idx >> 3) % kTile, c = idx & 7;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (t < nv) v = *reinterpret_cast<const uint4*>(src + size_t(t) * row_bytes + box * 128 + c * 16);
    *reinterpret_cast<uint4*>(d + box * kTile * 128 + t * 128 + ((c ^ (t & 7)) << 4)) = v;
  }
  fence_proxy_async();   // generic-proxy stores -> visible to the tensor core
  __syncwarp();
}

// ------------------------------------------------------------------ kernel

template <int NP, bool BF16, int RC>
__global__ void __launch_bounds__(kThreadsCl, 1)
k_split_cl(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_q,
           const uint8_t* __restrict__ cache, const int32_t* __restrict__ sched,
           float* __restrict__ pm, float* __restrict__ pl, float* __restrict__ pz,
           int32_t* __restrict__ status, int B, int H, int r, int max_len, int G, int nt) {
  constexpr int QS = 2, PS = BF16 ? 2 : 1;
  constexpr int SW = QS * NP;                 // S accumulator columns per buffer
  constexpr int ZC0 = 2 * SW;                 // first Z column
  using Z = ClSizes<NP, RC>;
  constexpr int NBX = Z::NBX, NCH = RC / 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const ClSmem s = cl_carve<NP, RC, PS>(base, nt);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int CS = r / RC;                      // CTAs per cluster
  const uint32_t rank = cluster_rank();
  const int g = int(blockIdx.x) / CS;         // split = cluster
  const int ch0 = int(rank) * RC;             // this CTA's first channel
  const long long T = sched[B];
  const long long tb = dev::split_begin(g, G, T);
  const long long te = dev::split_begin(g + 1, G, T);
  if (tb >= te) return;   // the same for every CTA of the cluster: none touches a peer
  const int n = int(te - tb);

  if (threadIdx.x == 0) {
    for (int i = 0; i < nt; ++i) {
      mbar_init(saddr(&s.t_full[i]), 1);
      mbar_init(saddr(&s.t_empty[i]), 1);
    }
    mbar_init(saddr(s.q_full), 1);
    mbar_init(saddr(s.q_free), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(saddr(&s.acc_full[i]), 1);
      mbar_init(saddr(&s.p_full[i]), 1);
      mbar_init(saddr(&s.z_done[i]), 1);
      mbar_init(saddr(&s.x_full[i]), uint32_t(CS));    // one arrive per CTA of the cluster
      mbar_init(saddr(&s.x_empty[i]), uint32_t(CS));
      mbar_init(saddr(&s.drain[i]), 1);
    }
    *s.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;" ::"r"(
                     saddr(s.tmem_holder))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    tc_fence_before();
  }
  // every CTA's barriers are initialised before any peer arrives on them
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *s.tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const size_t row_bytes = size_t(r) * 2;
    const uint64_t policy = policy_evict_first();   // the latent is read once
    TileIter it;
    it.init(sched, B, tb, te);
    Ring rg(nt);
    long long k = 0;   // tile loads issued
    int qn = 0;        // query loads issued
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int b = it.b, nv = it.nvalid();
      const int row = b * max_len + it.t0();
      if (it.first(tb)) {
        // a sequence starts: its query slice replaces the last one once the
        // S MMAs of the last one are complete
        if (qn > 0 && !__all_sync(0xffffffffu, mbar_wait(saddr(s.q_free), uint32_t(qn - 1) & 1u))) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_expect_tx(saddr(s.q_full), uint32_t(Z::kQBuf));
        __syncwarp();
        if (lane < NBX)
          tma_load_4d(saddr(s.qbuf) + uint32_t(lane * Z::kQBox), &tm_q, 0, 0, QS * b, ch0 / 64 + lane,
                      saddr(s.q_full));
        ++qn;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(saddr(&s.t_empty[rg.slot]), rg.phase ^ 1u))) {
        ok = false;
        break;
      }
      const uint32_t fb = saddr(&s.t_full[rg.slot]);
      uint8_t* slot = s.ring + size_t(rg.slot) * Z::kSlot;
      if (nv == kTile) {
        if (lane == 0) mbar_expect_tx(fb, uint32_t(Z::kSlot));
        __syncwarp();
        if (lane < NBX)   // one box per lane: a thread's TMA operations run one after another
          tma_load_2d_hint(saddr(slot) + uint32_t(lane * kClBox), &tm_c, ch0 + 64 * lane, row, fb, policy);
      } else {
        // last tile of a sequence: rows past its length are written as zeros
        cl_ragged(slot, cache + size_t(row) * row_bytes + size_t(ch0) * 2, row_bytes, NBX, nv, lane);
        if (lane == 0) mbar_arrive(fb);
      }
      __syncwarp();
      rg.advance();
      ++k;
      it.next();
      if (__any_sync(0xffffffffu, *s.abort_flag)) { ok = false; break; }
    }
    if (!ok && lane == 0) {
      cl_abort(s, status);
      // no copy may be in flight when the CTA leaves
      for (long long kk = (k > nt ? k - nt : 0); kk < k; ++kk)
        mbar_wait(saddr(&s.t_full[int(kk % nt)]), uint32_t(kk / nt) & 1u);
      if (qn > 0) mbar_wait(saddr(s.q_full), uint32_t(qn - 1) & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ S MMAs
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_f16(128, SW, BF16, false, false);
      const uint64_t da0 = sdesc(saddr(s.ring), 16, 1024);   // K-major, 128B swizzle
      const uint64_t qd0 = sdesc(saddr(s.qbuf), 16, 1024);
      TileIter it;
      it.init(sched, B, tb, te);
      Ring rg(nt);
      int qn = 0;
      bool ok = true;
      for (int i = 0; i < n && ok; ++i) {
        if (it.first(tb)) {
          if (!mbar_wait(saddr(s.q_full), uint32_t(qn) & 1u)) { ok = false; break; }
          ++qn;
        }
        // S buffer i & 1 was last read by the softmax of tile i - 2
        if (i >= 2 && !mbar_wait(saddr(&s.p_full[i & 1]), uint32_t((i - 2) >> 1) & 1u)) { ok = false; break; }
        if (!mbar_wait(saddr(&s.t_full[rg.slot]), rg.phase)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + uint32_t((i & 1) * SW);
#pragma unroll
        for (int u = 0; u < NBX; ++u) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {   // K = 16 channels per MMA
            const uint64_t a = da0 + uint64_t((rg.slot * Z::kSlot + u * kClBox + kk * 32) >> 4);
            const uint64_t bq = qd0 + uint64_t((u * Z::kQBox + kk * 32) >> 4);
            tc_mma(d, a, bq, id_s, (u | kk) != 0);
          }
        }
        tc_commit(saddr(&s.acc_full[i & 1]));
        if (it.last()) tc_commit(saddr(s.q_free));   // the query slice may be replaced
        rg.advance();
        it.next();
        if (*s.abort_flag) ok = false;
      }
      if (!ok) cl_abort(s, status);
      tc_commit(saddr(&s.drain[0]));
      mbar_wait(saddr(&s.drain[0]), 0);
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------------------ Z MMAs
    if (lane == 0) {
      constexpr uint32_t id_z = idesc_f16(128, NP, BF16, true, false);
      const uint64_t za0 = sdesc(saddr(s.ring), kClBox, 1024);   // MN-major C^T, boxes kClBox apart
      const uint64_t pb0 = sdesc(saddr(s.pbuf), 16, 1024);       // P^T, K-major
      TileIter it;
      it.init(sched, B, tb, te);
      Ring rg(nt);
      bool ok = true;
      for (int i = 0; i < n && ok; ++i) {
        const bool first = it.first(tb);
        if (!mbar_wait(saddr(&s.p_full[i & 1]), uint32_t(i >> 1) & 1u)) { ok = false; break; }
        if (!mbar_wait(saddr(&s.t_full[rg.slot]), rg.phase)) { ok = false; break; }   // complete already
        tc_fence_after();
        const uint64_t pb = pb0 + uint64_t(((i & 1) * PS * Z::kPPart) >> 4);
#pragma unroll
        for (int j = 0; j < NCH; ++j) {   // 128-channel chunk = boxes 2j, 2j + 1
          const uint32_t d = tmem + uint32_t(ZC0 + j * NP);
          const uint64_t za = za0 + uint64_t((rg.slot * Z::kSlot + 2 * j * kClBox) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {   // K = 16 tokens per MMA
            const uint64_t a = za + uint64_t((kk * 16 * 128) >> 4);
#pragma unroll
            for (int part = 0; part < PS; ++part) {   // P = P_hi (+ P_lo for bf16)
              const uint64_t bd =
                  pb + uint64_t((part * Z::kPPart + (kk >> 2) * NP * 128 + (kk & 3) * 32) >> 4);
              tc_mma(d, a, bd, id_z, (first && kk == 0 && part == 0) ? 0u : 1u);
            }
          }
        }
        tc_commit(saddr(&s.t_empty[rg.slot]));
        tc_commit(saddr(&s.z_done[i & 1]));
        rg.advance();
        it.next();
        if (*s.abort_flag) ok = false;
      }
      if (!ok) cl_abort(s, status);
      tc_commit(saddr(&s.drain[1]));
      mbar_wait(saddr(&s.drain[1]), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------- exchange, softmax and epilogue
    const int q = warp & 3;
    const int t = 32 * q + lane;              // token row in the tile == TMEM lane
    const uint32_t lane_off = uint32_t(32 * q) << 16;
    const uint32_t xb0 = saddr(s.xbuf);
    TileIter it;
    it.init(sched, B, tb, te);
    for (int i = 0; i < n; ++i) {
      const int pb = i & 1;
      const bool first = it.first(tb), last = it.last();
      const int nv = it.nvalid();
      // this CTA's S partial, S_k = C_k (q_hi + q_lo)_k, out of TMEM
      int fail = !mbar_wait(saddr(&s.acc_full[pb]), uint32_t(i >> 1) & 1u);
      if (group_or(fail)) { if (t == 0) cl_abort(s, status); break; }
      tc_fence_after();
      float sv[NP];
      {
        float lo[NP];
#pragma unroll
        for (int c = 0; c < NP / 16; ++c) {
          tmem_ld16(tmem + lane_off + uint32_t(pb * SW + 16 * c), sv + 16 * c);
          tmem_ld16(tmem + lane_off + uint32_t(pb * SW + NP + 16 * c), lo + 16 * c);
        }
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < NP; ++h) sv[h] += lo[h];
      }
      tc_fence_before();
      // exchange buffer pb is free once every CTA has read what tile i - 2 left in it
      if (i >= 2) {
        fail = !mbar_wait_cluster(saddr(&s.x_empty[pb]), uint32_t((i - 2) >> 1) & 1u);
        if (group_or(fail)) { if (t == 0) cl_abort(s, status); break; }
      }
      const uint32_t xb = xb0 + uint32_t(pb * Z::kXBuf);
#pragma unroll
      for (int h4 = 0; h4 < NP / 4; ++h4)
        st_shared_v4(xb + uint32_t((h4 * kTile + t) * 16),
                     make_float4(sv[4 * h4], sv[4 * h4 + 1], sv[4 * h4 + 2], sv[4 * h4 + 3]));
      fence_cluster();
      group_sync();
      if (t < CS) mbar_arrive_remote(peer_addr(saddr(&s.x_full[pb]), uint32_t(t)));   // one peer per thread
      fail = !mbar_wait_cluster(saddr(&s.x_full[pb]), uint32_t(i >> 1) & 1u);
      if (group_or(fail)) { if (t == 0) cl_abort(s, status); break; }
      // S = S_0 + ... + S_{CS-1} in rank order: every CTA holds the same bits
#pragma unroll
      for (int h = 0; h < NP; ++h) sv[h] = 0.f;
      for (int k = 0; k < CS; ++k) {
        const uint32_t src = peer_addr(xb, uint32_t(k)) + uint32_t(t * 16);
#pragma unroll
        for (int h4 = 0; h4 < NP / 4; ++h4) {
          const float4 v = ld_cluster_v4(src + uint32_t(h4 * kTile * 16));
          sv[4 * h4] += v.x;
          sv[4 * h4 + 1] += v.y;
          sv[4 * h4 + 2] += v.z;
          sv[4 * h4 + 3] += v.w;
        }
      }
      fence_cluster();
      group_sync();
      if (t < CS) mbar_arrive_remote(peer_addr(saddr(&s.x_empty[pb]), uint32_t(t)));

      // online softmax, m and l per head in shared memory (thread t < NP owns head t)
      const bool valid = t < nv;
      int need = first;
#pragma unroll
      for (int h = 0; h < NP; ++h) {
        if (!valid) sv[h] = -INFINITY;
        need |= sv[h] > s.m_run[h] + kRescaleLog2Cl;
      }
      if (group_or(need)) {
        {
          float tmp[NP];
#pragma unroll
          for (int h = 0; h < NP; ++h) tmp[h] = sv[h];
          reduce_heads<NP>(tmp, s.red + q * NP, lane, dev::OpMax());
        }
        group_sync();
        if (t < NP) {
          const float mt = fmaxf(fmaxf(s.red[t], s.red[NP + t]), fmaxf(s.red[2 * NP + t], s.red[3 * NP + t]));
          const float mo = first ? -INFINITY : s.m_run[t];
          const float mn = fmaxf(mo, mt);
          const float a = exp2f(mo - mn);
          s.alpha[t] = a;
          s.m_run[t] = mn;
          s.l_run[t] = first ? 0.f : s.l_run[t] * a;
        }
        group_sync();
        if (!first) {
          // Z of the previous tile must be complete before it is rescaled
          fail = !mbar_wait(saddr(&s.z_done[(i - 1) & 1]), uint32_t((i - 1) >> 1) & 1u);
          if (group_or(fail)) { if (t == 0) cl_abort(s, status); break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
#pragma unroll
            for (int h16 = 0; h16 < NP / 16; ++h16) {
              float z[16];
              const uint32_t ta = tmem + lane_off + uint32_t(ZC0 + c * NP + 16 * h16);
              tmem_ld16(ta, z);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) z[e] *= s.alpha[16 * h16 + e];
              tmem_st16(ta, z);
            }
          }
          tmem_wait_st();
        }
      }
      // P = 2^(s - m) as the B operand of the Z MMA: P^T, K-major, 128B swizzle
      if (i >= 2) {
        fail = !mbar_wait(saddr(&s.z_done[pb]), uint32_t((i - 2) >> 1) & 1u);
        if (group_or(fail)) { if (t == 0) cl_abort(s, status); break; }
      }
      uint8_t* pbase = s.pbuf + pb * PS * Z::kPPart + (t >> 6) * NP * 128;
      const int chunk = (t & 63) >> 3, within = (t & 7) * 2;
      float mr[NP];   // m into registers first: the P stores below would order each reload
#pragma unroll
      for (int h4 = 0; h4 < NP / 4; ++h4) {
        const float4 v = reinterpret_cast<const float4*>(s.m_run)[h4];
        mr[4 * h4] = v.x;
        mr[4 * h4 + 1] = v.y;
        mr[4 * h4 + 2] = v.z;
        mr[4 * h4 + 3] = v.w;
      }
#pragma unroll
      for (int h = 0; h < NP; ++h) {
        const float p = valid ? exp2f(sv[h] - mr[h]) : 0.f;
        sv[h] = p;
        uint8_t* dst = pbase + h * 128 + ((chunk ^ (h & 7)) << 4) + within;
        if (PS == 2) {
          const __nv_bfloat16 hi = __float2bfloat16_rn(p);
          *reinterpret_cast<__nv_bfloat16*>(dst) = hi;
          *reinterpret_cast<__nv_bfloat16*>(dst + Z::kPPart) = __float2bfloat16_rn(p - __bfloat162float(hi));
        } else {
          *reinterpret_cast<__half*>(dst) = __float2half_rn(p);
        }
      }
      fence_proxy_async();
      tc_fence_before();
      group_sync();
      if (t == 0) mbar_arrive(saddr(&s.p_full[pb]));
      // l += this tile's P summed over its 128 tokens (after the hand-off)
      reduce_heads<NP>(sv, s.red + q * NP, lane, dev::OpAdd());
      group_sync();
      if (t < NP) s.l_run[t] += (s.red[t] + s.red[NP + t]) + (s.red[2 * NP + t] + s.red[3 * NP + t]);
      if (last) {
        fail = !mbar_wait(saddr(&s.z_done[pb]), uint32_t(i >> 1) & 1u);
        if (group_or(fail)) { if (t == 0) cl_abort(s, status); break; }
        tc_fence_after();
        const size_t slot = size_t(g) + it.b;
        // z^T chunk c of this CTA's slice: TMEM lane = channel ch0 + 128 c + t,
        // column = head; EW head columns per pass, the next chunk's load in
        // flight while this one is stored
        constexpr int EW = NP % 32 == 0 ? 32 : 16;
        float* zrow = pz + slot * size_t(H) * r + ch0 + t;
#pragma unroll 1
        for (int hg = 0; hg < NP / EW; ++hg) {
          float zc[EW], zn[EW];
          const uint32_t tcol = tmem + lane_off + uint32_t(ZC0 + hg * EW);
#pragma unroll
          for (int e16 = 0; e16 < EW / 16; ++e16) tmem_ld16(tcol + uint32_t(16 * e16), zc + 16 * e16);
          tmem_wait_ld();
          for (int c = 0; c < NCH; ++c) {
            if (c + 1 < NCH) {
#pragma unroll
              for (int e16 = 0; e16 < EW / 16; ++e16)
                tmem_ld16(tcol + uint32_t((c + 1) * NP + 16 * e16), zn + 16 * e16);
            }
            float* zp = zrow + size_t(hg * EW) * r + 128 * c;   // stepped by r per head
#pragma unroll
            for (int e = 0; e < EW; ++e) {
              if (hg * EW + e < H) *zp = zc[e];
              zp += r;
            }
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < EW; ++e) zc[e] = zn[e];
          }
        }
        if (rank == 0 && t < H && t < NP) {   // m and l are the same in every CTA of the cluster
          pl[slot * H + t] = s.l_run[t];
          pm[slot * H + t] = s.m_run[t];
        }
      }
      it.next();
      if (group_or(*s.abort_flag)) break;
    }
  }
  // no CTA leaves while a peer may still read its shared memory or arrive on
  // its barriers; every role reaches this point through bounded waits
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem) : "memory");
  }
}

// ------------------------------------------------------------------ host

constexpr int kClSmemLimit = 232448;   // opt-in dynamic shared memory per block on sm_100

// Channel slice per CTA: 256 channels (two Z chunks) when that gives 2..8
// CTAs, else 128; 0 when no cluster of 2..8 CTAs covers r.
int cl_slice(int r) {
  if (r % 256 == 0 && r / 256 >= 2 && r / 256 <= 8) return 256;
  if (r % 128 == 0 && r / 128 >= 2 && r / 128 <= 8) return 128;
  return 0;
}
int cl_heads_padded(int H) { return H <= 16 ? 16 : (H <= 32 ? 32 : 0); }

template <int NP, bool BF16, int RC>
struct ClPlan {
  static constexpr int PS = BF16 ? 2 : 1;
  using Z = ClSizes<NP, RC>;
  static int slots() {
    const int avail = kClSmemLimit - 1024 - kClMisc - Z::kQBuf - 2 * Z::kXBuf - 2 * PS * Z::kPPart;
    int nt = avail / Z::kSlot;
    return nt > kClMaxSlots ? kClMaxSlots : nt;
  }
  static size_t smem(int nt) {
    return 1024 + size_t(nt) * Z::kSlot + Z::kQBuf + 2 * Z::kXBuf + 2 * PS * Z::kPPart + kClMisc;
  }
  // Launch configuration for G clusters of CS CTAs (attr must outlive cfg).
  static cudaError_t config(int CS, int G, cudaStream_t s, cudaLaunchConfig_t* cfg,
                            cudaLaunchAttribute* attr, int* nt) {
    *nt = slots();
    if (*nt < 2) return cudaErrorInvalidConfiguration;
    const size_t sm = smem(*nt);
    cudaError_t e = cudaFuncSetAttribute(k_split_cl<NP, BF16, RC>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm));
    if (e != cudaSuccess) return e;
    memset(cfg, 0, sizeof(*cfg));
    cfg->gridDim = dim3(unsigned(G * CS));
    cfg->blockDim = dim3(kThreadsCl);
    cfg->dynamicSmemBytes = sm;
    cfg->stream = s;
    attr->id = cudaLaunchAttributeClusterDimension;
    attr->val.clusterDim.x = unsigned(CS);
    attr->val.clusterDim.y = 1;
    attr->val.clusterDim.z = 1;
    cfg->attrs = attr;
    cfg->numAttrs = 1;
    return cudaSuccess;
  }
  static int clusters(const qsvd_dims& d) {
    const int CS = d.r / RC;
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr;
    int nt = 0, n = 0;
    if (config(CS, 1, nullptr, &cfg, &attr, &nt) != cudaSuccess) return 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_split_cl<NP, BF16, RC>, &cfg) != cudaSuccess) return 0;
    return n;
  }
  static cudaError_t launch(const qsvd_dims& d, const void* cache, const void* qt16, const int32_t* sched,
                            int G, float* pm, float* pl, float* pz, int32_t* status, cudaStream_t s) {
    TensorMapEncode enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    constexpr int QS = 2;
    const CUtensorMapDataType dt = BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUtensorMap tc, tq;
    memset(&tc, 0, sizeof(tc));
    memset(&tq, 0, sizeof(tq));
    {
      // latent rows [B * max_len][r]: one box {64 channels, 128 rows}
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
      // query parts [B][QS][H][r] as {64 channels, head, sequence * part,
      // 64-channel box}; box {64, NP, QS, 1} lands as [part][head][64];
      // heads H..NP-1 are outside the map and arrive as zeros
      const cuuint64_t dims[4] = {64, cuuint64_t(d.H), cuuint64_t(d.batch) * QS, cuuint64_t(d.r / 64)};
      const cuuint64_t strides[3] = {cuuint64_t(d.r) * 2, cuuint64_t(d.H) * d.r * 2, 128};
      const cuuint32_t box[4] = {64, cuuint32_t(NP), QS, 1};
      const cuuint32_t es[4] = {1, 1, 1, 1};
      if (enc(&tq, dt, 4, const_cast<void*>(qt16), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
    const int CS = d.r / RC;
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr;
    int nt = 0;
    cudaError_t e = config(CS, G, s, &cfg, &attr, &nt);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, k_split_cl<NP, BF16, RC>, tc, tq, static_cast<const uint8_t*>(cache),
                           sched, pm, pl, pz, status, d.batch, d.H, d.r, d.max_len, G, nt);
    if (e != cudaSuccess) return e;
    note_launch();
    return check_launch();
  }
};

template <template <int, bool, int> class F, typename... A>
auto cl_dispatch(const qsvd_dims& d, A&&... a) {
  const bool bf = d.cache_dtype == QSVD_BF16;
  const int np = cl_heads_padded(d.H), rc = cl_slice(d.r);
  if (np == 16) {
    if (rc == 256) return bf ? F<16, true, 256>::run(d, a...) : F<16, false, 256>::run(d, a...);
    return bf ? F<16, true, 128>::run(d, a...) : F<16, false, 128>::run(d, a...);
  }
  if (rc == 256) return bf ? F<32, true, 256>::run(d, a...) : F<32, false, 256>::run(d, a...);
  return bf ? F<32, true, 128>::run(d, a...) : F<32, false, 128>::run(d, a...);
}
template <int NP, bool BF16, int RC>
struct ClClusters {
  static int run(const qsvd_dims& d) { return ClPlan<NP, BF16, RC>::clusters(d); }
};
template <int NP, bool BF16, int RC>
struct ClLaunch {
  static cudaError_t run(const qsvd_dims& d, const void* cache, const void* qt16, const int32_t* sched,
                         int G, float* pm, float* pl, float* pz, int32_t* status, cudaStream_t s) {
    return ClPlan<NP, BF16, RC>::launch(d, cache, qt16, sched, G, pm, pl, pz, status, s);
  }
};

}  // namespace

bool split_cl_supported(const qsvd_dims& d) {
  if (d.rope) return false;
  if (d.cache_dtype != QSVD_F16 && d.cache_dtype != QSVD_BF16) return false;
  return cl_slice(d.r) != 0 && cl_heads_padded(d.H) != 0;
}

int split_cl_clusters(const qsvd_dims& d) {
  if (!split_cl_supported(d)) return 0;
  return cl_dispatch<ClClusters>(d);
}

cudaError_t launch_split_cl(const qsvd_dims& d, const void* cache, const void* qt16, const int32_t* sched,
                            int G, float* pm, float* pl, float* pz, int32_t* status, cudaStream_t s) {
  if (!split_cl_supported(d)) return cudaErrorInvalidConfiguration;
  return cl_dispatch<ClLaunch>(d, cache, qt16, sched, G, pm, pl, pz, status, s);
}

}  // namespace qsvd
