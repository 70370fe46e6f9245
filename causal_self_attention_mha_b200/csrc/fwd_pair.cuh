// fwd_pair.cuh -- causal attention forward on CTA pairs (tcgen05 cta_group::2), d = 128.
//
// Same result as attn_fwd_kernel (fwd.cuh): for every head and 128-row query tile,
// S = scale * Q K^T (causal / document / window masks), online softmax, O = P V / l, LSE,
// as in "Stanford CS336 walkthrough" (lmnt.cn), section 5.1, CausalSelfAttention.forward.
//
// A cluster of two CTAs (a CTA pair) works on an item: two adjacent query tiles of one
// head, one per CTA (rank r takes query tile 2m + r).  Its MMAs are issued once, by one
// thread of rank 0, for both CTAs (M = 256 rows: each CTA's 128 rows land in its own TMEM):
//   S = Q K_j^T   A = each CTA's Q tile, B = K_j split by keys: rank r holds keys
//                 64r .. 64r+63 of the tile (both swizzle chunks of d)
//   O += P V_j    A = each CTA's P in its TMEM, B = V_j split by d: rank r holds the
//                 64-column swizzle chunk r of the tile
// so each CTA loads half of every K and V tile, and each TMEM holds only one query tile:
// S is double-buffered (S(j+2) is computed while the softmax of S(j+1) runs, instead of
// waiting for the PV of tile j as in the single-CTA kernel), the MMA stream keeps the S
// products two key tiles ahead of the PV products across item boundaries, and Q is
// double-buffered, so the next item's first S products are ready when its softmax starts.
// Both CTAs walk the union of the two tiles' key ranges; where a tile is fully masked for
// a CTA's rows its weights are zero (no exponentials are evaluated).
//
// Threads per CTA: 384 = twelve warps.  Warps 0-7 the softmax: warps q and q + 4 share the
// 32 query rows of TMEM lanes 32q .. 32q+31 (one row per lane), warp q taking key columns
// 0-63 of each tile and warp q + 4 columns 64-127; the two exchange their partial row
// maxima through shared memory once per tile (a named barrier of the two warps), and their
// partial row sums once per item.  Warp 8 the loads (lane 0: Q and the K ring; lane 1: the
// V ring), warp 9 the TMEM allocation and (rank 0, lane 0) the MMA issue, warp 10 the O
// stores.
// TMEM per CTA (512 columns): S buffers at 0 and 128; the weights P of key columns
// 64h .. 64h+63, packed bf16, over the first 32 of those S columns; O at 256 (columns
// 64h .. 64h+63 of O rescaled and read by the warps of half h).
//
// Barriers: the full barriers of the loads (q_full, k_full, v_full) and the softmax /
// epilogue handshakes the MMA issuer waits on (p_full, o_free) are counted in rank 0's
// shared memory: both CTAs' loads signal rank 0's barriers (the tensor copies of a CTA pair
// can complete on the peer's barrier) and both CTAs' softmax warps arrive there.  Every MMA
// completion the CTAs wait on (s_full, pv_done, o_done, and the empty barriers of the
// loads) is committed to both CTAs' barriers at once.
#pragma once

#include "fwd.cuh"

namespace ca {

// ------------------------------------------------------------ cluster helpers
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// All threads of both CTAs of the cluster.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_shared_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// Arrive on an mbarrier of any CTA of the cluster.  Release at CTA scope (the default): what
// the arrival hands over is TMEM contents whose tcgen05 stores or loads have completed
// (tcgen05.wait) and been fenced (tcgen05.fence::before_thread_sync); a cluster-scope release
// would add a cluster-wide memory fence to every handoff.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

// Tiled load into this CTA's shared memory whose completion is counted on an mbarrier of
// the pair (rank 0's).  c0 * 2 bytes is a multiple of 16.
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* m, int c0, int c1,
                                                 int c2, uint32_t bar_cluster) {
  if (!tma_coords_ok(c0, c2)) return;
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(bar_cluster)
      : "memory");
}

__device__ __forceinline__ void mma_ss_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t id,
                                            uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(id), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_ts_pair(uint32_t d, uint32_t a, uint64_t b, uint32_t id,
                                            uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
      "r"(a), "l"(b), "r"(id), "r"(acc)
      : "memory");
}

// Arrive on the mbarrier at this offset in both CTAs once all earlier MMAs have completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"((uint16_t)0x3)
      : "memory");
}

// Generic address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ volatile int* map_generic_rank(volatile int* ptr, uint32_t rank) {
  uint64_t r;
  asm volatile("mapa.u64 %0, %1, %2;" : "=l"(r) : "l"(reinterpret_cast<uint64_t>(ptr)), "r"(rank));
  return reinterpret_cast<volatile int*>(r);
}

// Bounded waits of a CTA pair: a timeout (or an abort seen) in one CTA aborts the other too.
struct PairGuard {
  Guard g;
  volatile int* peer_flag;
};

__device__ __forceinline__ bool wait_pair(uint32_t bar, uint32_t parity, const PairGuard& pg,
                                          unsigned site) {
  if (wait_bounded(bar, parity, pg.g, site)) return true;
  *pg.peer_flag = 1;
  return false;
}

// The MMA-issuing thread's wait: the phase is tested once before the (sleeping) bounded wait.
__device__ __forceinline__ bool wait_pair_fast(uint32_t bar, uint32_t parity, const PairGuard& pg,
                                               unsigned site) {
  return mbar_test(bar, parity) || wait_pair(bar, parity, pg, site);
}

__device__ __forceinline__ bool wait_pair_warp(uint32_t bar, uint32_t parity, const PairGuard& pg,
                                               unsigned site) {
  return __all_sync(0xffffffffu, wait_pair(bar, parity, pg, site));
}

// softmax pairs e with e % 4 == this evaluate their exponentials with exp2_fma2
constexpr int kExp2FmaPhase = 0;

struct PairLayout {
  static constexpr int D = 128;
  static constexpr int QB = kRows * D * 2;          // own Q tile: 32 KB (2 swizzle chunks)
  static constexpr int KB = 64 * D * 2;             // own half of a K tile: 64 keys, 16 KB
  static constexpr int KCH = 64 * 128;              // one 64-row swizzle chunk of it: 8 KB
  static constexpr int VB = kRows * 64 * 2;         // own half of a V tile: 64 columns, 16 KB
  static constexpr int NK = 4, NV = 3;              // ring depths
  static constexpr int Q_OFF = 0;                   // + b * QB, b = 0, 1
  static constexpr int K_OFF = Q_OFF + 2 * QB;      // + s * KB
  static constexpr int V_OFF = K_OFF + NK * KB;     // + s * VB
  static constexpr int STG_OFF = V_OFF + NV * VB;   // bf16 O staging tile (Tile<128> layout)
  // values the two softmax warps of a row exchange: [exchange parity][half][row][2] floats
  static constexpr int XCH_OFF = STG_OFF + Tile<128>::BYTES;
  static constexpr int BAR_OFF = XCH_OFF + 2 * 2 * kRows * 2 * 4;
  // q_full[2] q_empty[2] k_full[NK] k_empty[NK] v_full[NV] v_empty[NV] s_full[2] p_full[2]
  // pv_done o_done[2] o_free[2] stg_full stg_free drain
  static constexpr int NBAR = 4 + 2 * NK + 2 * NV + 4 + 8;
  // tmem slot, abort flag, then (rank 0's) copies issued: own Q, K, V and the peer's
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int CNT_OFF = MISC_OFF + 8;
  static constexpr int RING_OFF = CNT_OFF + 6 * 4;  // the MMA issuer's item tile counts
  static constexpr int BYTES = RING_OFF + 4 * 4;
  static constexpr int SMEM = BYTES + 1024;
  static_assert(SMEM <= kMaxDynSmem, "pair forward shared-memory layout");
  static constexpr int THREADS = 384;
  static constexpr uint32_t TMEM_COLS = 512;
};

// Barrier `id` (1-15) of the `n` threads of some warps of this CTA.
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(384, 1)
    attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmKh,
                         const __grid_constant__ CUtensorMap tmV,
                         const __grid_constant__ CUtensorMap tmO, const FwdParams p) {
  constexpr int D = 128;
  using L = PairLayout;
  constexpr int NK = L::NK, NV = L::NV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* gsm;
  const uint32_t sbase = aligned_smem_base(smem_raw, &gsm);
  // the same layout (and so the same barrier offsets) in both CTAs: both check alike
  if (sbase - smem_u32(smem_raw) + L::BYTES > dynamic_smem_bytes()) {
    if (threadIdx.x == 0) report_smem_shortfall();
    return;
  }
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const uint32_t bar0 = sbase + L::BAR_OFF;
  auto q_full = [&](int b) { return bar0 + 8u * b; };
  auto q_empty = [&](int b) { return bar0 + 8u * (2 + b); };
  auto k_full = [&](int s) { return bar0 + 8u * (4 + s); };
  auto k_empty = [&](int s) { return bar0 + 8u * (4 + NK + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (4 + 2 * NK + s); };
  auto v_empty = [&](int s) { return bar0 + 8u * (4 + 2 * NK + NV + s); };
  const uint32_t xb = bar0 + 8u * (4 + 2 * NK + 2 * NV);
  auto s_full = [&](int b) { return xb + 8u * b; };
  auto p_full = [&](int b) { return xb + 8u * (2 + b); };
  const uint32_t pv_done = xb + 32u;
  auto o_done = [&](int x) { return xb + 40u + 8u * x; };  // O buffer x holds a finished item
  auto o_free = [&](int x) { return xb + 56u + 8u * x; };  // ... and has been read
  const uint32_t stg_full = xb + 72u, stg_free = xb + 80u, drain = xb + 88u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gsm + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gsm + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  const int ci = blockIdx.x >> 1, G = gridDim.x >> 1;  // this pair, number of pairs

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(q_full(b), 1);    // rank 0's: its producer's arrive + both CTAs' bytes
      mbar_init(q_empty(b), 1);
      mbar_init(s_full(b), 1);
      mbar_init(p_full(b), 16);   // rank 0's: eight softmax warps of each CTA
    }
    for (int s = 0; s < NK; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    mbar_init(pv_done, 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(o_done(x), 1);
      mbar_init(o_free(x), 16);   // rank 0's: eight epilogue warps of each CTA
    }
    mbar_init(stg_full, 8);
    mbar_init(stg_free, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(L::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const PairGuard g{Guard{abort_flag, p.wait_limit_ns}, map_generic_rank(abort_flag, rank ^ 1u)};
  // copies issued, published to rank 0 for the drain after an abort
  volatile int* cnt = map_generic_rank(reinterpret_cast<volatile int*>(gsm + L::CNT_OFF), 0) +
                      3 * (int)rank;

  if (warp >= 8) {
    // third warpgroup: give registers to the softmax warpgroups, then specialise
    // (launched at 168 per thread: 2 * 128 * 184 + 128 * 136 = 384 * 168)
    regs_shrink<136>();
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {  // Q (double-buffered by item) and the K ring (own halves)
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmKh);
      int nq = 0, gk = 0;
      bool ok = true;
      for (int k_ = 0; ok && k_ * G < p.n_items; ++k_) {
        const int w = snake_item(k_, ci, G, p.n_items);
        if (w < 0) break;
        const FwdItem I = fwd_item(p, w);
        const int qb = nq & 1;
        if (nq >= 2 && !wait_pair(q_empty(qb), ((nq - 2) >> 1) & 1, g, 1)) { ok = false; break; }
        if (leader) mbar_arrive_expect_tx(q_full(qb), 2 * L::QB);
        const uint32_t qbar = map_shared_rank(q_full(qb), 0);
        // this CTA's query tile (past T for rank 1 of a last, single tile: zeros)
        const int q0 = (rank ? I.qt[1] : I.qt[0]) * kRows;
        for (int c = 0; c < 2; ++c)
          tma_load_3d_pair(sbase + L::Q_OFF + qb * L::QB + c * 16384, &tmQ, c * 64, q0, I.bh, qbar);
        ++nq;
        for (int j = I.j_lo; j <= I.j_hi; ++j, ++gk) {
          const int s = gk % NK, u = gk / NK;
          if (u > 0 && !wait_pair(k_empty(s), (u - 1) & 1, g, 1)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(k_full(s), 2 * L::KB);
          const uint32_t kbar = map_shared_rank(k_full(s), 0);
          for (int c = 0; c < 2; ++c)
            tma_load_3d_pair(sbase + L::K_OFF + s * L::KB + c * L::KCH, &tmKh, c * 64,
                             j * kRows + 64 * (int)rank, I.bh, kbar);
        }
      }
      cnt[0] = nq;
      cnt[1] = gk;
    } else if (lane == 1) {  // the V ring (own d-chunk of every V tile)
      tma_prefetch_desc(&tmV);
      int gv = 0;
      bool ok = true;
      for (int k_ = 0; ok && k_ * G < p.n_items; ++k_) {
        const int w = snake_item(k_, ci, G, p.n_items);
        if (w < 0) break;
        const FwdItem I = fwd_item(p, w);
        for (int j = I.j_lo; j <= I.j_hi; ++j, ++gv) {
          const int s = gv % NV, u = gv / NV;
          if (u > 0 && !wait_pair(v_empty(s), (u - 1) & 1, g, 1)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(v_full(s), 2 * L::VB);
          tma_load_3d_pair(sbase + L::V_OFF + s * L::VB, &tmV, 64 * (int)rank, j * kRows, I.bh,
                           map_shared_rank(v_full(s), 0));
        }
      }
      cnt[2] = gv;
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---------------------------------------------------------- MMA issuer
    // Each tcgen05.mma blocks its issuing thread about as long as it runs, so everything else
    // this thread does (waits, bookkeeping) leaves the tensor pipe idle: state is kept in
    // registers and descriptors are bases plus constant offsets.
    if (leader && lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(256, 128, false);  // S: N = 128 keys
      constexpr uint32_t kIdO = idesc_bf16_f32(256, D, true);     // O: N = d, B MN-major
      const uint64_t dQ = sdesc(sbase + L::Q_OFF, 16u, 1024u, 2u);
      const uint64_t dK = sdesc(sbase + L::K_OFF, 16u, 1024u, 2u);
      const uint64_t dV = sdesc(sbase + L::V_OFF, 16384u, 1024u, 2u);
      // key tiles of the pair's items by item position & 3, written by the S cursor (at most
      // two key tiles, so at most two items, ahead of the PV cursor) and read by the PV cursor
      int* const ring_n = reinterpret_cast<int*>(gsm + L::RING_OFF);
      auto n_tiles = [&](int k) -> int {  // 0 past the pair's last item
        const int w = (k * G < p.n_items) ? snake_item(k, ci, G, p.n_items) : -1;
        if (w < 0) return 0;
        const FwdItem I = fwd_item(p, w);
        return I.j_hi - I.j_lo + 1;
      };
      // S cursor: item position sk, its tile sj of sn, global tile st, K slot ks / phase kph
      int sk = 0, sj = 0, sn = n_tiles(0), st = 0, ks = 0;
      uint32_t kph = 0;
      ring_n[0] = sn;
      // PV cursor: item position pk, its tile pj of pn, global tile pt, V slot vs / phase vph
      int pk = 0, pj = 0, pn = sn, pt = 0, vs = 0;
      uint32_t vph = 0;
      bool ok = true;
      // S(st) into buffer st & 1; S runs two key tiles ahead of PV, so S(t+2) follows PV(t)
      // in the in-order MMA stream and overwrites P(t) only after PV(t) has read it
      auto issue_s = [&]() -> bool {
        const int b = st & 1, qb = sk & 1;
        if (sj == 0 && !wait_pair_fast(q_full(qb), (sk >> 1) & 1, g, 2)) return false;
        if (!wait_pair_fast(k_full(ks), kph, g, 3)) return false;
        tc_fence_after();
        const uint64_t a0 = dQ + (uint64_t)((qb * L::QB) >> 4);
        const uint64_t b0 = dK + (uint64_t)((ks * L::KB) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qo = (uint32_t)((kk * 32) / 128) * 16384u + (uint32_t)(kk * 32) % 128u;
          const uint32_t ko = (uint32_t)((kk * 32) / 128) * (uint32_t)L::KCH + (uint32_t)(kk * 32) % 128u;
          mma_ss_pair(tmem + 128u * (uint32_t)b, a0 + (qo >> 4), b0 + (ko >> 4), kIdS, kk > 0);
        }
        tc_commit_pair(s_full(b));
        tc_commit_pair(k_empty(ks));
        if (sj == sn - 1) tc_commit_pair(q_empty(qb));  // the item's last S has read its Q
        if (++ks == NK) {
          ks = 0;
          kph ^= 1u;
        }
        ++st;
        if (++sj == sn) {
          sj = 0;
          ++sk;
          sn = n_tiles(sk);
          ring_n[sk & 3] = sn;
        }
        return true;
      };
      for (int i = 0; ok && i < 2 && sn > 0; ++i) ok = issue_s();
      while (ok && pn > 0) {
        const int b = pt & 1;
        const bool first_pv = (pj == 0), last_pv = (pj == pn - 1);
        // O buffer pk & 1 is overwritten by item pk's first PV: the epilogue of item pk - 2
        // must have read it
        if (first_pv && pk >= 2 && !wait_pair_fast(o_free(pk & 1), ((pk >> 1) - 1) & 1, g, 4)) {
          ok = false;
          break;
        }
        if (!wait_pair_fast(p_full(b), (pt >> 1) & 1, g, 5) || !wait_pair_fast(v_full(vs), vph, g, 6)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t v0 = dV + (uint64_t)((vs * L::VB) >> 4);
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          mma_ts_pair(tmem + 256u + 128u * (uint32_t)(pk & 1),
                      tmem + 128u * (uint32_t)b + 64u * (kk >> 2) + 8u * (kk & 3),
                      v0 + (uint64_t)((kk * 16 * 128) >> 4), kIdO, (!first_pv || kk > 0));
        tc_commit_pair(pv_done);
        tc_commit_pair(v_empty(vs));
        if (last_pv) tc_commit_pair(o_done(pk & 1));
        if (++vs == NV) {
          vs = 0;
          vph ^= 1u;
        }
        ++pt;
        if (++pj == pn) {
          pj = 0;
          ++pk;
          pn = ring_n[pk & 3];
        }
        if (sn > 0) ok = issue_s();  // S(pt + 1), into the buffer PV(pt - 1) has just read
      }
      if (!ok) {
        *abort_flag = 1;
        *g.peer_flag = 1;
      }
    }
    if (lane == 0) {  // every MMA issued has completed (and signalled both CTAs)
      if (leader) tc_commit_pair(drain);
      drain_wait(drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else if (warp == 10) {
    // ------------------------------------------------------------- O stores
    if (lane == 0) {
      tma_prefetch_desc(&tmO);
      int u = 0;
      for (int k_ = 0; k_ * G < p.n_items; ++k_, ++u) {
        const int w = snake_item(k_, ci, G, p.n_items);
        if (w < 0) break;
        const FwdItem I = fwd_item(p, w);
        if (!wait_pair(stg_full, u & 1, g, 11)) break;
        // rows past T are dropped; rank 1 of a last, single tile has none inside T
        const int qt = rank ? I.qt[1] : I.qt[0];
        if (qt < p.n_qt) store_tile<D>(&tmO, sbase + L::STG_OFF, qt * kRows, I.bh);
        bulk_commit();
        bulk_wait_read_all();
        mbar_arrive(stg_free);
      }
      bulk_wait_all();
    }
    __syncwarp();
  }
  } else {
    regs_grow<184>();
    // ------------------------------------------------------ softmax warps
    // Control flow is the same in both warps of a row quarter whatever happens (the named
    // barrier of the two must be reached by both equally often): a failed wait only clears
    // `ok`, which gates the work, and the loops run on to the end.
    const int qd = warp & 3, h = warp >> 2;  // TMEM lane quarter, key-column half
    const int rl = qd * 32 + lane;           // row within the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    // this warp's half of O buffer 0 (+ 128 columns: buffer 1); item k accumulates in k & 1
    const uint32_t tO0 = tmem + lane_off + 256u + 64u * (uint32_t)h;
    const uint32_t xbar = 1u + (uint32_t)qd;                         // named barrier of the two
    float* const xch = reinterpret_cast<float*>(gsm + L::XCH_OFF);
    int nx = 0;  // exchanges so far (slot nx & 1)
    // publish (a, b) for this row, meet the partner warp, return the partner's pair
    auto exchange = [&](float a, float b, float& pa, float& pb) {
      float* mine = xch + (((nx & 1) * 2 + h) * kRows + rl) * 2;
      float* theirs = xch + (((nx & 1) * 2 + (h ^ 1)) * kRows + rl) * 2;
      mine[0] = a;
      mine[1] = b;
      named_bar_sync(xbar, 64);
      pa = theirs[0];
      pb = theirs[1];
      ++nx;
    };
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2(sl2, sl2);
    const uint32_t lead_p0 = map_shared_rank(p_full(0), 0), lead_p1 = map_shared_rank(p_full(1), 0);
    const uint32_t lead_ofree0 = map_shared_rank(o_free(0), 0);
    const uint32_t lead_ofree1 = map_shared_rank(o_free(1), 0);
    bool ok = true;
    int t = 0;  // global key-tile index (s_full / p_full / pv_done phases)
    // The epilogue of item k (normalise its O, LSE, stage the tile for the store warp) runs
    // after the first key tile of item k + 1, when its last PV has long completed; O is
    // double-buffered by item, so item k + 1's PVs go to the other buffer meanwhile.
    auto epilogue = [&](int k, float m, float l, float lr, int row, int bh) {
      ok = ok && wait_pair_warp(o_done(k & 1), (k >> 1) & 1, g, 10);
      tc_fence_after();
      float xl, xlr;  // the partner warp's partial sums of the row
      exchange(l, lr, xl, xlr);
      if (!ok) return;
      l += xl;
      lr += xlr;
      const float mu = (m == -INFINITY) ? 0.f : m;
      if (h == 0 && row < T)
        st_chk(p.lse, (size_t)bh * T + row, (size_t)p.BH * T, (mu + lg2(l)) * kLn2);
      const float inv = 1.0f / lr;
      const uint32_t tO = tO0 + 128u * (uint32_t)(k & 1);
      uint32_t wo[32];
      {
        uint32_t r[2][32];
#pragma unroll
        for (int c = 0; c < 2; ++c) tmem_ld32(tO + 32u * c, r[c]);
        tc_wait_ld();
#pragma unroll
        for (int c = 0; c < 2; ++c) reg_fence(r[c]);
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int e = 0; e < 16; ++e)
            wo[16 * c + e] = pack_bf16(__uint_as_float(r[c][2 * e]) * inv,
                                       __uint_as_float(r[c][2 * e + 1]) * inv);
      }
      // this half of O buffer k & 1 has been read: item k + 2's first PV may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster((k & 1) ? lead_ofree1 : lead_ofree0);
      ok = k == 0 || wait_pair_warp(stg_free, (k - 1) & 1, g, 12);
      if (!ok) return;
      stage_row<D>(gsm + L::STG_OFF, rl, 64 * h, wo);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(stg_full);
    };
    // the previous item, whose epilogue is pending
    int pk_ = -1, prow = 0, pbh = 0;
    float pm = 0.f, pl = 0.f, plr = 0.f;
    for (int k_ = 0; k_ * G < p.n_items; ++k_) {
      const int w = snake_item(k_, ci, G, p.n_items);
      if (w < 0) break;
      const FwdItem I = fwd_item(p, w);
      const int row = (rank ? I.qt[1] : I.qt[0]) * kRows + rl;
      const uint32_t tO = tO0 + 128u * (uint32_t)(k_ & 1);
      int ds = p.doc ? ld_chk(p.doc, (size_t)I.b * T + (row < T ? row : T - 1),
                              (size_t)(p.BH / p.H) * T)
                     : 0;
      ds = ds > row - p.window + 1 ? ds : row - p.window + 1;
      // rows of this quarter: the first and last visible key over its 32 rows (a tile outside
      // every row's range of visible keys gets zero weights without exponentials); the same
      // in both warps of the quarter
      const int row_hi = __reduce_max_sync(0xffffffffu, row);
      const int ds_lo = __reduce_min_sync(0xffffffffu, ds);
      float m = -INFINITY;
      uint64_t acc_l[2], acc_lr[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) acc_l[i] = acc_lr[i] = f2(0.f, 0.f);
      for (int j = I.j_lo; j <= I.j_hi; ++j, ++t) {
        const int c0 = j * kRows + 64 * h;  // first key of this warp's columns
        const int b = t & 1;
        const uint32_t tS = tmem + lane_off + 128u * (uint32_t)b + 64u * (uint32_t)h;
        ok = ok && wait_pair_warp(s_full(b), (t >> 1) & 1, g, 8);
        tc_fence_after();
        if (j * kRows > row_hi || j * kRows + kRows - 1 < ds_lo) {
          // no row of this quarter sees a key of this tile: zero weights
          if (ok) {
            uint32_t z[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) z[e] = 0u;
            tmem_st16(tS, z);
            tmem_st16(tS + 16u, z);
          }
        } else {
          uint32_t sr[2][32];
          float mx = -INFINITY;
          if (ok) {
            tmem_ld32(tS, sr[0]);
            tmem_ld32(tS + 32u, sr[1]);
            tc_wait_ld();
            reg_fence(sr[0]);
            reg_fence(sr[1]);
            if (!((c0 + 63 <= row) && (c0 >= ds))) {
              const int hi = row - c0, lo = ds - c0;  // visible columns: e in [lo, hi]
#pragma unroll
              for (int e = 0; e < 64; ++e)
                if (e > hi || e < lo) sr[e >> 5][e & 31] = 0xFF800000u;  // -inf
            }
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int e = 0; e < 64; e += 8)
#pragma unroll
              for (int q = 0; q < 4; ++q)
                mx4[q] = fmax3(mx4[q], __uint_as_float(sr[(e + 2 * q) >> 5][(e + 2 * q) & 31]),
                               __uint_as_float(sr[(e + 2 * q + 1) >> 5][(e + 2 * q + 1) & 31]));
            mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
          }
          float pmx, unused;
          exchange(mx, 0.f, pmx, unused);
          if (ok) {
            const float m_new = fmaxf(m, fmaxf(mx, pmx) * sl2);
            const bool grow = m_new > m + 8.0f;  // also true the first time a row sees a key
            // the same in both warps: they hold the same m and m_new for each row
            if (__any_sync(0xffffffffu, grow)) {
              const float alpha = grow ? ex2(m - m_new) : 1.0f;
              if (j > I.j_lo) {
                // O holds the PVs up to tile t-1: the last of them must have completed
                // (PV(t-2) has, since S(t) was issued after it)
                ok = wait_pair_warp(pv_done, (t - 1) & 1, g, 9);
                tc_fence_after();
                const uint64_t a2 = f2(alpha, alpha);
#pragma unroll 1
                for (int c = 0; ok && c < 4; ++c) {
                  uint32_t r[16];
                  tmem_ld16(tO + 16u * c, r);
                  tc_wait_ld();
                  reg_fence16(r);
#pragma unroll
                  for (int e = 0; e < 16; e += 2) {
                    const float2 y = f2split(fmul2(f2u(r[e], r[e + 1]), a2));
                    r[e] = __float_as_uint(y.x);
                    r[e + 1] = __float_as_uint(y.y);
                  }
                  tmem_st16(tO + 16u * c, r);
                }
              }
              if (grow) {
                const uint64_t a2 = f2(alpha, alpha);
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                  acc_l[i] = fmul2(acc_l[i], a2);
                  acc_lr[i] = fmul2(acc_lr[i], a2);
                }
                m = m_new;
              }
            }
          }
          if (ok) {
            const float mu = (m == -INFINITY) ? 0.f : m;
            const uint64_t nmu2 = f2(-mu, -mu);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              uint32_t pk[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const uint64_t x2 = ffma2(f2u(sr[c][2 * e], sr[c][2 * e + 1]), sl2x2, nmu2);
                float p0, p1;
                if ((e & 3) == kExp2FmaPhase) {
                  // a quarter of the exponentials on the FMA pipe (the MUFU pipe is the
                  // softmax's bottleneck)
                  const float2 pe = f2split(exp2_fma2(x2));
                  p0 = pe.x;
                  p1 = pe.y;
                } else {
                  const float2 xx = f2split(x2);
                  p0 = ex2(xx.x);
                  p1 = ex2(xx.y);
                }
                const uint32_t v = pack_bf16(p0, p1);
                acc_l[e & 1] = fadd2(acc_l[e & 1], f2(p0, p1));
                acc_lr[e & 1] = fadd2(acc_lr[e & 1], bf16x2_to_f2(v));
                pk[e] = v;
              }
              tmem_st16(tS + 16u * c, pk);
            }
          }
        }
        if (ok) {
          tc_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(b ? lead_p1 : lead_p0);
        }
        if (j == I.j_lo && pk_ >= 0) epilogue(pk_, pm, pl, plr, prow, pbh);
      }
      float l = 0.f, lr = 0.f;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float2 a = f2split(acc_l[i]), bq = f2split(acc_lr[i]);
        l += a.x + a.y;
        lr += bq.x + bq.y;
      }
      pk_ = k_;
      pm = m;
      pl = l;
      plr = lr;
      prow = row;
      pbh = I.bh;
    }
    if (pk_ >= 0) epilogue(pk_, pm, pl, plr, prow, pbh);
  }

  tc_fence_before();
  cluster_sync_all();  // every copy of both CTAs issued, every MMA completed
  if (leader && warp == 8 && lane == 0 && *abort_flag) {
    // an aborted run may leave copies in flight: rank 0's full barriers count both CTAs'
    // copies, so wait (bounded) for the larger of the two counts on each of them
    const volatile int* c = reinterpret_cast<const volatile int*>(gsm + L::CNT_OFF);
    const int nq = max(c[0], c[3]), gk = max(c[1], c[4]), gv = max(c[2], c[5]);
    for (int b = 0; b < 2; ++b) {
      const int n = nq > b ? (nq - b + 1) / 2 : 0;
      if (n > 0) drain_wait(q_full(b), (n - 1) & 1, p.wait_limit_ns);
    }
    for (int s = 0; s < NK; ++s) {
      const int n = gk > s ? (gk - s + NK - 1) / NK : 0;
      if (n > 0) drain_wait(k_full(s), (n - 1) & 1, p.wait_limit_ns);
    }
    for (int s = 0; s < NV; ++s) {
      const int n = gv > s ? (gv - s + NV - 1) / NV : 0;
      if (n > 0) drain_wait(v_full(s), (n - 1) & 1, p.wait_limit_ns);
    }
  }
  cluster_sync_all();  // both CTAs done with TMEM, with rank 0's barriers and with the copies
  if (warp == 9) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(L::TMEM_COLS)
                 : "memory");
  }
}

}  // namespace ca
