// fwd.cuh -- causal attention forward on sm_100a.
//
// Computes, for every head and 128-row query tile,
//   S = scale * Q K^T  (upper triangle and other documents masked to -inf),
//   P = softmax(S) row-wise,  O = P V,  LSE = log sum exp(S)  (natural log)
// as in "Stanford CS336 walkthrough" (lmnt.cn), section 5.1 model.py,
// CausalSelfAttention.forward, and section 3.3 (masked weights are zero after
// the softmax).  The softmax is evaluated online over 128-column key tiles
// (running max m and sums, in base 2), so the T x T matrix never exists.
//
// Persistent kernel: one CTA per SM walks work items w = blockIdx.x,
// blockIdx.x + gridDim.x, ...  An item is a PAIR of adjacent 128-row query
// tiles (A = 2m, B = 2m+1) of one head, so every K/V tile brought on chip
// serves 256 query rows.  Items are numbered heaviest first.  All roles walk
// the same item / key-tile sequence; the K/V rings run on across items.
//
// Warp roles (384 threads = three warpgroups):
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: one thread per
//              query row (= TMEM lane), so row max and sums are in-thread
//   warp 8     TMA producer: lane 0 loads Q_A, Q_B and the K ring, lane 1 the V ring
//   warp 9     TMEM allocator and single-thread tcgen05.mma issuer
//   warp 10    TMA stores of O
//   warp 11    idle
// Registers: launched at 168 per thread; the third warpgroup drops to 88 and
// the two softmax warpgroups rise to 208 (2*128*208 + 128*88 = 384*168), room
// for a whole 128-column row of S in registers.
// TMEM (512 columns): S_A at 0, S_B at 128 (P, packed bf16, overwrites the
// first 64 columns of its own S), O_A at 256, O_B at 256 + D.
//
// MMA order per key tile j: PV_A(j-1), S_A(j), PV_B(j-1), S_B(j).  Each tile's
// chain alternates softmax and MMA; the two chains run half a period apart,
// so the tensor pipe works on one tile while the other tile's softmax runs.
// S_X(j) overwrites P_X(j-1) only after PV_X(j-1) in the same in-order MMA
// stream.  A K slot is released once both S MMAs that read it are done, a V
// slot after its last PV.  O_X is rescaled in TMEM only when a row max grows
// by more than 2^8.  Normalisation uses the sum of the bf16-rounded weights
// the MMA actually multiplied (the weights of each output row sum to one);
// the LSE uses the sum of the fp32 weights.
//
// O leaves through TMA stores of a staged bf16 tile: after an item's key tiles
// the producer hands the next K-ring slot to the epilogue instead of loading
// it; O_A and then O_B are staged there in turn, and the store warp returns the
// slot once the last store has read it.  Row-per-thread global stores from
// every SM at the same item boundary congest the memory system.
#pragma once

#include "tiles.cuh"

namespace ca {

struct FwdParams {
  const int32_t* doc;     // [B, T] document start of each position, or nullptr
  __nv_bfloat16* o;       // [B, H, T, D]
  float* lse;             // [B, H, T]
  int H, T, BH, n_qt, n_pairs, n_items;
  int window;             // keys a query sees, itself included (T: no window)
  float scale_log2;       // scale * log2(e)
  uint64_t wait_limit_ns;
};

template <int D>
struct FwdLayout {
  static constexpr int STK = (D == 128) ? 3 : 4;            // K ring depth
  static constexpr int STV = (D == 128) ? 2 : 3;            // V ring depth
  static constexpr int Q_OFF = 0;                            // Q_A, Q_B
  static constexpr int K_OFF = Q_OFF + 2 * Tile<D>::BYTES;
  static constexpr int V_OFF = K_OFF + STK * Tile<D>::BYTES;
  static constexpr int BAR_OFF = V_OFF + STV * Tile<D>::BYTES;
  // barriers: q_full[2] q_empty[2] k_full[STK] k_empty[STK] v_full[STV] v_empty[STV]
  //           s_full[2] p_full[2] o_done[2] o_free[2] drain stg_full stg_free
  static constexpr int NBAR = 4 + 2 * STK + 2 * STV + 8 + 3;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;       // tmem base slot, abort flag
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int SMEM = BYTES + 1024;                  // + alignment slack
  static constexpr int SOFTMAX_WARPS = 8;
  static constexpr int THREADS = 384;
  static constexpr uint32_t TMEM_COLS = 512;
};

// One work item: query tiles A = 2*pm and B = 2*pm + 1 of head bh.
struct FwdItem {
  int bh, b;
  int qt[2];       // query tile of A and B
  bool hasB;       // B lies (at least partly) inside T
  int j_lo, j_hi;  // key tiles streamed for the pair
  int lo[2];       // first key tile each of A / B needs (A: j_lo; B: >= j_lo)
  int hi[2];       // last key tile each needs (its diagonal)
};

__device__ __forceinline__ FwdItem fwd_item(const FwdParams& p, int w) {
  FwdItem I;
  const int pm = p.n_pairs - 1 - w / p.BH;  // heaviest pairs first
  I.bh = w % p.BH;
  I.b = I.bh / p.H;
  I.qt[0] = 2 * pm;
  I.qt[1] = 2 * pm + 1;
  I.hasB = I.qt[1] < p.n_qt;
  for (int x = 0; x < 2; ++x) {
    int lo = 0;
    if (x == 0 || I.hasB) {
      // the first key any row of the tile sees: its first row's window / document start
      const int q0 = I.qt[x] * kRows;
      int first = q0 - p.window + 1;
      if (p.doc) {
        const int ds = ld_chk(p.doc, (size_t)I.b * p.T + q0, (size_t)(p.BH / p.H) * p.T);
        first = first > ds ? first : ds;
      }
      lo = first < 0 ? 0 : first / kRows;
      lo = lo > I.qt[x] ? I.qt[x] : lo;
    }
    I.lo[x] = lo;
    I.hi[x] = I.qt[x];
  }
  if (I.lo[1] < I.lo[0]) I.lo[1] = I.lo[0];
  I.j_lo = I.lo[0];
  I.j_hi = I.hasB ? I.hi[1] : I.hi[0];
  return I;
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const FwdParams p) {
  using Tl = Tile<D>;
  using L = FwdLayout<D>;
  constexpr int STK = L::STK, STV = L::STV;
  constexpr int kProducerWarp = L::SOFTMAX_WARPS, kMmaWarp = L::SOFTMAX_WARPS + 1;
  constexpr int kStoreWarp = L::SOFTMAX_WARPS + 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* gsm;
  const uint32_t sbase = aligned_smem_base(smem_raw, &gsm);
  const uint32_t sQ = sbase + L::Q_OFF, sK = sbase + L::K_OFF, sV = sbase + L::V_OFF;
  const uint32_t bar0 = sbase + L::BAR_OFF;
  auto q_full = [&](int x) { return bar0 + 8u * x; };
  auto q_empty = [&](int x) { return bar0 + 8u * (2 + x); };
  auto k_full = [&](int s) { return bar0 + 8u * (4 + s); };
  auto k_empty = [&](int s) { return bar0 + 8u * (4 + STK + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (4 + 2 * STK + s); };
  auto v_empty = [&](int s) { return bar0 + 8u * (4 + 2 * STK + STV + s); };
  const uint32_t xb = bar0 + 8u * (4 + 2 * STK + 2 * STV);
  auto s_full = [&](int x) { return xb + 8u * x; };
  auto p_full = [&](int x) { return xb + 8u * (2 + x); };
  auto o_done = [&](int x) { return xb + 8u * (4 + x); };
  auto o_free = [&](int x) { return xb + 8u * (6 + x); };
  const uint32_t drain = xb + 8u * 8;
  // staging use u (O_A, then O_B, of each item in turn) is complete / has been read
  const uint32_t stg_full = xb + 8u * 9, stg_free = xb + 8u * 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gsm + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gsm + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  const int w0 = blockIdx.x, dw = gridDim.x;

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(q_full(x), 1);
      mbar_init(q_empty(x), 1);
      mbar_init(s_full(x), 1);
      mbar_init(p_full(x), 4);
      mbar_init(o_done(x), 1);
      mbar_init(o_free(x), 4);
    }
    for (int s = 0; s < STK; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
    }
    for (int s = 0; s < STV; ++s) {
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    mbar_init(drain, 1);
    mbar_init(stg_full, 4);
    mbar_init(stg_free, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Guard g{abort_flag, p.wait_limit_ns};
  if (warp >= L::SOFTMAX_WARPS) {
    // third warpgroup: give registers to the softmax warpgroups, then specialise
    regs_shrink<88>();
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {  // Q_A, Q_B and the K ring
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      int nq[2] = {0, 0};  // Q loads issued into buffer A / B
      int gk = 0;          // K loads issued
      bool ok = true;
      for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;  // past the last item: no later round has one either
        const FwdItem I = fwd_item(p, w);
        for (int x = 0; x < 2; ++x) {
          if (x == 1 && !I.hasB) continue;
          if (nq[x] >= 1 && !wait_bounded(q_empty(x), (nq[x] - 1) & 1, g, 1)) { ok = false; break; }
          mbar_arrive_expect_tx(q_full(x), Tl::BYTES);
          load_tile<D>(sQ + x * Tl::BYTES, &tmQ, I.qt[x] * kRows, I.bh, q_full(x));
          ++nq[x];
        }
        // the item's key tiles, then one more ring element: the slot that stages O
        for (int j = I.j_lo; ok && j <= I.j_hi + 1; ++j) {
          const int s = gk % STK, u = gk / STK;
          if (u > 0 && !wait_bounded(k_empty(s), (u - 1) & 1, g, 1)) { ok = false; break; }
          if (j <= I.j_hi) {
            mbar_arrive_expect_tx(k_full(s), Tl::BYTES);
            load_tile<D>(sK + s * Tl::BYTES, &tmK, j * kRows, I.bh, k_full(s));
          } else {
            mbar_arrive(k_full(s));  // hand the slot to the epilogue
          }
          ++gk;
        }
      }
      if (*abort_flag) {  // let every copy already issued land before the CTA exits
        for (int x = 0; x < 2; ++x)
          if (nq[x] > 0) drain_wait(q_full(x), (nq[x] - 1) & 1, p.wait_limit_ns);
        for (int s = 0; s < STK; ++s) {
          const int cnt = gk > s ? (gk - s + STK - 1) / STK : 0;
          if (cnt > 0) drain_wait(k_full(s), (cnt - 1) & 1, p.wait_limit_ns);
        }
      }
    } else if (lane == 1) {  // the V ring
      tma_prefetch_desc(&tmV);
      int gv = 0;
      bool ok = true;
      for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;  // past the last item: no later round has one either
        const FwdItem I = fwd_item(p, w);
        for (int j = I.j_lo; j <= I.j_hi; ++j) {
          const int s = gv % STV, u = gv / STV;
          if (u > 0 && !wait_bounded(v_empty(s), (u - 1) & 1, g, 1)) { ok = false; break; }
          mbar_arrive_expect_tx(v_full(s), Tl::BYTES);
          load_tile<D>(sV + s * Tl::BYTES, &tmV, j * kRows, I.bh, v_full(s));
          ++gv;
        }
      }
      if (*abort_flag) {
        for (int s = 0; s < STV; ++s) {
          const int cnt = gv > s ? (gv - s + STV - 1) / STV : 0;
          if (cnt > 0) drain_wait(v_full(s), (cnt - 1) & 1, p.wait_limit_ns);
        }
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t kIdO = idesc_bf16_f32(128, D, true);
      int nq[2] = {0, 0};   // items started per query tile slot (q_full phases)
      int tx[2] = {0, 0};   // S MMAs issued per slot (s_full / p_full / o_done phases)
      int gk = 0, gv = 0;   // key tiles consumed from the K / V rings
      bool ok = true;
      // pending PV of slot x: its global tile index, V slot, "first of item", "last user of V"
      int pend_t[2] = {-1, -1}, pend_v[2] = {0, 0};
      bool pend_first[2] = {false, false}, pend_rel[2] = {false, false};
      auto issue_pv = [&](int x) -> bool {
        const int tp = pend_t[x];
        if (pend_first[x] && nq[x] >= 2 && !wait_bounded_fast(o_free(x), (nq[x] - 2) & 1, g, 4))
          return false;  // the previous item's epilogue must have read O_x
        if (!wait_bounded_fast(p_full(x), tp & 1, g, 5)) return false;
        const int sv = pend_v[x] % STV;
        if (!wait_bounded_fast(v_full(sv), (pend_v[x] / STV) & 1, g, 6)) return false;
        tc_fence_after();
        const uint32_t sVs = sV + sv * Tl::BYTES;
        const uint32_t tP = tmem + 128u * x, tO = tmem + 256u + x * D;
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          mma_ts(tO, tP + 8u * kk, desc_mn<D>(sVs, kk), kIdO, (!pend_first[x] || kk > 0));
        tc_commit(o_done(x));
        if (pend_rel[x]) tc_commit(v_empty(sv));
        pend_t[x] = -1;
        return true;
      };
      for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;  // past the last item: no later round has one either
        const FwdItem I = fwd_item(p, w);
        // each slot's Q is waited for right before its first S: B's Q can only be loaded once
        // B's last S of the previous item has read the old one, a key tile later than A's
        for (int j = I.j_lo; ok && j <= I.j_hi; ++j, ++gk, ++gv) {
          const int sk = gk % STK;
          if (!wait_bounded_fast(k_full(sk), (gk / STK) & 1, g, 3)) { ok = false; break; }
          const bool actB = I.hasB && j >= I.lo[1] && j <= I.hi[1];
          // slot x: the pending PV of x (previous key tile), then S_x for this key tile
          auto step = [&](int x, bool act) -> bool {
            if (pend_t[x] >= 0 && !issue_pv(x)) return false;
            if (!act) return true;
            if (j == I.lo[x]) {  // first S of this query tile: its Q must have landed
              if (!wait_bounded_fast(q_full(x), nq[x] & 1, g, 2)) return false;
              ++nq[x];
            }
            tc_fence_after();
            const uint32_t tS = tmem + 128u * x;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tS, desc_k<D>(sQ + x * Tl::BYTES, kk), desc_k<D>(sK + sk * Tl::BYTES, kk),
                     kIdS, kk > 0);
            tc_commit(s_full(x));
            if (j == I.hi[x]) tc_commit(q_empty(x));  // last S of this query tile
            pend_t[x] = tx[x]++;
            pend_v[x] = gv;
            pend_first[x] = (j == I.lo[x]);
            pend_rel[x] = (x == 1) || !actB;  // the last PV to read V_j releases it
            return true;
          };
          if (!step(0, j <= I.hi[0]) || !step(1, actB)) { ok = false; break; }
          tc_commit(k_empty(sk));
        }
        if (ok && pend_t[0] >= 0 && !issue_pv(0)) ok = false;
        if (ok && pend_t[1] >= 0 && !issue_pv(1)) ok = false;
        ++gk;  // the ring element that stages O
      }
      tc_commit(drain);
      drain_wait(drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else if (warp == kStoreWarp) {
    // ------------------------------------------------------------- O stores
    if (lane == 0) {
      tma_prefetch_desc(&tmO);
      int gk = 0, u = 0;  // K-ring elements, staging uses so far
      bool ok = true;
      for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;  // past the last item: no later round has one either
        const FwdItem I = fwd_item(p, w);
        gk += I.j_hi - I.j_lo + 1;
        const uint32_t stage = sK + (gk % STK) * Tl::BYTES;
        for (int x = 0; x < (I.hasB ? 2 : 1); ++x, ++u) {
          if (!wait_bounded(stg_full, u & 1, g, 11)) { ok = false; break; }
          store_tile<D>(&tmO, stage, I.qt[x] * kRows, I.bh);
          bulk_commit();
          bulk_wait_read_all();  // the stage may be overwritten from here on
          mbar_arrive(stg_free);
          if (x == (I.hasB ? 1 : 0)) mbar_arrive(k_empty(gk % STK));  // back to the K ring
        }
        ++gk;
      }
      bulk_wait_all();
    }
    __syncwarp();
  }
  } else {
    regs_grow<208>();
    // ------------------------------------------------------ softmax warps
    const int x = warp >> 2;             // 0: tile A, 1: tile B
    const int rl = (warp & 3) * 32 + lane;  // row within the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + 128u * x;
    const uint32_t tO = tmem + lane_off + 256u + x * D;
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2(sl2, sl2);
    bool ok = true;
    int t = 0;   // tiles processed by this slot (s_full / p_full / o_done phases)
    int gk = 0, u0 = 0;  // K-ring elements and staging uses before this item
    for (int k_ = 0; k_ * dw < p.n_items; ++k_) {
      const int w = snake_item(k_, w0, dw, p.n_items);
      if (w < 0) break;  // past the last item: no later round has one either
      const FwdItem I = fwd_item(p, w);
      const int ks = gk + (I.j_hi - I.j_lo + 1);  // this item's staging element
      const int u = u0 + x;                        // this tile's staging use
      gk = ks + 1;
      u0 += I.hasB ? 2 : 1;
      if (x == 1 && !I.hasB) continue;
      const int row = I.qt[x] * kRows + rl;
      // first visible key of this row: its document start or the window's start
      int ds = p.doc ? ld_chk(p.doc, (size_t)I.b * T + (row < T ? row : T - 1),
                              (size_t)(p.BH / p.H) * T)
                     : 0;
      ds = ds > row - p.window + 1 ? ds : row - p.window + 1;
      float m = -INFINITY;
      // acc_l: sum of the fp32 weights (for the LSE); acc_lr: sum of the bf16-rounded weights
      // the PV MMA actually multiplies (for normalising O).  Packed pairs, independent chains.
      uint64_t acc_l[4], acc_lr[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc_l[i] = acc_lr[i] = f2(0.f, 0.f);
      const int n = I.hi[x] - I.lo[x] + 1;
      const int t_last = t + n - 1;
      for (int it = 0; ok && it < n; ++it, ++t) {
        const int c0 = (I.lo[x] + it) * kRows;  // first key of the tile
        if (!wait_bounded_warp(s_full(x), t & 1, g, 8)) { ok = false; break; }
        // s_full(t) also means PV(t-1) has completed: O_x may be read and rescaled
        tc_fence_after();
        // two load waves: the max over the first 64 columns overlaps the second wave
        uint32_t sr[4][32];
        tmem_ld32(tS, sr[0]);
        tmem_ld32(tS + 32u, sr[1]);
        tc_wait_ld();
        reg_fence(sr[0]);
        reg_fence(sr[1]);
        tmem_ld32(tS + 64u, sr[2]);
        tmem_ld32(tS + 96u, sr[3]);
        const bool need_mask = !((c0 + kRows - 1 <= row) && (c0 >= ds));
        const int hi = row - c0, lo = ds - c0;  // visible keys: e in [lo, hi]
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (half == 1) {
            tc_wait_ld();
            reg_fence(sr[2]);
            reg_fence(sr[3]);
          }
          if (need_mask) {
#pragma unroll
            for (int e = 64 * half; e < 64 * half + 64; ++e)
              if (e > hi || e < lo) sr[e >> 5][e & 31] = 0xFF800000u;  // -inf
          }
#pragma unroll
          for (int e = 64 * half; e < 64 * half + 64; e += 8)
#pragma unroll
            for (int q = 0; q < 4; ++q)
              mx4[q] = fmax3(mx4[q], __uint_as_float(sr[(e + 2 * q) >> 5][(e + 2 * q) & 31]),
                             __uint_as_float(sr[(e + 2 * q + 1) >> 5][(e + 2 * q + 1) & 31]));
        }
        const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * sl2;
        const float m_new = fmaxf(m, mx);
        const bool grow = m_new > m + 8.0f;  // also true the first time a row sees a key
        const float alpha = grow ? ex2(m - m_new) : 1.0f;
        if (it > 0 && __any_sync(0xffffffffu, grow)) {
          const uint64_t a2 = f2(alpha, alpha);
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
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
          for (int i = 0; i < 4; ++i) {
            acc_l[i] = fmul2(acc_l[i], a2);
            acc_lr[i] = fmul2(acc_lr[i], a2);
          }
          m = m_new;
        }
        const float mu = (m == -INFINITY) ? 0.f : m;
        const uint64_t nmu2 = f2(-mu, -mu);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 xx = f2split(ffma2(f2u(sr[c][2 * e], sr[c][2 * e + 1]), sl2x2, nmu2));
            const float p0 = ex2(xx.x), p1 = ex2(xx.y);
            const uint32_t v = pack_bf16(p0, p1);
            acc_l[e & 3] = fadd2(acc_l[e & 3], f2(p0, p1));
            acc_lr[e & 3] = fadd2(acc_lr[e & 3], bf16x2_to_f2(v));
            pk[e] = v;
          }
          tmem_st16(tS + 16u * c, pk);
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(x));
      }
      t = t_last + 1;
      // ---------------------------------------------------------- epilogue
      if (ok && wait_bounded_warp(o_done(x), t_last & 1, g, 10)) {
        tc_fence_after();
        float l = 0.f, lr = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 a = f2split(acc_l[i]), bq = f2split(acc_lr[i]);
          l += a.x + a.y;
          lr += bq.x + bq.y;
        }
        const float mu = (m == -INFINITY) ? 0.f : m;
        if (row < T) st_chk(p.lse, (size_t)I.bh * T + row, (size_t)p.BH * T, (mu + lg2(l)) * kLn2);
        const float inv = 1.0f / lr;
        // the row, normalised, as packed bf16: up to two waves of 64 columns, loads in flight together
        uint32_t wo[D / 2];
#pragma unroll
        for (int w2 = 0; w2 < (D + 63) / 64; ++w2) {
          constexpr int NC = (D >= 64) ? 2 : 1;
          uint32_t r[NC][32];
#pragma unroll
          for (int c = 0; c < NC; ++c) tmem_ld32(tO + 64u * w2 + 32u * c, r[c]);
          tc_wait_ld();
#pragma unroll
          for (int c = 0; c < NC; ++c) reg_fence(r[c]);
#pragma unroll
          for (int c = 0; c < NC; ++c)
#pragma unroll
            for (int e = 0; e < 16; ++e)
              wo[32 * w2 + 16 * c + e] = pack_bf16(__uint_as_float(r[c][2 * e]) * inv,
                                                   __uint_as_float(r[c][2 * e + 1]) * inv);
        }
        // O_x has been read: the next item's first PV may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free(x));
        // stage the row once the slot is ours (handed over by the producer) and the store of
        // the previous staging use has read it; rows past T are dropped by the store
        if (!wait_bounded_warp(k_full(ks % STK), (ks / STK) & 1, g, 12) ||
            (u > 0 && !wait_bounded_warp(stg_free, (u - 1) & 1, g, 13))) {
          ok = false;
        } else {
          stage_row<D>(gsm + L::K_OFF + (ks % STK) * Tl::BYTES, rl, 0, wo);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(stg_full);
        }
      } else {
        ok = false;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace ca
