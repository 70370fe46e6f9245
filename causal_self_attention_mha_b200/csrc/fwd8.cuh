// fwd8.cuh -- FP8 (e4m3) causal attention forward on sm_100a.
//
// "How to build an LLM by hand" (agmtopy.github.io), section 5, item 4: the
// in-house FP8 training runs the forward matmuls with e4m3 operands (through
// torch._scaled_mm, one fixed scale per tensor).  Applied to the attention
// forward of "Stanford CS336 walkthrough" (lmnt.cn), section 5.1, both of its
// products take e4m3 operands:
//   S = scale * dq * dk * Q8 K8^T            (Q8, K8: e4m3 codes, dq, dk: descales)
//   r = exp(S - rowmax S)                    (in (0, 1], exact softmax numerators)
//   W8 = e4m3(2^8 r)                         (the weights, rounded to e4m3)
//   O = dv * (W8 V8) / rowsum(W8),  LSE = rowmax S + log rowsum(r)   (natural log)
// with the causal / document / window masks of the bf16 kernel.  The weights are
// rounded relative to the row's FINAL maximum, so every item makes two passes
// over its key tiles: pass 1 forms S and keeps only the row maxima; pass 2 forms
// S again, the weights, their e4m3 codes (written to TMEM as the A operand of the
// second product) and O.  No running-maximum rescaling exists.
//
// Same persistent schedule, warp roles and TMEM map as attn_fwd_kernel (fwd.cuh):
// an item is a pair of adjacent 128-row query tiles (A, B) of one head; warps
// 0-3 / 4-7 own the rows of A / B (one thread per row), warp 8 loads (lane 0: Q
// and the K ring, which runs through every item's key tiles twice; lane 1: the V
// ring, pass 2 only), warp 9 issues the tcgen05.mma (kind::f8f6f4, K = 32 per
// instruction), warp 10 stores O.  TMEM: S_A at 0, S_B at 128 (the weight codes
// overwrite the first 32 columns of their own S), O_A at 256, O_B at 256 + D.
// O leaves through a dedicated staging tile (bf16) and TMA stores.
#pragma once

#include "fwd.cuh"

namespace ca {

// One 128-row tile of e4m3 codes: D bytes per row, a single swizzle chunk
// (128-byte swizzle for D = 128, 64-byte for 64, 32-byte for 32).
template <int D>
struct Tile8 {
  static_assert(D == 32 || D == 64 || D == 128, "head dim");
  static constexpr int SW = D;                  // swizzle span = bytes per row
  static constexpr int BYTES = kRows * D;
  static constexpr uint32_t LAYOUT = (SW == 128) ? 2u : (SW == 64 ? 4u : 6u);
};

// K-major operand for MMA-K step kk (32 e4m3 = 32 bytes of the row).
template <int D>
__device__ __forceinline__ uint64_t desc_k8(uint32_t tile, int kk) {
  return sdesc(tile + (uint32_t)kk * 32u, 16u, 8u * Tile8<D>::SW, Tile8<D>::LAYOUT);
}

// MN-major operand (contraction over the tile's rows, N along d) for MMA-K step kk (32 rows).
template <int D>
__device__ __forceinline__ uint64_t desc_mn8(uint32_t tile, int kk) {
  return sdesc(tile + (uint32_t)kk * 32u * Tile8<D>::SW, (uint32_t)Tile8<D>::BYTES,
               8u * Tile8<D>::SW, Tile8<D>::LAYOUT);
}

template <int D>
__device__ __forceinline__ void load_tile8(uint32_t dst, const CUtensorMap* m, int row0, int bh,
                                           uint32_t bar) {
  tma_load_3d(dst, m, 0, row0, bh, bar);
}

struct Fwd8Params {
  FwdParams f;          // geometry, masks, outputs (f.scale_log2 = scale * dq * dk * log2 e)
  float descale_v;      // O = descale_v * (W8 V8) / rowsum(W8)
};

template <int D>
struct Fwd8Layout {
  static constexpr int STK = 4;                              // K ring depth
  static constexpr int STV = 3;                              // V ring depth
  static constexpr int Q_OFF = 0;                            // Q_A, Q_B
  static constexpr int K_OFF = Q_OFF + 2 * Tile8<D>::BYTES;
  static constexpr int V_OFF = K_OFF + STK * Tile8<D>::BYTES;
  static constexpr int STG_OFF = V_OFF + STV * Tile8<D>::BYTES;  // bf16 O staging tile
  static constexpr int BAR_OFF = STG_OFF + Tile<D>::BYTES;
  // barriers: q_full[2] q_empty[2] k_full[STK] k_empty[STK] v_full[STV] v_empty[STV]
  //           s_full[2] s_free[2] p_full[2] o_done[2] o_free[2] drain stg_full stg_free
  static constexpr int NBAR = 4 + 2 * STK + 2 * STV + 10 + 3;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;       // tmem base slot, abort flag
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int SMEM = BYTES + 1024;                  // + alignment slack
  static_assert(SMEM <= kMaxDynSmem, "FP8 forward shared-memory layout");
  static constexpr int SOFTMAX_WARPS = 8;
  static constexpr int THREADS = 384;
  static constexpr uint32_t TMEM_COLS = 512;
};

template <int D>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                        const Fwd8Params p8) {
  using T8 = Tile8<D>;
  using L = Fwd8Layout<D>;
  const FwdParams& p = p8.f;
  constexpr int STK = L::STK, STV = L::STV;
  constexpr int kProducerWarp = L::SOFTMAX_WARPS, kMmaWarp = L::SOFTMAX_WARPS + 1;
  constexpr int kStoreWarp = L::SOFTMAX_WARPS + 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* gsm;
  const uint32_t sbase = aligned_smem_base(smem_raw, &gsm);
  if (sbase - smem_u32(smem_raw) + L::BYTES > dynamic_smem_bytes()) {
    if (threadIdx.x == 0) report_smem_shortfall();
    return;  // uniform across the CTA, before any barrier
  }
  const uint32_t sQ = sbase + L::Q_OFF, sK = sbase + L::K_OFF, sV = sbase + L::V_OFF;
  const uint32_t sStg = sbase + L::STG_OFF;
  const uint32_t bar0 = sbase + L::BAR_OFF;
  auto q_full = [&](int x) { return bar0 + 8u * x; };
  auto q_empty = [&](int x) { return bar0 + 8u * (2 + x); };
  auto k_full = [&](int s) { return bar0 + 8u * (4 + s); };
  auto k_empty = [&](int s) { return bar0 + 8u * (4 + STK + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (4 + 2 * STK + s); };
  auto v_empty = [&](int s) { return bar0 + 8u * (4 + 2 * STK + STV + s); };
  const uint32_t xb = bar0 + 8u * (4 + 2 * STK + 2 * STV);
  auto s_full = [&](int x) { return xb + 8u * x; };         // an S MMA of tile x completed
  auto s_free = [&](int x) { return xb + 8u * (2 + x); };   // pass 1: S_x has been read
  auto p_full = [&](int x) { return xb + 8u * (4 + x); };   // pass 2: weights of tile x in TMEM
  auto o_done = [&](int x) { return xb + 8u * (6 + x); };
  auto o_free = [&](int x) { return xb + 8u * (8 + x); };
  const uint32_t drain = xb + 8u * 10;
  const uint32_t stg_full = xb + 8u * 11, stg_free = xb + 8u * 12;
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
      mbar_init(s_free(x), 4);
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
    regs_shrink<88>();
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {  // Q_A, Q_B and the K ring (each item's key tiles twice)
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      int nq[2] = {0, 0};
      int gk = 0;
      bool ok = true;
      for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;
        const FwdItem I = fwd_item(p, w);
        for (int x = 0; x < 2; ++x) {
          if (x == 1 && !I.hasB) continue;
          if (nq[x] >= 1 && !wait_bounded(q_empty(x), (nq[x] - 1) & 1, g, 1)) { ok = false; break; }
          mbar_arrive_expect_tx(q_full(x), T8::BYTES);
          load_tile8<D>(sQ + x * T8::BYTES, &tmQ, I.qt[x] * kRows, I.bh, q_full(x));
          ++nq[x];
        }
        for (int pass = 0; ok && pass < 2; ++pass) {
          for (int j = I.j_lo; j <= I.j_hi; ++j) {
            const int s = gk % STK, u = gk / STK;
            if (u > 0 && !wait_bounded(k_empty(s), (u - 1) & 1, g, 1)) { ok = false; break; }
            mbar_arrive_expect_tx(k_full(s), T8::BYTES);
            load_tile8<D>(sK + s * T8::BYTES, &tmK, j * kRows, I.bh, k_full(s));
            ++gk;
          }
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
    } else if (lane == 1) {  // the V ring (pass 2)
      tma_prefetch_desc(&tmV);
      int gv = 0;
      bool ok = true;
      for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;
        const FwdItem I = fwd_item(p, w);
        for (int j = I.j_lo; j <= I.j_hi; ++j) {
          const int s = gv % STV, u = gv / STV;
          if (u > 0 && !wait_bounded(v_empty(s), (u - 1) & 1, g, 1)) { ok = false; break; }
          mbar_arrive_expect_tx(v_full(s), T8::BYTES);
          load_tile8<D>(sV + s * T8::BYTES, &tmV, j * kRows, I.bh, v_full(s));
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
      constexpr uint32_t kIdS = idesc_e4m3_f32(128, 128, false);
      constexpr uint32_t kIdO = idesc_e4m3_f32(128, D, true);
      int nq[2] = {0, 0};   // items started per query tile slot
      int nf[2] = {0, 0};   // pass-1 tiles per slot (s_free phases)
      int np[2] = {0, 0};   // pass-2 tiles per slot (p_full / o_done phases)
      int gk = 0, gv = 0;
      bool ok = true;
      // S_x = Q_x K^T for the K ring element gk
      auto issue_s = [&](int x, int sk) {
        tc_fence_after();
        const uint32_t tS = tmem + 128u * x;
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          mma_ss_f8(tS, desc_k8<D>(sQ + x * T8::BYTES, kk), desc_k8<D>(sK + sk * T8::BYTES, kk),
                    kIdS, kk > 0);
        tc_commit(s_full(x));
      };
      // pending PV of slot x (pass 2): weights of tile np[x]-1 against the V ring element pend_v
      int pend_v[2] = {-1, -1};
      bool pend_first[2] = {false, false}, pend_rel[2] = {false, false};
      auto issue_pv = [&](int x) -> bool {
        if (pend_first[x] && nq[x] >= 2 && !wait_bounded(o_free(x), (nq[x] - 2) & 1, g, 4))
          return false;  // the previous item's epilogue must have read O_x
        if (!wait_bounded(p_full(x), (np[x] - 1) & 1, g, 5)) return false;
        const int sv = pend_v[x] % STV;
        if (!wait_bounded(v_full(sv), (pend_v[x] / STV) & 1, g, 6)) return false;
        tc_fence_after();
        const uint32_t sVs = sV + sv * T8::BYTES;
        const uint32_t tP = tmem + 128u * x, tO = tmem + 256u + x * D;
#pragma unroll
        for (int kk = 0; kk < kRows / 32; ++kk)
          mma_ts_f8(tO, tP + 8u * kk, desc_mn8<D>(sVs, kk), kIdO, (!pend_first[x] || kk > 0));
        tc_commit(o_done(x));
        if (pend_rel[x]) tc_commit(v_empty(sv));
        pend_v[x] = -1;
        return true;
      };
      for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;
        const FwdItem I = fwd_item(p, w);
        for (int x = 0; x < 2; ++x) {
          if (x == 1 && !I.hasB) continue;
          if (!wait_bounded(q_full(x), nq[x] & 1, g, 2)) { ok = false; break; }
          ++nq[x];
        }
        // ---- pass 1: S only; S_x may be overwritten once its rows have been read
        for (int j = I.j_lo; ok && j <= I.j_hi; ++j, ++gk) {
          const int sk = gk % STK;
          if (!wait_bounded(k_full(sk), (gk / STK) & 1, g, 3)) { ok = false; break; }
          for (int x = 0; x < 2; ++x) {
            const bool act = (x == 0) ? (j <= I.hi[0]) : (I.hasB && j >= I.lo[1] && j <= I.hi[1]);
            if (!act) continue;
            // the previous S of this slot (pass 1 of this item, or the previous item's last
            // pass-2 tile, whose weights its PV has consumed in stream order) has been read
            if (nf[x] > 0 && !wait_bounded(s_free(x), (nf[x] - 1) & 1, g, 7)) { ok = false; break; }
            issue_s(x, sk);
            ++nf[x];
          }
          if (!ok) break;
          tc_commit(k_empty(sk));
        }
        // ---- pass 2: S again, weights, PV
        for (int j = I.j_lo; ok && j <= I.j_hi; ++j, ++gk, ++gv) {
          const int sk = gk % STK;
          if (!wait_bounded(k_full(sk), (gk / STK) & 1, g, 3)) { ok = false; break; }
          const bool actB = I.hasB && j >= I.lo[1] && j <= I.hi[1];
          auto step = [&](int x, bool act) -> bool {
            if (pend_v[x] >= 0 && !issue_pv(x)) return false;
            if (!act) return true;
            // the first pass-2 S of the slot overwrites the last pass-1 S: read by now?
            if (j == I.lo[x] && !wait_bounded(s_free(x), (nf[x] - 1) & 1, g, 7)) return false;
            issue_s(x, sk);
            if (j == I.hi[x]) tc_commit(q_empty(x));  // last S of this query tile
            ++np[x];
            pend_v[x] = gv;
            pend_first[x] = (j == I.lo[x]);
            pend_rel[x] = (x == 1) || !actB;  // the last PV to read V_j releases it
            return true;
          };
          if (!step(0, j <= I.hi[0]) || !step(1, actB)) { ok = false; break; }
          tc_commit(k_empty(sk));
        }
        if (ok && pend_v[0] >= 0 && !issue_pv(0)) ok = false;
        if (ok && pend_v[1] >= 0 && !issue_pv(1)) ok = false;
      }
      tc_commit(drain);
      drain_wait(drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else if (warp == kStoreWarp) {
    // ------------------------------------------------------------- O stores
    if (lane == 0) {
      tma_prefetch_desc(&tmO);
      int u = 0;  // staging uses so far
      bool ok = true;
      for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;
        const FwdItem I = fwd_item(p, w);
        for (int x = 0; x < (I.hasB ? 2 : 1); ++x, ++u) {
          if (!wait_bounded(stg_full, u & 1, g, 11)) { ok = false; break; }
          store_tile<D>(&tmO, sStg, I.qt[x] * kRows, I.bh);
          bulk_commit();
          bulk_wait_read_all();  // the staging tile may be overwritten from here on
          mbar_arrive(stg_free);
        }
      }
      bulk_wait_all();
    }
    __syncwarp();
  }
  } else {
    regs_grow<208>();
    // ------------------------------------------------------ softmax warps
    const int x = warp >> 2;                // 0: tile A, 1: tile B
    const int rl = (warp & 3) * 32 + lane;  // row within the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + 128u * x;
    const uint32_t tO = tmem + lane_off + 256u + x * D;
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2(sl2, sl2);
    bool ok = true;
    int ts = 0;   // S tiles of this slot read so far (s_full phases)
    int tp = 0;   // pass-2 tiles (o_done phases)
    int u0 = 0;   // staging uses before this item
    for (int k_ = 0; k_ * dw < p.n_items; ++k_) {
      const int w = snake_item(k_, w0, dw, p.n_items);
      if (w < 0) break;
      const FwdItem I = fwd_item(p, w);
      const int u = u0 + x;
      u0 += I.hasB ? 2 : 1;
      if (x == 1 && !I.hasB) continue;
      if (!ok) continue;
      const int row = I.qt[x] * kRows + rl;
      int ds = p.doc ? ld_chk(p.doc, (size_t)I.b * T + (row < T ? row : T - 1),
                              (size_t)(p.BH / p.H) * T)
                     : 0;
      ds = ds > row - p.window + 1 ? ds : row - p.window + 1;
      const int n = I.hi[x] - I.lo[x] + 1;
      // S of this thread's row for key tile c0, masked; returns false on a failed wait
      uint32_t sr[4][32];
      auto load_s = [&](int c0) -> bool {
        if (!wait_bounded_warp(s_full(x), ts & 1, g, 8)) return false;
        ++ts;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32u * c, sr[c]);
        tc_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) reg_fence(sr[c]);
        if (!((c0 + kRows - 1 <= row) && (c0 >= ds))) {
          const int hi = row - c0, lo = ds - c0;  // visible keys: e in [lo, hi]
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (e > hi || e < lo) sr[e >> 5][e & 31] = 0xFF800000u;  // -inf
        }
        return true;
      };
      // ---- pass 1: the row maximum (of the scaled scores, base 2)
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      for (int it = 0; it < n; ++it) {
        if (!load_s((I.lo[x] + it) * kRows)) { ok = false; break; }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free(x));  // S_x is in registers
#pragma unroll
        for (int e = 0; e < 128; e += 8)
#pragma unroll
          for (int q = 0; q < 4; ++q)
            mx4[q] = fmax3(mx4[q], __uint_as_float(sr[(e + 2 * q) >> 5][(e + 2 * q) & 31]),
                           __uint_as_float(sr[(e + 2 * q + 1) >> 5][(e + 2 * q + 1) & 31]));
      }
      if (!ok) continue;
      const float m = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * sl2;
      // ---- pass 2: weights 2^8 * exp(S - m) (exp2 of the base-2 exponent + 8), their e4m3
      // codes to TMEM; acc_l sums the weights before rounding (for the LSE), acc_q after
      const uint64_t nmu2 = f2(8.0f - m, 8.0f - m);
      uint64_t acc_l[4];
      float acc_q[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 4; ++i) acc_l[i] = f2(0.f, 0.f);
      for (int it = 0; it < n; ++it, ++tp) {
        if (!load_s((I.lo[x] + it) * kRows)) { ok = false; break; }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 a = f2split(ffma2(f2u(sr[c][4 * e], sr[c][4 * e + 1]), sl2x2, nmu2));
            const float2 b = f2split(ffma2(f2u(sr[c][4 * e + 2], sr[c][4 * e + 3]), sl2x2, nmu2));
            const float p0 = ex2(a.x), p1 = ex2(a.y), p2 = ex2(b.x), p3 = ex2(b.y);
            const uint32_t v = pack_e4m3x4(p0, p1, p2, p3);
            acc_l[e & 3] = fadd2(acc_l[e & 3], fadd2(f2(p0, p1), f2(p2, p3)));
            add_e4m3x4(v, acc_q[0], acc_q[1], acc_q[2], acc_q[3]);
            pk[e] = v;
          }
          tmem_st8(tS + 8u * c, pk);
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(x));
      }
      if (!ok) continue;
      // ---------------------------------------------------------- epilogue
      if (wait_bounded_warp(o_done(x), (tp - 1) & 1, g, 10)) {
        tc_fence_after();
        float l = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 a = f2split(acc_l[i]);
          l += a.x + a.y;
        }
        const float lq = (acc_q[0] + acc_q[1]) + (acc_q[2] + acc_q[3]);
        // l sums 2^8 * exp(S - m): LSE = m + log2(l) - 8, in base 2, to natural log
        if (row < T)
          st_chk(p.lse, (size_t)I.bh * T + row, (size_t)p.BH * T, (m + lg2(l) - 8.0f) * kLn2);
        const float mul = p8.descale_v / lq;
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
              wo[32 * w2 + 16 * c + e] = pack_bf16(__uint_as_float(r[c][2 * e]) * mul,
                                                   __uint_as_float(r[c][2 * e + 1]) * mul);
        }
        // O_x has been read: the next item's first PV may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free(x));
        // stage the row once the store of the previous staging use has read the tile
        if (u > 0 && !wait_bounded_warp(stg_free, (u - 1) & 1, g, 13)) {
          ok = false;
        } else {
          stage_row<D>(gsm + L::STG_OFF, rl, 0, wo);
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
