// fwd.cuh -- causal attention forward on sm_100a.
//
// Computes, for one head and one 128-row query tile per CTA,
//   S = scale * Q K^T  (upper triangle and other documents masked to -inf),
//   P = softmax(S) row-wise,  O = P V,  LSE = log sum exp(S)  (natural log)
// as in "Stanford CS336 walkthrough" (lmnt.cn), section 5.1 model.py,
// CausalSelfAttention.forward, and section 3.3 (masked weights are zero after
// the softmax).  The softmax is evaluated online over 128-column key tiles
// (running max m and sum l, in base 2), so the T x T matrix never exists.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t of the tile (= TMEM lane t);
//              row max and row sum are in-thread, no shuffles needed
//   warp 4     TMA producer: Q once, then K/V tiles through an ST-stage ring
//   warp 5     TMEM allocator and single-thread tcgen05.mma issuer
// TMEM (512 columns): S double buffer at columns 0 and 128 (P, as packed bf16,
// overwrites the first 64 columns of its own S buffer), O accumulator at 256.
//
// Per key tile j the MMA issuer runs S_{j+1} = Q K_{j+1}^T while the softmax
// warps turn S_j into P_j; then O += P_j V_j with P_j read straight from TMEM.
// O is rescaled in TMEM only when a row max grows by more than 2^8 (the
// bound keeps unnormalised weights within bf16/fp32 range); the final
// normalisation by 1/l happens once, in fp32, before rounding to bf16.
#pragma once

#include "tiles.cuh"

namespace ca {

struct FwdParams {
  const int32_t* doc;     // [B, T] document start of each position, or nullptr
  __nv_bfloat16* o;       // [B, H, T, D]
  float* lse;             // [B, H, T]
  int H, T, BH, n_qt;
  float scale_log2;       // scale * log2(e)
  uint64_t wait_limit_ns;
};

template <int D>
struct FwdLayout {
  static constexpr int ST = (D == 128) ? 2 : 3;             // K/V ring depth
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + Tile<D>::BYTES;
  static constexpr int V_OFF = K_OFF + ST * Tile<D>::BYTES;
  static constexpr int BAR_OFF = V_OFF + ST * Tile<D>::BYTES;
  // barriers: q_full | k_full[ST] | v_full[ST] | kv_empty[ST] | s_full[2] | p_full | o_done | drain
  static constexpr int NBAR = 1 + 3 * ST + 2 + 3;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;       // tmem base slot, abort flag
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int SMEM = BYTES + 1024;                  // + alignment slack
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using Tl = Tile<D>;
  using L = FwdLayout<D>;
  constexpr int ST = L::ST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* gsm;
  const uint32_t sbase = aligned_smem_base(smem_raw, &gsm);
  const uint32_t sQ = sbase + L::Q_OFF, sK = sbase + L::K_OFF, sV = sbase + L::V_OFF;
  const uint32_t bar0 = sbase + L::BAR_OFF;
  const uint32_t q_full = bar0;
  auto k_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (1 + ST + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (1 + 2 * ST + s); };
  auto s_full = [&](int b) { return bar0 + 8u * (1 + 3 * ST + b); };
  const uint32_t p_full = bar0 + 8u * (3 + 3 * ST);
  const uint32_t o_done = bar0 + 8u * (4 + 3 * ST);
  const uint32_t drain = bar0 + 8u * (5 + 3 * ST);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gsm + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gsm + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  // Work item: heaviest query tiles (most key tiles) are launched first.
  const int qt = p.n_qt - 1 - (int)(blockIdx.x / p.BH);
  const int bh = (int)(blockIdx.x % p.BH);
  const int b = bh / p.H;
  const int q0 = qt * kRows;
  int kv_lo = 0;
  if (p.doc) {
    kv_lo = p.doc[(size_t)b * T + q0] / kRows;
    kv_lo = kv_lo < 0 ? 0 : (kv_lo > qt ? qt : kv_lo);
  }
  const int n = qt - kv_lo + 1;  // key tiles to visit (>= 1)

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(s_full(0), 1);
    mbar_init(s_full(1), 1);
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Guard g{abort_flag, p.wait_limit_ns};

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, Tl::BYTES);
      load_tile<D>(sQ, &tmQ, q0, bh, q_full);
      int it = 0;
      for (; it < n; ++it) {
        const int s = it % ST, u = it / ST;
        if (u > 0 && !wait_bounded(kv_empty(s), (u - 1) & 1, g, 1)) break;
        const int row = (kv_lo + it) * kRows;
        mbar_arrive_expect_tx(k_full(s), Tl::BYTES);
        load_tile<D>(sK + s * Tl::BYTES, &tmK, row, bh, k_full(s));
        mbar_arrive_expect_tx(v_full(s), Tl::BYTES);
        load_tile<D>(sV + s * Tl::BYTES, &tmV, row, bh, v_full(s));
      }
      if (*abort_flag) {  // let every copy already issued land before the CTA exits
        drain_wait(q_full, 0, p.wait_limit_ns);
        for (int s = 0; s < ST; ++s) {
          const int cnt = it > s ? (it - s + ST - 1) / ST : 0;
          if (cnt > 0) {
            drain_wait(k_full(s), (cnt - 1) & 1, p.wait_limit_ns);
            drain_wait(v_full(s), (cnt - 1) & 1, p.wait_limit_ns);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t kIdO = idesc_bf16_f32(128, D, true);
      const uint32_t tO = tmem + 256;
      auto issue_s = [&](int it) -> bool {
        const int s = it % ST;
        if (!wait_bounded(k_full(s), (it / ST) & 1, g, 3)) return false;
        tc_fence_after();
        const uint32_t tS = tmem + 128u * (it & 1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tS, desc_k<D>(sQ, kk), desc_k<D>(sK + s * Tl::BYTES, kk), kIdS, kk > 0);
        tc_commit(s_full(it & 1));
        return true;
      };
      bool ok = wait_bounded(q_full, 0, g, 2) && issue_s(0);
      for (int it = 0; ok && it < n; ++it) {
        const int s = it % ST;
        if (it + 1 < n) {
          // S_{it+1} reuses the TMEM buffer that held P_{it-1}: PV_{it-1} must be done with it.
          if (it >= 1 && !wait_bounded(o_done, (it - 1) & 1, g, 4)) break;
          if (!issue_s(it + 1)) break;
        }
        if (!wait_bounded(p_full, it & 1, g, 5)) break;
        if (!wait_bounded(v_full(s), (it / ST) & 1, g, 6)) break;
        tc_fence_after();
        const uint32_t tP = tmem + 128u * (it & 1);
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          mma_ts(tO, tP + 8u * kk, desc_mn<D>(sV + s * Tl::BYTES, kk), kIdO, (it > 0 || kk > 0));
        tc_commit(o_done);
        tc_commit(kv_empty(s));
      }
      tc_commit(drain);
      drain_wait(drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ softmax warps
    const int t = threadIdx.x;  // row within the tile == TMEM lane
    const int row = q0 + t;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const int ds = p.doc ? p.doc[(size_t)b * T + (row < T ? row : T - 1)] : 0;
    const float sl2 = p.scale_log2;
    // l: sum of the fp32 weights (for the LSE); lr: sum of the bf16-rounded weights that the
    // PV MMA actually multiplies (for normalising O, so its weights sum to one exactly)
    float m = -INFINITY, l = 0.f, lr = 0.f;
    bool ok = true;
    for (int it = 0; it < n; ++it) {
      const int j = kv_lo + it;
      const uint32_t tS = tmem + lane_off + 128u * (it & 1);
      if (!wait_bounded_warp(s_full(it & 1), (it >> 1) & 1, g, 7)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32u * c, sr[c]);
      tc_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence(sr[c]);
      // mask only where needed: the diagonal tile and tiles that cross a document start
      const bool full = (j < qt) && (j * kRows >= ds);
      float x[128];
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < 128; ++e) {
        float v = __uint_as_float(sr[e >> 5][e & 31]) * sl2;
        if (!full) {
          const int col = j * kRows + e;
          if (col > row || col < ds) v = -INFINITY;
        }
        x[e] = v;
        mx = fmaxf(mx, v);
      }
      const float m_new = fmaxf(m, mx);
      const bool grow = m_new > m + 8.0f;  // also true the first time a row sees a key
      const float alpha = grow ? ex2(m - m_new) : 1.0f;
      if (it > 0 && __any_sync(0xffffffffu, grow)) {
        // rescale the running O of this row: PV_{it-1} must have landed first
        if (!wait_bounded_warp(o_done, (it - 1) & 1, g, 8)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tO = tmem + lane_off + 256u;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + 32u * c, r);
          tc_wait_ld();
          reg_fence(r);
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(tO + 32u * c, r);
        }
      }
      if (grow) {
        l *= alpha;
        lr *= alpha;
        m = m_new;
      }
      const float mu = (m == -INFINITY) ? 0.f : m;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ex2(x[32 * c + 2 * e] - mu), p1 = ex2(x[32 * c + 2 * e + 1] - mu);
          const uint32_t v = pack_bf16(p0, p1);
          l += p0 + p1;
          lr += bf16_lo(v) + bf16_hi(v);
          pk[e] = v;
        }
        tmem_st16(tS + 16u * c, pk);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // ------------------------------------------------------------ epilogue
    if (ok && wait_bounded_warp(o_done, (n - 1) & 1, g, 9)) {
      tc_fence_after();
      const float inv = 1.0f / lr;
      const uint32_t tO = tmem + lane_off + 256u;
      __nv_bfloat16* orow = p.o + ((size_t)bh * T + row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + 32u * c, r);
        tc_wait_ld();
        reg_fence(r);
        if (row < T) store_row_chunk_bf16(orow + 32 * c, r, inv);
      }
      if (row < T) p.lse[(size_t)bh * T + row] = (m + lg2(l)) * kLn2;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace ca
