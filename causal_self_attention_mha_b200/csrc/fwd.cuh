// fwd.cuh -- causal attention forward on sm_100a.
//
// Computes, for one head and one 128-row query tile per CTA,
//   S = scale * Q K^T  (upper triangle and other documents masked to -inf),
//   P = softmax(S) row-wise,  O = P V,  LSE = log sum exp(S)  (natural log)
// as in "Stanford CS336 walkthrough" (lmnt.cn), section 5.1 model.py,
// CausalSelfAttention.forward, and section 3.3 (masked weights are zero after
// the softmax).  The softmax is evaluated online over 128-column key tiles
// (running max m and sums, in base 2), so the T x T matrix never exists.
//
// Warp roles (320 threads):
//   warps 0-7  softmax.  Warp w owns TMEM lanes 32*(w%4).. (32 query rows) and
//              key half kh = w/4 of every key tile (64 keys).  Each half keeps
//              its own running max, sums and O accumulator, so a row is never
//              exchanged between threads inside the loop; the two halves are
//              merged once, in the epilogue.
//   warp 8     TMA producer: Q once, then K/V tiles through an ST-stage ring
//   warp 9     TMEM allocator and single-thread tcgen05.mma issuer
// TMEM (512 columns): S double buffer at columns 0 and 128 (each key half's P,
// as packed bf16, overwrites the first 32 of its own 64 S columns); O for key
// half 0 at column 256, for key half 1 at 256 + D.
//
// Per key tile j the MMA issuer runs S_{j+1} = Q K_{j+1}^T while the softmax
// warps turn S_j into P_j; then O_h += P_j,h V_j,h for both halves, with P read
// straight from TMEM.  O_h is rescaled in TMEM only when its row max grows by
// more than 2^8.  Normalisation uses the sum of the bf16-rounded weights the
// MMA actually multiplied (the weights of each output row sum to one); the LSE
// uses the sum of the fp32 weights.
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
  static constexpr int RED_OFF = V_OFF + ST * Tile<D>::BYTES;  // [2 halves][3][128] floats
  static constexpr int BAR_OFF = RED_OFF + 2 * 3 * kRows * 4;
  // barriers: q_full | k_full[ST] | v_full[ST] | kv_empty[ST] | s_full[2] | p_full[2] | o_done | drain
  static constexpr int NBAR = 1 + 3 * ST + 2 + 2 + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;       // tmem base slot, abort flag
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int SMEM = BYTES + 1024;                  // + alignment slack
  static constexpr int SOFTMAX_WARPS = 8;
  static constexpr int THREADS = (SOFTMAX_WARPS + 2) * 32;
  static constexpr uint32_t TMEM_COLS = 512;
};

template <int D>
__global__ void __launch_bounds__(320, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using Tl = Tile<D>;
  using L = FwdLayout<D>;
  constexpr int ST = L::ST;
  constexpr int kProducerWarp = L::SOFTMAX_WARPS, kMmaWarp = L::SOFTMAX_WARPS + 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* gsm;
  const uint32_t sbase = aligned_smem_base(smem_raw, &gsm);
  const uint32_t sQ = sbase + L::Q_OFF, sK = sbase + L::K_OFF, sV = sbase + L::V_OFF;
  float* red = reinterpret_cast<float*>(gsm + L::RED_OFF);
  const uint32_t bar0 = sbase + L::BAR_OFF;
  const uint32_t q_full = bar0;
  auto k_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (1 + ST + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (1 + 2 * ST + s); };
  auto s_full = [&](int b) { return bar0 + 8u * (1 + 3 * ST + b); };
  auto p_full = [&](int b) { return bar0 + 8u * (3 + 3 * ST + b); };
  const uint32_t o_done = bar0 + 8u * (5 + 3 * ST);
  const uint32_t drain = bar0 + 8u * (6 + 3 * ST);
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(p_full(i), L::SOFTMAX_WARPS);
    }
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
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

  if (warp == kProducerWarp) {
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
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t kIdO = idesc_bf16_f32(128, D, true);
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
        const int s = it % ST, bb = it & 1;
        if (it + 1 < n) {
          // S_{it+1} reuses the TMEM buffer that held P_{it-1}: PV_{it-1} must be done with it.
          if (it >= 1 && !wait_bounded(o_done, (it - 1) & 1, g, 4)) break;
          if (!issue_s(it + 1)) break;
        }
        if (!wait_bounded(p_full(bb), (it >> 1) & 1, g, 5)) break;
        if (!wait_bounded(v_full(s), (it / ST) & 1, g, 6)) break;
        tc_fence_after();
        const uint32_t tP = tmem + 128u * bb;
        const uint32_t sVs = sV + s * Tl::BYTES;
#pragma unroll
        for (int kh = 0; kh < 2; ++kh)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts(tmem + 256u + kh * D, tP + 64u * kh + 8u * kk, desc_mn<D>(sVs, 4 * kh + kk),
                   kIdO, (it > 0 || kk > 0));
        tc_commit(o_done);
        tc_commit(kv_empty(s));
      }
      tc_commit(drain);
      drain_wait(drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ softmax warps
    const int qd = warp & 3, kh = warp >> 2;
    const int rl = qd * 32 + lane;  // row within the tile == TMEM lane
    const int row = q0 + rl;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const uint32_t tO = tmem + lane_off + 256u + kh * D;
    const int ds = p.doc ? p.doc[(size_t)b * T + (row < T ? row : T - 1)] : 0;
    const float sl2 = p.scale_log2;
    // acc_l: sum of the fp32 weights (for the LSE); acc_lr: sum of the bf16-rounded weights
    // the PV MMA actually multiplies (for normalising O).  Four packed fp32 pairs each, so
    // the additions form independent chains.
    float m = -INFINITY;
    uint64_t acc_l[4], acc_lr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc_l[i] = acc_lr[i] = f2(0.f, 0.f);
    const uint64_t sl2x2 = f2(sl2, sl2);
    bool ok = true;
    for (int it = 0; it < n; ++it) {
      const int bb = it & 1;
      const int c0 = (kv_lo + it) * kRows + 64 * kh;  // first key of this thread's half
      const uint32_t tS = tmem + lane_off + 128u * bb + 64u * kh;
      if (!wait_bounded_warp(s_full(bb), (it >> 1) & 1, g, 7)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[2][32];
      tmem_ld32(tS, sr[0]);
      tmem_ld32(tS + 32u, sr[1]);
      tc_wait_ld();
      reg_fence(sr[0]);
      reg_fence(sr[1]);
      // mask only where needed: keys past the row, or before the row's document
      if (!((c0 + 63 <= row) && (c0 >= ds))) {
        const int hi = row - c0, lo = ds - c0;  // visible keys: e in [lo, hi]
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (e > hi || e < lo) sr[e >> 5][e & 31] = 0xFF800000u;  // -inf
      }
      // row max of the raw scores (scale > 0 commutes with max), four independent chains
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int e = 0; e < 64; e += 8)
#pragma unroll
        for (int q = 0; q < 4; ++q)
          mx4[q] = fmax3(mx4[q], __uint_as_float(sr[(e + 2 * q) >> 5][(e + 2 * q) & 31]),
                         __uint_as_float(sr[(e + 2 * q + 1) >> 5][(e + 2 * q + 1) & 31]));
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * sl2;
      const float m_new = fmaxf(m, mx);
      const bool grow = m_new > m + 8.0f;  // also true the first time this half sees a key
      const float alpha = grow ? ex2(m - m_new) : 1.0f;
      if (it > 0 && __any_sync(0xffffffffu, grow)) {
        // rescale this half's running O: PV_{it-1} must have landed first
        if (!wait_bounded_warp(o_done, (it - 1) & 1, g, 8)) { ok = false; break; }
        tc_fence_after();
        const uint64_t a2 = f2(alpha, alpha);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + 32u * c, r);
          tc_wait_ld();
          reg_fence(r);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 y = f2split(fmul2(f2u(r[e], r[e + 1]), a2));
            r[e] = __float_as_uint(y.x);
            r[e + 1] = __float_as_uint(y.y);
          }
          tmem_st32(tO + 32u * c, r);
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
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 x = f2split(ffma2(f2u(sr[c][2 * e], sr[c][2 * e + 1]), sl2x2, nmu2));
          const float p0 = ex2(x.x), p1 = ex2(x.y);
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
      if (lane == 0) mbar_arrive(p_full(bb));
    }
    float l = 0.f, lr = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 a = f2split(acc_l[i]), bq = f2split(acc_lr[i]);
      l += a.x + a.y;
      lr += bq.x + bq.y;
    }
    // ------------------------------------------------------------ epilogue
    ok = ok && wait_bounded_warp(o_done, (n - 1) & 1, g, 9);
    red[(kh * 3 + 0) * kRows + rl] = m;
    red[(kh * 3 + 1) * kRows + rl] = lr;
    red[(kh * 3 + 2) * kRows + rl] = l;
    named_barrier(1, L::SOFTMAX_WARPS * 32);  // every softmax thread reaches this exactly once
    if (ok) {
      tc_fence_after();
      const int oh = kh ^ 1;
      const float mo = red[(oh * 3 + 0) * kRows + rl];
      const float lro = red[(oh * 3 + 1) * kRows + rl];
      const float lo = red[(oh * 3 + 2) * kRows + rl];
      float M = fmaxf(m, mo);
      if (M == -INFINITY) M = 0.f;
      const float a_self = ex2(m - M), a_oth = ex2(mo - M);
      const float LR = lr * a_self + lro * a_oth;
      const float LX = l * a_self + lo * a_oth;
      if (kh == 0 && row < T) p.lse[(size_t)bh * T + row] = (M + lg2(LX)) * kLn2;
      const float inv = 1.0f / LR;
      const float w0 = (kh == 0 ? a_self : a_oth) * inv;  // weight of O_half0
      const float w1 = (kh == 0 ? a_oth : a_self) * inv;  // weight of O_half1
      const uint32_t tO0 = tmem + lane_off + 256u, tO1 = tO0 + D;
      __nv_bfloat16* orow = p.o + ((size_t)bh * T + row) * D;
      // this thread writes output columns [kh*D/2, (kh+1)*D/2)
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        const int col = kh * (D / 2) + 16 * c;
        uint32_t r0[16], r1[16];
        tmem_ld16(tO0 + col, r0);
        tmem_ld16(tO1 + col, r1);
        tc_wait_ld();
        reg_fence16(r0);
        reg_fence16(r1);
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float y0 = __uint_as_float(r0[2 * e]) * w0 + __uint_as_float(r1[2 * e]) * w1;
          const float y1 = __uint_as_float(r0[2 * e + 1]) * w0 + __uint_as_float(r1[2 * e + 1]) * w1;
          pk[e] = pack_bf16(y0, y1);
        }
        if (row < T) {
          uint4* d4 = reinterpret_cast<uint4*>(orow + col);
          d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
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
