// bwd.cuh -- causal attention backward on sm_100a.
//
// The pages only call loss.backward() ("Stanford CS336 walkthrough", lmnt.cn,
// section 5.2 train.py); the gradients below are the chain rule through the
// forward of section 5.1, with the softmax Jacobian applied through the
// identity  sum_k P_ik dP_ik = <dO_i, O_i>  (= delta_i):
//   P    = exp(scale * Q K^T - LSE)        (recomputed from the saved LSE)
//   dV   = P^T dO
//   dP   = dO V^T
//   dS   = P o (dP - delta)
//   dQ   = scale * dS K,   dK = scale * dS^T Q
// Three kernels, stream-ordered:
//   attn_bwd_delta_kernel  delta_i = rowsum(dO_i o O_i)             (HBM bound)
//   attn_bwd_dkdv_kernel   one 128-row key tile per CTA, loops over query tiles
//   attn_bwd_dq_kernel     one 128-row query tile per CTA, loops over key tiles
// Both tiled kernels recompute S and dP in TMEM with tcgen05.mma, turn them
// into P and dS (bf16, written back into the same TMEM columns) and feed those
// straight from TMEM into the next MMAs.  No atomics: every output element is
// written by exactly one CTA, so results are deterministic.
#pragma once

#include "tiles.cuh"

namespace ca {

// ----------------------------------------------------------------- delta
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                             const __nv_bfloat16* __restrict__ dout,
                                                             float* __restrict__ delta, long rows) {
  constexpr int TPR = D / 8;  // threads per row, 8 bf16 (16 bytes) each
  const long total = rows * TPR;
  const long stride = (long)gridDim.x * blockDim.x;
  const int lane = threadIdx.x & 31;
  for (long base = (long)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < total;
       base += stride) {
    const long e = base + lane;
    float acc = 0.f;
    if (e < total) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(o) + e);
      const uint4 c = __ldg(reinterpret_cast<const uint4*>(dout) + e);
      const uint32_t av[4] = {a.x, a.y, a.z, a.w}, cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        acc += bf16_lo(av[i]) * bf16_lo(cv[i]) + bf16_hi(av[i]) * bf16_hi(cv[i]);
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (e < total && (lane % TPR) == 0) delta[e / TPR] = acc;
  }
}

struct BwdParams {
  const int32_t* doc;     // [B, T] or nullptr
  const float* lse;       // [B, H, T] natural log
  const float* delta;     // [B, H, T]
  __nv_bfloat16* g0;      // dK (dkdv kernel) or dQ (dq kernel)   [B, H, T, D]
  __nv_bfloat16* g1;      // dV (dkdv kernel) or unused
  int H, T, BH, n_t;      // n_t = number of 128-row tiles along T
  int n_items;            // n_t * BH work items (one 128-row tile of one head each)
  float scale;            // softmax scale (1/sqrt(d))
  float scale_log2;       // scale * log2(e)
  uint64_t wait_limit_ns;
};


// Store 16 fp32 values (one TMEM x16 chunk of a row), times `mul`, as 16 bf16 to global.
__device__ __forceinline__ void store16_bf16(__nv_bfloat16* dst, const uint32_t (&r)[16], float mul) {
  uint32_t pk[8];
#pragma unroll
  for (int e = 0; e < 8; ++e)
    pk[e] = pack_bf16(__uint_as_float(r[2 * e]) * mul, __uint_as_float(r[2 * e + 1]) * mul);
  uint4* d4 = reinterpret_cast<uint4*>(dst);
  d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

// Half a row of a D-column fp32 TMEM accumulator (columns [half*D/2, (half+1)*D/2)
// of this thread's lane), times `mul`, to bf16 in global memory: all TMEM loads
// of the half row in flight together, one wait, then contiguous stores.
template <int D>
__device__ __forceinline__ void epilogue_rows(uint32_t tacc, __nv_bfloat16* row, int half,
                                              bool store, float mul) {
  constexpr int NC = (D / 2 + 15) / 16;  // 16-column chunks per half row
  uint32_t r[NC][16];
#pragma unroll
  for (int c = 0; c < NC; ++c) tmem_ld16(tacc + (uint32_t)(half * (D / 2) + 16 * c), r[c]);
  tc_wait_ld();
#pragma unroll
  for (int c = 0; c < NC; ++c) reg_fence16(r[c]);
  if (store) {
#pragma unroll
    for (int c = 0; c < NC; ++c) store16_bf16(row + half * (D / 2) + 16 * c, r[c], mul);
  }
}


// Both tiled backward kernels are persistent: one CTA per SM walks work items
// (serpentine, heaviest first) and streams the partner operand through a ring
// of whole 128-row tiles, so every S / dP product is one M=128, N=128 MMA
// chain.  384 threads = three warpgroups: warpgroups 0-1 are the element-wise
// warps (warp w owns TMEM lanes 32*(w%4).. and columns 64*(w/4).. of each
// tile), the third holds the TMA producer and the single MMA-issuing thread;
// registers are rebalanced with setmaxnreg (168 at launch; 208 for the
// element-wise warpgroups, 88 for the third).  An element-wise thread keeps its
// 64 fp32 P values in registers while it waits for dP.  P and dS go back to
// TMEM as packed bf16 over the first half of the columns the same warp has
// just read, and feed the gradient MMAs as their A operand.  At an item
// boundary the gradient accumulators are handed over with acc_done (MMA ->
// epilogue) and acc_free (epilogue -> next item's first gradient MMA).

// ------------------------------------------------------------------ dK/dV
// TMEM: S^T (keys x 128 queries) at 0, dP^T at 128, dV at 256, dK at 256 + D.
// MMA stream per query tile t:  dV(t), S^T(t+1), dK(t), dP^T(t+1).  S^T(t+1)
// overwrites P^T(t) only after dV(t) in the in-order stream (likewise dP^T(t+1)
// after dK(t)), and it runs while the element-wise warps finish dS^T(t).
template <int D>
struct DkdvLayout {
  static constexpr int ST = (D == 128) ? 2 : 3;   // Q/dO ring depth (128-row tiles)
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + Tile<D>::BYTES;
  static constexpr int Q_OFF = V_OFF + Tile<D>::BYTES;             // + s * BYTES
  static constexpr int DO_OFF = Q_OFF + ST * Tile<D>::BYTES;       // + s * BYTES
  static constexpr int VEC_OFF = DO_OFF + ST * Tile<D>::BYTES;     // per stage: -lse2, -delta, dsq
  static constexpr int VEC_STAGE = 3 * kRows * 4;
  static constexpr int BAR_OFF = VEC_OFF + ST * VEC_STAGE;
  // barriers: kv_full kv_empty | q_full[ST] q_empty[ST] | st_full dpt_full p_ready ds_ready |
  //           acc_done acc_free drain
  static constexpr int NBAR = 2 + 2 * ST + 4 + 3;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;   // tmem slot, abort flag
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int SMEM = BYTES + 1024;
  static constexpr int COMPUTE_WARPS = 8;
  static constexpr int THREADS = 384;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_ST = 0, T_DPT = 128, T_DV = 256, T_DK = 256 + D;
};

struct DkdvItem {
  int jt, bh, b, k0, i_lo, n;  // key tile, head, batch, first key row, query tiles [i_lo, i_lo+n)
};

// Key tiles near the start of the sequence see the most query tiles: they come first.
__device__ __forceinline__ DkdvItem dkdv_item(const BwdParams& p, int w) {
  DkdvItem I;
  I.jt = w / p.BH;
  I.bh = w % p.BH;
  I.b = I.bh / p.H;
  I.k0 = I.jt * kRows;
  I.i_lo = I.jt;
  int i_hi = p.n_t - 1;
  if (p.doc) {
    // last query row that can see the last key row of this tile: end of its document - 1
    const int32_t* drow = p.doc + (size_t)I.b * p.T;
    const int c_last = (I.k0 + kRows - 1 < p.T) ? I.k0 + kRows - 1 : p.T - 1;
    int lo = c_last + 1, hi = p.T;  // first r in (c_last, T) with drow[r] > c_last, else T
    while (lo < hi) {
      const int mid = lo + ((hi - lo) >> 1);
      if (drow[mid] > c_last) hi = mid; else lo = mid + 1;
    }
    i_hi = (lo - 1) / kRows;
    i_hi = i_hi < I.jt ? I.jt : (i_hi > p.n_t - 1 ? p.n_t - 1 : i_hi);
  }
  I.n = i_hi - I.i_lo + 1;
  return I;
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV,
                         const __grid_constant__ CUtensorMap tmdO, const BwdParams p) {
  using Tl = Tile<D>;
  using L = DkdvLayout<D>;
  constexpr int ST = L::ST;
  constexpr int kProducerWarp = L::COMPUTE_WARPS, kMmaWarp = L::COMPUTE_WARPS + 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* gsm;
  const uint32_t sbase = aligned_smem_base(smem_raw, &gsm);
  const uint32_t sK = sbase + L::K_OFF, sV = sbase + L::V_OFF;
  auto sQ = [&](int s) { return sbase + L::Q_OFF + s * Tl::BYTES; };
  auto sdO = [&](int s) { return sbase + L::DO_OFF + s * Tl::BYTES; };
  float* vec = reinterpret_cast<float*>(gsm + L::VEC_OFF);   // [ST][3][128]
  const uint32_t bar0 = sbase + L::BAR_OFF;
  const uint32_t kv_full = bar0, kv_empty = bar0 + 8u;
  auto q_full = [&](int s) { return bar0 + 8u * (2 + s); };
  auto q_empty = [&](int s) { return bar0 + 8u * (2 + ST + s); };
  const uint32_t xb = bar0 + 8u * (2 + 2 * ST);
  const uint32_t st_full = xb, dpt_full = xb + 8u, p_ready = xb + 16u, ds_ready = xb + 24u;
  const uint32_t acc_done = xb + 32u, acc_free = xb + 40u, drain = xb + 48u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gsm + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gsm + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  const int w0 = blockIdx.x, dw = gridDim.x;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(q_full(s), 32);
      mbar_init(q_empty(s), 1);
    }
    mbar_init(st_full, 1);
    mbar_init(dpt_full, 1);
    mbar_init(p_ready, L::COMPUTE_WARPS);
    mbar_init(ds_ready, L::COMPUTE_WARPS);
    mbar_init(acc_done, 1);
    mbar_init(acc_free, L::COMPUTE_WARPS);
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

  if (warp >= L::COMPUTE_WARPS) {
    regs_shrink<88>();
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
    }
    int li = 0, gq = 0;  // items whose K/V were loaded, query tiles loaded
    bool ok = true;
    for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
      const int w = snake_item(k_, w0, dw, p.n_items);
      if (w < 0) break;  // past the last item: no later round has one either
      const DkdvItem I = dkdv_item(p, w);
      // K/V of this item: the previous item's MMAs must be done with the old ones
      if (li >= 1 && !wait_bounded_warp(kv_empty, (li - 1) & 1, g, 1)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(kv_full, 2 * Tl::BYTES);
        load_tile<D>(sK, &tmK, I.k0, I.bh, kv_full);
        load_tile<D>(sV, &tmV, I.k0, I.bh, kv_full);
      }
      ++li;
      for (int it = 0; it < I.n; ++it) {
        const int s = gq % ST, u = gq / ST;
        if (u > 0 && !wait_bounded_warp(q_empty(s), (u - 1) & 1, g, 1)) { ok = false; break; }
        const int r0 = (I.i_lo + it) * kRows;
        float* lse2 = vec + s * 3 * kRows;
        float* dl = lse2 + kRows;
        int* dsq = reinterpret_cast<int*>(dl + kRows);
#pragma unroll
        for (int k = 0; k < kRows / 32; ++k) {
          const int rl = lane + 32 * k, r = r0 + rl;
          if (r < T) {  // stored negated: -LSE*log2(e) and -delta
            lse2[rl] = -p.lse[(size_t)I.bh * T + r] * kLog2e;
            dl[rl] = -p.delta[(size_t)I.bh * T + r];
            dsq[rl] = p.doc ? p.doc[(size_t)I.b * T + r] : 0;
          } else {  // rows past the end: no key is visible
            lse2[rl] = -INFINITY;
            dl[rl] = 0.f;
            dsq[rl] = 0x7fffffff;
          }
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(q_full(s), 2 * Tl::BYTES);
          load_tile<D>(sQ(s), &tmQ, r0, I.bh, q_full(s));
          load_tile<D>(sdO(s), &tmdO, r0, I.bh, q_full(s));
        } else {
          mbar_arrive(q_full(s));
        }
        ++gq;
      }
    }
    if (lane == 0 && *abort_flag) {  // let every copy already issued land before the CTA exits
      if (li > 0) drain_wait(kv_full, (li - 1) & 1, p.wait_limit_ns);
      for (int s = 0; s < ST; ++s) {
        const int cnt = gq > s ? (gq - s + ST - 1) / ST : 0;
        if (cnt > 0) drain_wait(q_full(s), (cnt - 1) & 1, p.wait_limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false);  // S^T, dP^T: M = keys, N = queries
      constexpr uint32_t kIdG = idesc_bf16_f32(128, D, true);     // dV, dK: N = d, B is MN-major
      const uint32_t tST = tmem + L::T_ST, tDPT = tmem + L::T_DPT;
      const uint32_t tdV = tmem + L::T_DV, tdK = tmem + L::T_DK;
      auto issue_st = [&](int s) {  // S^T = K Q_s^T
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tST, desc_k<D>(sK, kk), desc_k<D>(sQ(s), kk), kIdS, kk > 0);
        tc_commit(st_full);
      };
      auto issue_dpt = [&](int s) {  // dP^T = V dO_s^T
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tDPT, desc_k<D>(sV, kk), desc_k<D>(sdO(s), kk), kIdS, kk > 0);
        tc_commit(dpt_full);
      };
      int li = 0, gq = 0;
      bool ok = true;
      for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;  // past the last item: no later round has one either
        const DkdvItem I = dkdv_item(p, w);
        if (!wait_bounded(kv_full, li & 1, g, 2)) break;
        const int s0 = gq % ST;
        if (!wait_bounded(q_full(s0), (gq / ST) & 1, g, 3)) break;
        issue_st(s0);
        issue_dpt(s0);
        if (I.n == 1) tc_commit(kv_empty);  // K, V of this item no longer read after these
        for (int it = 0; it < I.n; ++it, ++gq) {
          const int t = gq, s = t % ST;
          // dV += P^T dO: the first one of an item overwrites dV, so the previous
          // item's epilogue must have read it
          if (it == 0 && li >= 1 && !wait_bounded(acc_free, (li - 1) & 1, g, 4)) { ok = false; break; }
          if (!wait_bounded(p_ready, t & 1, g, 5)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk)
            mma_ts(tdV, tST + 64u * (kk >> 2) + 8u * (kk & 3), desc_mn<D>(sdO(s), kk), kIdG,
                   (it > 0 || kk > 0));
          const bool more = it + 1 < I.n;
          const int s1 = (t + 1) % ST;
          if (more) {  // S^T of the next query tile, behind dV(t) in the stream
            if (!wait_bounded(q_full(s1), ((t + 1) / ST) & 1, g, 3)) { ok = false; break; }
            issue_st(s1);
          }
          if (!wait_bounded(ds_ready, t & 1, g, 6)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk)
            mma_ts(tdK, tDPT + 64u * (kk >> 2) + 8u * (kk & 3), desc_mn<D>(sQ(s), kk), kIdG,
                   (it > 0 || kk > 0));
          tc_commit(q_empty(s));  // Q_t, dO_t no longer read
          if (more) {
            issue_dpt(s1);
            if (it + 2 == I.n) tc_commit(kv_empty);  // that was the item's last S^T / dP^T
          }
        }
        if (!ok) break;
        tc_commit(acc_done);
        ++li;
      }
      tc_commit(drain);
      drain_wait(drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  }
  } else {
    regs_grow<208>();
    // ------------------------------------------- P^T / dS^T (thread = key row)
    const int qd = warp & 3, cs = warp >> 2;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const uint32_t tS = tmem + lane_off + L::T_ST + 64u * cs;   // my 64 columns of S^T
    const uint32_t tD = tmem + lane_off + L::T_DPT + 64u * cs;  // ... and of dP^T
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2(sl2, sl2);
    bool ok = true;
    int li = 0, gq = 0;
    for (int k_ = 0; k_ * dw < p.n_items; ++k_, ++li) {
      const int w = snake_item(k_, w0, dw, p.n_items);
      if (w < 0) break;  // past the last item: no later round has one either
      const DkdvItem I = dkdv_item(p, w);
      const int c = I.k0 + qd * 32 + lane;  // key position owned by this thread
      for (int it = 0; ok && it < I.n; ++it, ++gq) {
        const int t = gq, s = t % ST;
        if (!wait_bounded_warp(st_full, t & 1, g, 7) ||
            !wait_bounded_warp(q_full(s), (t / ST) & 1, g, 7)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float* lse2 = vec + s * 3 * kRows;
        const float* dl = lse2 + kRows;
        const int* dsq = reinterpret_cast<const int*>(dl + kRows);
        const int rb = 64 * cs;                       // first query row (in the tile) of my columns
        const int r0 = (I.i_lo + it) * kRows + rb;    // its position
        uint32_t sr[2][32];
        tmem_ld32(tS, sr[0]);
        tmem_ld32(tS + 32u, sr[1]);
        tc_wait_ld();
        reg_fence(sr[0]);
        reg_fence(sr[1]);
        // no mask needed when all my query rows are at or below this key and their
        // documents start at or before it (dsq is nondecreasing; huge past T)
        if (!((r0 >= c) && (dsq[rb + 63] <= c))) {
          const int4* ds4 = reinterpret_cast<const int4*>(dsq + rb);
#pragma unroll
          for (int q4 = 0; q4 < 16; ++q4) {
            const int4 dv4 = ds4[q4];
            const int dsv[4] = {dv4.x, dv4.y, dv4.z, dv4.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int e = 4 * q4 + k;
              if (c > r0 + e || c < dsv[k]) sr[e >> 5][e & 31] = 0xFF800000u;  // -inf: weight 0
            }
          }
        }
        // P^T = exp2(S^T * scale * log2e - LSE * log2e), kept in fp32 for dS^T
        const float4* l4 = reinterpret_cast<const float4*>(lse2 + rb);  // -LSE*log2(e)
        float pf[64];
        uint32_t pk[32];
#pragma unroll
        for (int q4 = 0; q4 < 16; ++q4) {
          const float4 lv = l4[q4];
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int e = 4 * q4 + 2 * h2;
            const uint64_t nl = h2 ? f2(lv.z, lv.w) : f2(lv.x, lv.y);
            const float2 x =
                f2split(ffma2(f2u(sr[e >> 5][e & 31], sr[e >> 5][(e & 31) + 1]), sl2x2, nl));
            pf[e] = ex2(x.x);
            pf[e + 1] = ex2(x.y);
            pk[e >> 1] = pack_bf16(pf[e], pf[e + 1]);
          }
        }
        {
          uint32_t (&lo)[16] = *reinterpret_cast<uint32_t(*)[16]>(&pk[0]);
          uint32_t (&hi)[16] = *reinterpret_cast<uint32_t(*)[16]>(&pk[16]);
          tmem_st16(tS, lo);
          tmem_st16(tS + 16u, hi);
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_ready);
        // dS^T = P^T * (dP^T - delta)
        if (!wait_bounded_warp(dpt_full, t & 1, g, 8)) { ok = false; break; }
        tc_fence_after();
        uint32_t dr[2][32];
        tmem_ld32(tD, dr[0]);
        tmem_ld32(tD + 32u, dr[1]);
        tc_wait_ld();
        reg_fence(dr[0]);
        reg_fence(dr[1]);
        const float4* d4 = reinterpret_cast<const float4*>(dl + rb);  // -delta
        uint32_t dk[32];
#pragma unroll
        for (int q4 = 0; q4 < 16; ++q4) {
          const float4 dv4 = d4[q4];
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int e = 4 * q4 + 2 * h2;
            const uint64_t nd = h2 ? f2(dv4.z, dv4.w) : f2(dv4.x, dv4.y);
            const float2 dd = f2split(fmul2(
                f2(pf[e], pf[e + 1]), fadd2(f2u(dr[e >> 5][e & 31], dr[e >> 5][(e & 31) + 1]), nd)));
            dk[e >> 1] = pack_bf16(dd.x, dd.y);
          }
        }
        {
          uint32_t (&lo)[16] = *reinterpret_cast<uint32_t(*)[16]>(&dk[0]);
          uint32_t (&hi)[16] = *reinterpret_cast<uint32_t(*)[16]>(&dk[16]);
          tmem_st16(tD, lo);
          tmem_st16(tD + 16u, hi);
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_ready);
      }
      // ---------------------------------------------------------- epilogue
      if (ok && wait_bounded_warp(acc_done, li & 1, g, 9)) {
        tc_fence_after();
        __nv_bfloat16* dk_row = p.g0 + ((size_t)I.bh * T + c) * D;
        __nv_bfloat16* dv_row = p.g1 + ((size_t)I.bh * T + c) * D;
        // the two warps sharing these lanes split the columns: [cs*D/2, (cs+1)*D/2)
        epilogue_rows<D>(tmem + lane_off + L::T_DV, dv_row, cs, c < T, 1.0f);
        epilogue_rows<D>(tmem + lane_off + L::T_DK, dk_row, cs, c < T, p.scale);
        // dV / dK have been read: the next item's first gradient MMA may overwrite them
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_free);
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

// --------------------------------------------------------------------- dQ
// Q and dO of the item's query tile stay in shared memory; K and V stream
// through rings of their own (K is read by S and by dQ, V only by dP).
// TMEM: S double-buffered at 0 / 128, dP at 256 (dS is written back over its
// first half), dQ at 384.  MMA stream per key tile t:  dQ(t), dP(t+1), S(t+2):
// S(t+1) is ready before the element-wise warps need it, and the only
// tensor-core work they wait for is dP.
template <int D>
struct DqLayout {
  static constexpr int STK = (D == 128) ? 3 : 4;  // K ring depth (128-row tiles)
  static constexpr int STV = (D == 128) ? 2 : 3;  // V ring depth
  static constexpr int Q_OFF = 0;
  static constexpr int DO_OFF = Q_OFF + Tile<D>::BYTES;
  static constexpr int K_OFF = DO_OFF + Tile<D>::BYTES;           // + s * BYTES
  static constexpr int V_OFF = K_OFF + STK * Tile<D>::BYTES;      // + s * BYTES
  static constexpr int BAR_OFF = V_OFF + STV * Tile<D>::BYTES;
  // barriers: qdo_full qdo_empty | k_full[STK] k_empty[STK] | v_full[STV] v_empty[STV] |
  //           s_full[2] dp_full ds_full | acc_done acc_free drain
  static constexpr int NBAR = 2 + 2 * STK + 2 * STV + 4 + 3;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int SMEM = BYTES + 1024;
  static constexpr int COMPUTE_WARPS = 8;
  static constexpr int THREADS = 384;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S = 0, T_DP = 256, T_DQ = 384;
};

struct DqItem {
  int qt, bh, b, q0, kv_lo, n;  // query tile, head, batch, first row, key tiles [kv_lo, kv_lo+n)
};

// Query tiles near the end of the sequence see the most key tiles: they come first.
__device__ __forceinline__ DqItem dq_item(const BwdParams& p, int w) {
  DqItem I;
  I.qt = p.n_t - 1 - w / p.BH;
  I.bh = w % p.BH;
  I.b = I.bh / p.H;
  I.q0 = I.qt * kRows;
  I.kv_lo = 0;
  if (p.doc) {  // no key before the document start of the tile's first row is visible
    const int lo = p.doc[(size_t)I.b * p.T + I.q0] / kRows;
    I.kv_lo = lo < 0 ? 0 : (lo > I.qt ? I.qt : lo);
  }
  I.n = I.qt - I.kv_lo + 1;
  return I;
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmdO, const BwdParams p) {
  using Tl = Tile<D>;
  using L = DqLayout<D>;
  constexpr int STK = L::STK, STV = L::STV;
  constexpr int kProducerWarp = L::COMPUTE_WARPS, kMmaWarp = L::COMPUTE_WARPS + 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* gsm;
  const uint32_t sbase = aligned_smem_base(smem_raw, &gsm);
  const uint32_t sQ = sbase + L::Q_OFF, sdO = sbase + L::DO_OFF;
  auto sK = [&](int s) { return sbase + L::K_OFF + s * Tl::BYTES; };
  auto sV = [&](int s) { return sbase + L::V_OFF + s * Tl::BYTES; };
  const uint32_t bar0 = sbase + L::BAR_OFF;
  const uint32_t qdo_full = bar0, qdo_empty = bar0 + 8u;
  auto k_full = [&](int s) { return bar0 + 8u * (2 + s); };
  auto k_empty = [&](int s) { return bar0 + 8u * (2 + STK + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (2 + 2 * STK + s); };
  auto v_empty = [&](int s) { return bar0 + 8u * (2 + 2 * STK + STV + s); };
  const uint32_t xb = bar0 + 8u * (2 + 2 * STK + 2 * STV);
  auto s_full = [&](int b) { return xb + 8u * b; };
  const uint32_t dp_full = xb + 16u, ds_full = xb + 24u;
  const uint32_t acc_done = xb + 32u, acc_free = xb + 40u, drain = xb + 48u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gsm + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gsm + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  const int w0 = blockIdx.x, dw = gridDim.x;

  if (threadIdx.x == 0) {
    mbar_init(qdo_full, 1);
    mbar_init(qdo_empty, 1);
    for (int s = 0; s < STK; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
    }
    for (int s = 0; s < STV; ++s) {
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    mbar_init(s_full(0), 1);
    mbar_init(s_full(1), 1);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, L::COMPUTE_WARPS);
    mbar_init(acc_done, 1);
    mbar_init(acc_free, L::COMPUTE_WARPS);
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

  if (warp >= L::COMPUTE_WARPS) {
    regs_shrink<88>();
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {  // Q / dO, one pair per item
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmdO);
      int li = 0;
      for (int k_ = 0; k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;  // past the last item: no later round has one either
        const DqItem I = dq_item(p, w);
        // the previous item's S / dP MMAs must be done with the old Q / dO
        if (li >= 1 && !wait_bounded(qdo_empty, (li - 1) & 1, g, 1)) break;
        mbar_arrive_expect_tx(qdo_full, 2 * Tl::BYTES);
        load_tile<D>(sQ, &tmQ, I.q0, I.bh, qdo_full);
        load_tile<D>(sdO, &tmdO, I.q0, I.bh, qdo_full);
        ++li;
      }
      if (*abort_flag && li > 0) drain_wait(qdo_full, (li - 1) & 1, p.wait_limit_ns);
    } else if (lane == 1 || lane == 2) {  // lane 1: the K ring, lane 2: the V ring
      const bool isK = (lane == 1);
      const int NS = isK ? STK : STV;
      const CUtensorMap* tm = isK ? &tmK : &tmV;
      tma_prefetch_desc(tm);
      int gk = 0;
      bool ok = true;
      for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;  // past the last item: no later round has one either
        const DqItem I = dq_item(p, w);
        for (int it = 0; it < I.n; ++it) {
          const int s = gk % NS, u = gk / NS;
          const uint32_t full = isK ? k_full(s) : v_full(s);
          if (u > 0 && !wait_bounded(isK ? k_empty(s) : v_empty(s), (u - 1) & 1, g, 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full, Tl::BYTES);
          load_tile<D>(isK ? sK(s) : sV(s), tm, (I.kv_lo + it) * kRows, I.bh, full);
          ++gk;
        }
      }
      if (*abort_flag) {  // let every copy already issued land before the CTA exits
        for (int s = 0; s < NS; ++s) {
          const int cnt = gk > s ? (gk - s + NS - 1) / NS : 0;
          if (cnt > 0) drain_wait(isK ? k_full(s) : v_full(s), (cnt - 1) & 1, p.wait_limit_ns);
        }
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false);  // S, dP: M = queries, N = keys
      constexpr uint32_t kIdG = idesc_bf16_f32(128, D, true);     // dQ: N = d, B (K) is MN-major
      const uint32_t tDP = tmem + L::T_DP, tdQ = tmem + L::T_DQ;
      auto issue_s = [&](int t) -> bool {  // S(t) = Q K_t^T into buffer t & 1
        const int s = t % STK;
        if (!wait_bounded(k_full(s), (t / STK) & 1, g, 3)) return false;
        tc_fence_after();
        const uint32_t tS = tmem + L::T_S + 128u * (uint32_t)(t & 1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tS, desc_k<D>(sQ, kk), desc_k<D>(sK(s), kk), kIdS, kk > 0);
        tc_commit(s_full(t & 1));
        return true;
      };
      auto issue_dp = [&](int t) -> bool {  // dP(t) = dO V_t^T
        const int s = t % STV;
        if (!wait_bounded(v_full(s), (t / STV) & 1, g, 3)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tDP, desc_k<D>(sdO, kk), desc_k<D>(sV(s), kk), kIdS, kk > 0);
        tc_commit(dp_full);
        tc_commit(v_empty(s));  // V of this key tile no longer read
        return true;
      };
      int li = 0, gk = 0;
      bool ok = true;
      for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;  // past the last item: no later round has one either
        const DqItem I = dq_item(p, w);
        if (!wait_bounded(qdo_full, li & 1, g, 2)) break;
        const int t0 = gk;
        ok = issue_s(t0) && issue_dp(t0);
        if (ok && I.n == 1) tc_commit(qdo_empty);  // Q, dO of this item no longer read
        if (ok && I.n > 1) ok = issue_s(t0 + 1);
        for (int it = 0; ok && it < I.n; ++it) {
          const int t = t0 + it;
          // the first dQ MMA of an item overwrites dQ: the previous epilogue must have read it
          if (it == 0 && li >= 1 && !wait_bounded(acc_free, (li - 1) & 1, g, 4)) { ok = false; break; }
          if (!wait_bounded(ds_full, t & 1, g, 5)) { ok = false; break; }
          tc_fence_after();
          const int s = t % STK;
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk)
            mma_ts(tdQ, tDP + 64u * (kk >> 2) + 8u * (kk & 3), desc_mn<D>(sK(s), kk), kIdG,
                   (it > 0 || kk > 0));
          tc_commit(k_empty(s));  // K of this key tile no longer read
          if (it + 1 < I.n) {
            if (!issue_dp(t + 1)) { ok = false; break; }
            if (it + 2 == I.n) tc_commit(qdo_empty);  // that was the item's last S / dP
          }
          if (it + 2 < I.n && !issue_s(t + 2)) { ok = false; break; }
        }
        if (!ok) break;
        gk += I.n;
        tc_commit(acc_done);
        ++li;
      }
      tc_commit(drain);
      drain_wait(drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  }
  } else {
    regs_grow<208>();
    // ----------------------------------------------- P / dS (thread = query row)
    const int qd = warp & 3, cs = warp >> 2;
    const int rl = qd * 32 + lane;  // row within the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const uint32_t tD = tmem + lane_off + L::T_DP + 64u * cs;  // my 64 columns of dP
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2(sl2, sl2);
    bool ok = true;
    int li = 0, gk = 0;
    for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_, ++li) {
      const int w = snake_item(k_, w0, dw, p.n_items);
      if (w < 0) break;  // past the last item: no later round has one either
      const DqItem I = dq_item(p, w);
      const int r = I.q0 + rl;  // query position owned by this thread
      // rows past T: -LSE = -inf makes every weight zero
      const float nlse2 = (r < T) ? -p.lse[(size_t)I.bh * T + r] * kLog2e : -INFINITY;
      const float ndlt = (r < T) ? -p.delta[(size_t)I.bh * T + r] : 0.f;
      const int ds = p.doc ? p.doc[(size_t)I.b * T + (r < T ? r : T - 1)] : 0;
      const uint64_t nlse2x2 = f2(nlse2, nlse2), ndltx2 = f2(ndlt, ndlt);
      for (int it = 0; it < I.n; ++it, ++gk) {
        const int t = gk;
        if (!wait_bounded_warp(s_full(t & 1), (t >> 1) & 1, g, 6)) { ok = false; break; }
        tc_fence_after();
        const int c0 = (I.kv_lo + it) * kRows + 64 * cs;  // first key of my columns
        const uint32_t tS = tmem + lane_off + L::T_S + 128u * (uint32_t)(t & 1) + 64u * cs;
        uint32_t sr[2][32];
        tmem_ld32(tS, sr[0]);
        tmem_ld32(tS + 32u, sr[1]);
        tc_wait_ld();
        reg_fence(sr[0]);
        reg_fence(sr[1]);
        if (!((c0 + 63 <= r) && (c0 >= ds))) {
          const int hi = r - c0, lo = ds - c0;  // visible keys: e in [lo, hi]
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (e > hi || e < lo) sr[e >> 5][e & 31] = 0xFF800000u;  // -inf: weight 0
        }
        // P = exp2(S * scale * log2e - LSE * log2e), kept in fp32 until dP arrives
        float pf[64];
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const float2 x =
              f2split(ffma2(f2u(sr[e >> 5][e & 31], sr[e >> 5][(e & 31) + 1]), sl2x2, nlse2x2));
          pf[e] = ex2(x.x);
          pf[e + 1] = ex2(x.y);
        }
        if (!wait_bounded_warp(dp_full, t & 1, g, 7)) { ok = false; break; }
        tc_fence_after();
        uint32_t dr[2][32];
        tmem_ld32(tD, dr[0]);
        tmem_ld32(tD + 32u, dr[1]);
        tc_wait_ld();
        reg_fence(dr[0]);
        reg_fence(dr[1]);
        // dS = P * (dP - delta), bf16, over the first 32 of my dP columns
        uint32_t dk[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const float2 d = f2split(fmul2(
              f2(pf[e], pf[e + 1]), fadd2(f2u(dr[e >> 5][e & 31], dr[e >> 5][(e & 31) + 1]), ndltx2)));
          dk[e >> 1] = pack_bf16(d.x, d.y);
        }
        {
          uint32_t (&lo)[16] = *reinterpret_cast<uint32_t(*)[16]>(&dk[0]);
          uint32_t (&hi)[16] = *reinterpret_cast<uint32_t(*)[16]>(&dk[16]);
          tmem_st16(tD, lo);
          tmem_st16(tD + 16u, hi);
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full);
      }
      // ---------------------------------------------------------- epilogue
      if (ok && wait_bounded_warp(acc_done, li & 1, g, 8)) {
        tc_fence_after();
        __nv_bfloat16* dq_row = p.g0 + ((size_t)I.bh * T + r) * D;
        epilogue_rows<D>(tmem + lane_off + L::T_DQ, dq_row, cs, r < T, p.scale);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_free);
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
