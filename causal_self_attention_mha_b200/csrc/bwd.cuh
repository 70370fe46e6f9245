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
  constexpr int U = 4;        // independent 16-byte loads of each tensor in flight per thread
  const long total = rows * TPR;
  const long stride = (long)gridDim.x * blockDim.x;
  const int lane = threadIdx.x & 31;
  for (long base = (long)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < total;
       base += U * stride) {
    uint4 a[U], c[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long e = base + u * stride + lane;
      if (e < total) {
        a[u] = __ldg(reinterpret_cast<const uint4*>(o) + e);
        c[u] = __ldg(reinterpret_cast<const uint4*>(dout) + e);
      } else {
        a[u] = make_uint4(0, 0, 0, 0);
        c[u] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long e = base + u * stride + lane;
      const uint32_t av[4] = {a[u].x, a[u].y, a[u].z, a[u].w}, cv[4] = {c[u].x, c[u].y, c[u].z, c[u].w};
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        acc += bf16_lo(av[i]) * bf16_lo(cv[i]) + bf16_hi(av[i]) * bf16_hi(cv[i]);
#pragma unroll
      for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (e < total && (lane % TPR) == 0) delta[e / TPR] = acc;
    }
  }
}

struct BwdParams {
  const int32_t* doc;     // [B, T] or nullptr
  const float* lse;       // [B, H, T] natural log
  const float* delta;     // [B, H, T]
  float* delta_out;       // dq kernel with delta fused: where it writes delta [B, H, T]
  __nv_bfloat16* g0;      // dK (dkdv kernel) or dQ (dq kernel)   [B, H, T, D]
  __nv_bfloat16* g1;      // dV (dkdv kernel) or unused
  int H, T, BH, n_t;      // n_t = number of 128-row tiles along T
  int n_items;            // n_t * BH work items (one 128-row tile of one head each)
  int window;             // keys a query sees, itself included (T: no window)
  float scale;            // softmax scale (1/sqrt(d))
  float scale_log2;       // scale * log2(e)
  uint64_t wait_limit_ns;
};


// Half a row of a D-column fp32 TMEM accumulator (columns [half*D/2, (half+1)*D/2)
// of this thread's lane), times `mul`, as packed bf16 pairs: all TMEM loads in
// flight together, one wait.
template <int D>
__device__ __forceinline__ void tmem_half_row_bf16(uint32_t tacc, int half, float mul,
                                                   uint32_t (&w)[D / 4]) {
  constexpr int NC = D / 32;  // 16-column chunks per half row
  uint32_t r[NC][16];
#pragma unroll
  for (int c = 0; c < NC; ++c) tmem_ld16(tacc + (uint32_t)(half * (D / 2) + 16 * c), r[c]);
  tc_wait_ld();
#pragma unroll
  for (int c = 0; c < NC; ++c) reg_fence16(r[c]);
#pragma unroll
  for (int c = 0; c < NC; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e)
      w[8 * c + e] = pack_bf16(__uint_as_float(r[c][2 * e]) * mul, __uint_as_float(r[c][2 * e + 1]) * mul);
}

// Both tiled backward kernels are persistent: one CTA per SM walks work items
// (serpentine, heaviest first) and streams the partner operand through a ring
// of whole 128-row tiles, so every S / dP product is one M=128, N=128 MMA
// chain.  384 threads = three warpgroups: warpgroups 0-1 are the element-wise
// warps (warp w owns TMEM lanes 32*(w%4).. and columns 64*(w/4).. of each
// tile), the third holds the TMA producer and the single MMA-issuing thread;
// registers are rebalanced with setmaxnreg (168 at launch; dQ: 208 for the
// element-wise warpgroups, 88 for the third; dK/dV: 192 and 120, where the third
// warpgroup's MMA issuer needs more).  An element-wise thread keeps its
// 64 fp32 P values in registers while it waits for dP.  P and dS go back to
// TMEM as packed bf16 over the first half of the columns the same warp has
// just read, and feed the gradient MMAs as their A operand.  At an item
// boundary the gradient accumulators are handed over with acc_done (MMA ->
// epilogue) and acc_free (epilogue -> next item's first gradient MMA).

// ------------------------------------------------------------------ dK/dV
// TMEM: S^T (keys x 128 queries) at 0, dP^T at 128, dV at 256, dK at 256 + D.
// MMA stream per query tile t:  dV(t), S^T(t+1), dK(t), dP^T(t+1).  S^T(t+1)
// overwrites P^T(t) only after dV(t) in the in-order stream (likewise dP^T(t+1)
// after dK(t)), and it runs while the element-wise warps finish dS^T(t).  dV(t)
// starts on the first half of P^T(t) while the second half is still being
// computed.  The per-row vectors -LSE*log2(e) and -delta ride with the dO
// stages.  dV and dK leave through one staged bf16 tile in shared memory and
// TMA stores issued by warp 10: row-per-thread global stores from every SM at
// the same item boundary congest the memory system for microseconds.
template <int D>
struct DkdvLayout {
  static constexpr int QST = (D == 128) ? 2 : 3;  // Q ring depth (128-row tiles)
  static constexpr int DST = (D == 128) ? 2 : 3;  // dO ring depth
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + Tile<D>::BYTES;
  static constexpr int Q_OFF = V_OFF + Tile<D>::BYTES;             // + s * BYTES
  static constexpr int DO_OFF = Q_OFF + QST * Tile<D>::BYTES;      // + s * BYTES
  static constexpr int VEC_OFF = DO_OFF + DST * Tile<D>::BYTES;    // per dO stage: -lse2, -delta
  static constexpr int VEC_STAGE = 2 * kRows * 4;
  static constexpr int STG_OFF = VEC_OFF + DST * VEC_STAGE;       // output staging tile
  static constexpr int BAR_OFF = STG_OFF + Tile<D>::BYTES;
  // barriers: kv_full kv_empty | q_full[QST] q_empty[QST] | do_full[DST] do_empty[DST]
  //           vec_full[DST] | st_full dpt_full p_ready[2] ds_ready | acc_done acc_free drain |
  //           stg_full stg_free
  static constexpr int NBAR = 2 + 2 * QST + 3 * DST + 5 + 3 + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;   // tmem slot, abort flag
  static constexpr int BYTES = MISC_OFF + 16;
  static_assert(BYTES <= kMaxDynSmem, "dK/dV shared-memory layout");
  // room to round the base up to 1 KB where the opt-in limit leaves it (the
  // kernel checks the rounded layout against what it was given)
  static constexpr int SMEM = (BYTES + 1024 <= kMaxDynSmem) ? BYTES + 1024 : kMaxDynSmem;
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
      if (ld_chk(drow, (size_t)mid, (size_t)p.T) > c_last) hi = mid; else lo = mid + 1;
    }
    i_hi = (lo - 1) / kRows;
    i_hi = i_hi < I.jt ? I.jt : (i_hi > p.n_t - 1 ? p.n_t - 1 : i_hi);
  }
  {  // the last query that still has the tile's last key in its window
    const int c_last = (I.k0 + kRows - 1 < p.T) ? I.k0 + kRows - 1 : p.T - 1;
    const int r_max = c_last + p.window - 1;
    const int i_w = r_max / kRows;
    i_hi = i_w < i_hi ? i_w : i_hi;
  }
  I.n = i_hi - I.i_lo + 1;
  return I;
}

// Number of the 64 query rows r0 .. r0+63 that lie in key c's document or an
// earlier one (and before T): those rows form a prefix because document starts
// never decrease.  Lane l holds the document start of rows r0 + l and
// r0 + 32 + l (INT_MAX past T); the search runs on shuffles, so every lane of
// the warp must call it.
__device__ __forceinline__ int rows_in_doc_prefix(int a, int b, int c) {
  int n = 0;
#pragma unroll
  for (int step = 32; step >= 1; step >>= 1) {
    const int probe = n + step - 1;
    const int va = __shfl_sync(0xffffffffu, a, probe & 31);
    const int vb = __shfl_sync(0xffffffffu, b, probe & 31);
    if ((probe < 32 ? va : vb) <= c) n += step;
  }
  const int va = __shfl_sync(0xffffffffu, a, n & 31);
  const int vb = __shfl_sync(0xffffffffu, b, n & 31);
  if (n < 64 && (n < 32 ? va : vb) <= c) ++n;
  return n;
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV,
                         const __grid_constant__ CUtensorMap tmdO,
                         const __grid_constant__ CUtensorMap tmdK,
                         const __grid_constant__ CUtensorMap tmdV, const BwdParams p) {
  using Tl = Tile<D>;
  using L = DkdvLayout<D>;
  constexpr int QST = L::QST, DST = L::DST;
  constexpr int kProducerWarp = L::COMPUTE_WARPS, kMmaWarp = L::COMPUTE_WARPS + 1;
  constexpr int kStoreWarp = L::COMPUTE_WARPS + 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* gsm;
  const uint32_t sbase = aligned_smem_base(smem_raw, &gsm);
  if (sbase - smem_u32(smem_raw) + L::BYTES > dynamic_smem_bytes()) {
    if (threadIdx.x == 0) report_smem_shortfall();
    return;  // uniform across the CTA, before any barrier
  }
  const uint32_t sK = sbase + L::K_OFF, sV = sbase + L::V_OFF;
  auto sQ = [&](int s) { return sbase + L::Q_OFF + s * Tl::BYTES; };
  auto sdO = [&](int s) { return sbase + L::DO_OFF + s * Tl::BYTES; };
  float* vec = reinterpret_cast<float*>(gsm + L::VEC_OFF);   // [DST][2][128]
  const uint32_t bar0 = sbase + L::BAR_OFF;
  const uint32_t kv_full = bar0, kv_empty = bar0 + 8u;
  auto q_full = [&](int s) { return bar0 + 8u * (2 + s); };
  auto q_empty = [&](int s) { return bar0 + 8u * (2 + QST + s); };
  auto do_full = [&](int s) { return bar0 + 8u * (2 + 2 * QST + s); };
  auto do_empty = [&](int s) { return bar0 + 8u * (2 + 2 * QST + DST + s); };
  auto vec_full = [&](int s) { return bar0 + 8u * (2 + 2 * QST + 2 * DST + s); };
  const uint32_t xb = bar0 + 8u * (2 + 2 * QST + 3 * DST);
  const uint32_t st_full = xb, dpt_full = xb + 8u, ds_ready = xb + 16u;
  auto p_ready = [&](int h) { return xb + 24u + 8u * h; };  // P^T query columns [32h, 32h+32) of each warp
  const uint32_t acc_done = xb + 40u, acc_free = xb + 48u, drain = xb + 56u;
  const uint32_t stg_full = xb + 64u, stg_free = xb + 72u;  // output staging tile handshake
  const uint32_t sStg = sbase + L::STG_OFF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gsm + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gsm + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  const int w0 = blockIdx.x, dw = gridDim.x;

  if (threadIdx.x == 0) {
    mbar_init(stg_full, L::COMPUTE_WARPS);
    mbar_init(stg_free, 1);
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < QST; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), 1);
    }
    for (int s = 0; s < DST; ++s) {
      mbar_init(do_full(s), 1);
      mbar_init(do_empty(s), 1);
      mbar_init(vec_full(s), 32);
    }
    mbar_init(st_full, 1);
    mbar_init(dpt_full, 1);
    mbar_init(p_ready(0), L::COMPUTE_WARPS);
    mbar_init(p_ready(1), L::COMPUTE_WARPS);
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
    regs_shrink<120>();
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
        const int t = gq;
        const int r0 = (I.i_lo + it) * kRows;
        const int sq = t % QST, uq = t / QST;
        if (uq > 0 && !wait_bounded_warp(q_empty(sq), (uq - 1) & 1, g, 1)) { ok = false; break; }
        if (lane == 0) {
          mbar_arrive_expect_tx(q_full(sq), Tl::BYTES);
          load_tile<D>(sQ(sq), &tmQ, r0, I.bh, q_full(sq));
        }
        const int sd = t % DST, ud = t / DST;
        if (ud > 0 && !wait_bounded_warp(do_empty(sd), (ud - 1) & 1, g, 1)) { ok = false; break; }
        if (lane == 0) {
          mbar_arrive_expect_tx(do_full(sd), Tl::BYTES);
          load_tile<D>(sdO(sd), &tmdO, r0, I.bh, do_full(sd));
        }
        float* lse2 = vec + sd * 2 * kRows;
        float* dl = lse2 + kRows;
#pragma unroll
        for (int k = 0; k < kRows / 32; ++k) {
          const int rl = lane + 32 * k, r = r0 + rl;
          if (r < T) {  // stored negated: -LSE*log2(e) and -delta
            lse2[rl] = -ld_chk(p.lse, (size_t)I.bh * T + r, (size_t)p.BH * T) * kLog2e;
            dl[rl] = -ld_chk(p.delta, (size_t)I.bh * T + r, (size_t)p.BH * T);
          } else {  // rows past the end: every weight is zero
            lse2[rl] = -INFINITY;
            dl[rl] = 0.f;
          }
        }
        mbar_arrive(vec_full(sd));
        ++gq;
      }
    }
    if (lane == 0 && *abort_flag) {  // let every copy already issued land before the CTA exits
      if (li > 0) drain_wait(kv_full, (li - 1) & 1, p.wait_limit_ns);
      for (int s = 0; s < QST; ++s) {
        const int cnt = gq > s ? (gq - s + QST - 1) / QST : 0;
        if (cnt > 0) drain_wait(q_full(s), (cnt - 1) & 1, p.wait_limit_ns);
      }
      for (int s = 0; s < DST; ++s) {
        const int cnt = gq > s ? (gq - s + DST - 1) / DST : 0;
        if (cnt > 0) drain_wait(do_full(s), (cnt - 1) & 1, p.wait_limit_ns);
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
      auto issue_st = [&](int t) -> bool {  // S^T = K Q_t^T
        const int s = t % QST;
        if (!wait_bounded_fast(q_full(s), (t / QST) & 1, g, 3)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tST, desc_k<D>(sK, kk), desc_k<D>(sQ(s), kk), kIdS, kk > 0);
        tc_commit(st_full);
        return true;
      };
      auto issue_dpt = [&](int t) -> bool {  // dP^T = V dO_t^T
        const int s = t % DST;
        if (!wait_bounded_fast(do_full(s), (t / DST) & 1, g, 3)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tDPT, desc_k<D>(sV, kk), desc_k<D>(sdO(s), kk), kIdS, kk > 0);
        tc_commit(dpt_full);
        return true;
      };
      int li = 0, gq = 0;
      bool ok = true;
      for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;  // past the last item: no later round has one either
        const DkdvItem I = dkdv_item(p, w);
        if (!wait_bounded_fast(kv_full, li & 1, g, 2)) break;
        if (!issue_st(gq) || !issue_dpt(gq)) break;
        if (I.n == 1) tc_commit(kv_empty);  // K, V of this item no longer read after these
        for (int it = 0; it < I.n; ++it, ++gq) {
          const int t = gq, sq = t % QST, sd = t % DST;
          // dV += P^T dO: the first one of an item overwrites dV, so the previous
          // item's epilogue must have read it
          if (it == 0 && li >= 1 && !wait_bounded_fast(acc_free, (li - 1) & 1, g, 4)) { ok = false; break; }
          // half h holds query rows 64c + 32h + [0, 32) of the tile, c = 0, 1: K-steps 4c + 2h + {0, 1}
          for (int h = 0; h < 2; ++h) {
            if (!wait_bounded_fast(p_ready(h), t & 1, g, 5)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int kk = 4 * (j >> 1) + 2 * h + (j & 1);
              mma_ts(tdV, tST + 64u * (kk >> 2) + 8u * (kk & 3), desc_mn<D>(sdO(sd), kk), kIdG,
                     (it > 0 || h > 0 || j > 0));
            }
          }
          if (!ok) break;
          const bool more = it + 1 < I.n;
          // S^T of the next query tile, behind dV(t) in the stream
          if (more && !issue_st(t + 1)) { ok = false; break; }
          if (!wait_bounded_fast(ds_ready, t & 1, g, 6)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk)
            mma_ts(tdK, tDPT + 64u * (kk >> 2) + 8u * (kk & 3), desc_mn<D>(sQ(sq), kk), kIdG,
                   (it > 0 || kk > 0));
          tc_commit(q_empty(sq));   // Q_t no longer read
          tc_commit(do_empty(sd));  // dO_t and its row vectors no longer read
          if (more) {
            if (!issue_dpt(t + 1)) { ok = false; break; }
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
  } else if (warp == kStoreWarp) {
    // ------------------------------------------- output stores (dV, then dK)
    if (lane == 0) {
      tma_prefetch_desc(&tmdK);
      tma_prefetch_desc(&tmdV);
      int u = 0;  // staging uses so far
      bool ok = true;
      for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;  // past the last item: no later round has one either
        const int k0 = (w / p.BH) * kRows, bh = w % p.BH;
        for (int j = 0; j < 2; ++j, ++u) {
          if (!wait_bounded(stg_full, u & 1, g, 10)) { ok = false; break; }
          store_tile<D>(j ? &tmdK : &tmdV, sStg, k0, bh);
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
    regs_grow<192>();
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
      const int32_t* drow = p.doc ? p.doc + (size_t)I.b * T : nullptr;
      for (int it = 0; ok && it < I.n; ++it, ++gq) {
        const int t = gq, sd = t % DST;
        const int rb = 64 * cs;                       // first query row (in the tile) of my columns
        const int r0 = (I.i_lo + it) * kRows + rb;    // its position
        // document start of my last query row (read before the wait hides its latency)
        const int dlast = (drow && r0 + 63 < T) ? ldg_chk(drow, (size_t)(r0 + 63), (size_t)T) : 0;
        if (!wait_bounded_warp(st_full, t & 1, g, 7) ||
            !wait_bounded_warp(vec_full(sd), (t / DST) & 1, g, 7)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float* lse2 = vec + sd * 2 * kRows;
        const float* dl = lse2 + kRows;
        uint32_t sr[2][32];
        tmem_ld32(tS, sr[0]);
        tmem_ld32(tS + 32u, sr[1]);
        tc_wait_ld();
        reg_fence(sr[0]);
        reg_fence(sr[1]);
        // no mask needed when all my query rows are at or below this key, before T,
        // and in its document (document starts never decrease along the rows)
        const bool full = (r0 >= c) && (r0 + 63 < T) && (dlast <= c) && (r0 + 63 <= c + p.window - 1);
        if (__any_sync(0xffffffffu, !full)) {
          int n_vis;  // rows r0 .. r0 + n_vis - 1 are in c's document or an earlier one, and < T
          if (drow) {
            const int ra = r0 + lane, rbb = r0 + 32 + lane;
            const int da = ra < T ? ldg_chk(drow, (size_t)ra, (size_t)T) : 0x7fffffff;
            const int db = rbb < T ? ldg_chk(drow, (size_t)rbb, (size_t)T) : 0x7fffffff;
            n_vis = rows_in_doc_prefix(da, db, c);
          } else {
            n_vis = T - r0 < 0 ? 0 : (T - r0 > 64 ? 64 : T - r0);
          }
          const int r_win = c + p.window - 1 - r0;  // my key leaves the window after row r0 + r_win
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (e >= n_vis || r0 + e < c || e > r_win) sr[e >> 5][e & 31] = 0xFF800000u;  // -inf
        }
        // P^T = exp2(S^T * scale * log2e - LSE * log2e), kept in fp32 for dS^T; each half of
        // my columns goes to the dV MMA as soon as it is in TMEM
        const float4* l4 = reinterpret_cast<const float4*>(lse2 + rb);  // -LSE*log2(e)
        float pf[64];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[16];
#pragma unroll
          for (int q4 = 8 * h; q4 < 8 * h + 8; ++q4) {
            const float4 lv = l4[q4];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int e = 4 * q4 + 2 * h2;
              const uint64_t nl = h2 ? f2(lv.z, lv.w) : f2(lv.x, lv.y);
              const float2 x =
                  f2split(ffma2(f2u(sr[e >> 5][e & 31], sr[e >> 5][(e & 31) + 1]), sl2x2, nl));
              pf[e] = ex2(x.x);
              pf[e + 1] = ex2(x.y);
              pk[(e & 31) >> 1] = pack_bf16(pf[e], pf[e + 1]);
            }
          }
          tmem_st16(tS + 16u * h, pk);
          tc_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_ready(h));
        }
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
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t dk[16];
#pragma unroll
          for (int q4 = 8 * h; q4 < 8 * h + 8; ++q4) {
            const float4 dv4 = d4[q4];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int e = 4 * q4 + 2 * h2;
              const uint64_t nd = h2 ? f2(dv4.z, dv4.w) : f2(dv4.x, dv4.y);
              const float2 dd = f2split(fmul2(
                  f2(pf[e], pf[e + 1]), fadd2(f2u(dr[e >> 5][e & 31], dr[e >> 5][(e & 31) + 1]), nd)));
              dk[(e & 31) >> 1] = pack_bf16(dd.x, dd.y);
            }
          }
          tmem_st16(tD + 16u * h, dk);
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_ready);
      }
      // ---------------------------------------------------------- epilogue
      // the two warps sharing these lanes split the columns: [cs*D/2, (cs+1)*D/2)
      if (ok && wait_bounded_warp(acc_done, li & 1, g, 9)) {
        tc_fence_after();
        uint32_t wv[D / 4], wk[D / 4];
        tmem_half_row_bf16<D>(tmem + lane_off + L::T_DV, cs, 1.0f, wv);
        tmem_half_row_bf16<D>(tmem + lane_off + L::T_DK, cs, p.scale, wk);
        // dV / dK have been read: the next item's first gradient MMA may overwrite them
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_free);
        const int r = qd * 32 + lane;  // row of the staged tile
        // staging use 2*li holds dV, 2*li + 1 dK; use u may start once the store of
        // use u - 1 has read the tile
        if (li > 0 && !wait_bounded_warp(stg_free, (2 * li - 1) & 1, g, 11)) {
          ok = false;
        } else {
          stage_row<D>(gsm + L::STG_OFF, r, cs * (D / 2), wv);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(stg_full);
          if (!wait_bounded_warp(stg_free, (2 * li) & 1, g, 11)) {
            ok = false;
          } else {
            stage_row<D>(gsm + L::STG_OFF, r, cs * (D / 2), wk);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(stg_full);
          }
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

// --------------------------------------------------------------------- dQ
// Q and dO of the item's query tile stay in shared memory; K and V stream
// through rings of their own (K is read by S and by dQ, V only by dP).
// TMEM: S double-buffered at 0 / 128, dP at 256, dQ at 384.  dS(t) is written
// back (packed bf16) over S(t)'s own buffer, already read out, so dP(t+1) may
// overwrite dP(t) as soon as the element-wise warps have loaded it.  MMA stream
// per key tile t:  dP(t+1), dQ(t), S(t+2): dP(t+1) runs while dS(t) is being
// formed, and S(t+2) follows dQ(t), which has consumed dS(t), in the in-order
// stream.  dQ leaves through a TMA store from a
// staged bf16 tile that borrows one slot of the K ring: after an item's key
// tiles the producer hands the next slot to the epilogue instead of loading
// it, and the store warp (warp 10) returns it once the store has read it.
template <int D>
struct DqLayout {
  static constexpr int STK = (D == 128) ? 3 : 4;  // K ring depth (128-row tiles)
  static constexpr int STV = (D == 128) ? 2 : 3;  // V ring depth
  static constexpr int Q_OFF = 0;
  static constexpr int DO_OFF = Q_OFF + Tile<D>::BYTES;
  static constexpr int K_OFF = DO_OFF + Tile<D>::BYTES;           // + s * BYTES
  static constexpr int V_OFF = K_OFF + STK * Tile<D>::BYTES;      // + s * BYTES
  static constexpr int DPART_OFF = V_OFF + STV * Tile<D>::BYTES;  // [2][128] partial deltas
  static constexpr int BAR_OFF = DPART_OFF + 2 * kRows * 4;
  // barriers: qdo_full qdo_empty | k_full[STK] k_empty[STK] | v_full[STV] v_empty[STV] |
  //           s_full[2] dp_full dp_read ds_full | acc_done acc_free drain | stg_full stg_free |
  //           dpart_full
  static constexpr int NBAR = 2 + 2 * STK + 2 * STV + 5 + 3 + 2 + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int SMEM = BYTES + 1024;
  static_assert(SMEM <= kMaxDynSmem, "dQ shared-memory layout");
  static constexpr int COMPUTE_WARPS = 8;
  static constexpr int THREADS = 384;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S = 0, T_DP = 256, T_DQ = 384;
};

// Reads this thread's half of row r of a staged tile (columns [half*D/2, (half+1)*D/2), the
// layout load_tile produces) and returns sum_c a_rc * b_rc over them, in fp32.
template <int D>
__device__ __forceinline__ float tile_half_row_dot(const uint8_t* a, const uint8_t* b, int r,
                                                   int half) {
  using Tl = Tile<D>;
  float acc = 0.f;
#pragma unroll
  for (int u = 0; u < D / 16; ++u) {
    const int col = half * (D / 2) + 8 * u;
    const int ch = col / Tl::BOX_COLS, cu = (col % Tl::BOX_COLS) / 8;
    const int phys = (Tl::SW == 128) ? (cu ^ (r & 7)) : (cu ^ ((r >> 1) & 3));
    const int off = ch * Tl::CHUNK_BYTES + r * Tl::SW + phys * 16;
    const uint4 x = *reinterpret_cast<const uint4*>(a + off);
    const uint4 y = *reinterpret_cast<const uint4*>(b + off);
    const uint32_t xv[4] = {x.x, x.y, x.z, x.w}, yv[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      acc += bf16_lo(xv[i]) * bf16_lo(yv[i]) + bf16_hi(xv[i]) * bf16_hi(yv[i]);
  }
  return acc;
}

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
  // no key before the tile's first row's document start or window start is visible
  int first = I.q0 - p.window + 1;
  if (p.doc) {
    const int ds = ld_chk(p.doc, (size_t)I.b * p.T + I.q0, (size_t)(p.BH / p.H) * p.T);
    first = first > ds ? first : ds;
  }
  const int lo = first < 0 ? 0 : first / kRows;
  I.kv_lo = lo > I.qt ? I.qt : lo;
  I.n = I.qt - I.kv_lo + 1;
  return I;
}

// kDelta: the kernel also computes delta = rowsum(dO o O) for its query tile (O staged through
// the K ring: one extra ring element at the start of every item), uses it, and writes it to
// p.delta_out for the dK/dV kernel; otherwise it reads delta from p.delta.
template <int D, bool kDelta>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmdO,
                       const __grid_constant__ CUtensorMap tmdQ,
                       const __grid_constant__ CUtensorMap tmO, const BwdParams p) {
  using Tl = Tile<D>;
  using L = DqLayout<D>;
  constexpr int STK = L::STK, STV = L::STV;
  // K-ring elements of item li: [O (kDelta)] [its n key tiles] [dQ staging]; with gk key tiles
  // before the item, its first element is gk + li * PER_ITEM
  constexpr int E = kDelta ? 1 : 0;
  constexpr int PER_ITEM = 1 + E;
  constexpr int kProducerWarp = L::COMPUTE_WARPS, kMmaWarp = L::COMPUTE_WARPS + 1;
  constexpr int kStoreWarp = L::COMPUTE_WARPS + 2;
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
  const uint32_t stg_full = xb + 56u;  // the staged dQ tile is complete
  const uint32_t stg_free = xb + 64u;  // ... and its store has read it
  const uint32_t dp_read = xb + 72u;   // dP(t) is in the element-wise warps' registers
  const uint32_t dpart_full = xb + 80u;  // every warp's partial delta is in shared memory
  float* dpart = reinterpret_cast<float*>(gsm + L::DPART_OFF);  // [2][128]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gsm + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gsm + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  const int w0 = blockIdx.x, dw = gridDim.x;

  if (threadIdx.x == 0) {
    mbar_init(stg_full, L::COMPUTE_WARPS);
    mbar_init(stg_free, 1);
    mbar_init(qdo_full, 1);
    // Q / dO may be replaced once the item's last S / dP MMAs are done and, with the delta
    // fused, once the element-wise warps have read dO for it
    mbar_init(qdo_empty, kDelta ? 2 : 1);
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
    mbar_init(dp_read, L::COMPUTE_WARPS);
    mbar_init(ds_full, L::COMPUTE_WARPS);
    mbar_init(acc_done, 1);
    mbar_init(acc_free, L::COMPUTE_WARPS);
    mbar_init(drain, 1);
    mbar_init(dpart_full, L::COMPUTE_WARPS);
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
      if (kDelta && isK) tma_prefetch_desc(&tmO);
      int gk = 0;
      bool ok = true;
      for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;  // past the last item: no later round has one either
        const DqItem I = dq_item(p, w);
        // the K ring carries PER_ITEM more elements per item: O (kDelta) and the dQ stage
        const int n_el = isK ? I.n + PER_ITEM : I.n;
        for (int it = 0; it < n_el; ++it) {
          const int s = gk % NS, u = gk / NS;
          const uint32_t full = isK ? k_full(s) : v_full(s);
          if (u > 0 && !wait_bounded(isK ? k_empty(s) : v_empty(s), (u - 1) & 1, g, 1)) {
            ok = false;
            break;
          }
          const int kt = isK ? it - E : it;  // key tile of this element
          if (isK && kDelta && it == 0) {
            mbar_arrive_expect_tx(full, Tl::BYTES);
            load_tile<D>(sK(s), &tmO, I.q0, I.bh, full);  // the item's O tile
          } else if (kt < I.n) {
            mbar_arrive_expect_tx(full, Tl::BYTES);
            load_tile<D>(isK ? sK(s) : sV(s), tm, (I.kv_lo + kt) * kRows, I.bh, full);
          } else {
            mbar_arrive(full);  // hand the slot to the epilogue
          }
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
      int li = 0, gk = 0;
      // key tile t (counted over all items) of item li is element t + li * PER_ITEM + E of the
      // K ring (the extra elements of earlier items, and this item's O)
      auto issue_s = [&](int t) -> bool {  // S(t) = Q K_t^T into buffer t & 1
        const int el = t + li * PER_ITEM + E;
        const int s = el % STK;
        if (!wait_bounded_fast(k_full(s), (el / STK) & 1, g, 3)) return false;
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
        if (!wait_bounded_fast(v_full(s), (t / STV) & 1, g, 3)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tDP, desc_k<D>(sdO, kk), desc_k<D>(sV(s), kk), kIdS, kk > 0);
        tc_commit(dp_full);
        tc_commit(v_empty(s));  // V of this key tile no longer read
        return true;
      };
      bool ok = true;
      for (int k_ = 0; ok && k_ * dw < p.n_items; ++k_) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;  // past the last item: no later round has one either
        const DqItem I = dq_item(p, w);
        if (!wait_bounded_fast(qdo_full, li & 1, g, 2)) break;
        const int t0 = gk;
        // dP(t0) overwrites dP(t0 - 1): the element-wise warps must have loaded it
        if (t0 > 0 && !wait_bounded_fast(dp_read, (t0 - 1) & 1, g, 9)) break;
        ok = issue_s(t0) && issue_dp(t0);
        if (ok && I.n == 1) tc_commit(qdo_empty);  // Q, dO of this item no longer read
        if (ok && I.n > 1) ok = issue_s(t0 + 1);
        for (int it = 0; ok && it < I.n; ++it) {
          const int t = t0 + it;
          // dP of the next key tile as soon as dP(t) has been read out of TMEM
          if (it + 1 < I.n) {
            if (!wait_bounded_fast(dp_read, t & 1, g, 9) || !issue_dp(t + 1)) { ok = false; break; }
            if (it + 2 == I.n) tc_commit(qdo_empty);  // that was the item's last S / dP
          }
          // the first dQ MMA of an item overwrites dQ: the previous epilogue must have read it
          if (it == 0 && li >= 1 && !wait_bounded_fast(acc_free, (li - 1) & 1, g, 4)) { ok = false; break; }
          if (!wait_bounded_fast(ds_full, t & 1, g, 5)) { ok = false; break; }
          tc_fence_after();
          const int s = (t + li * PER_ITEM + E) % STK;
          const uint32_t tdS = tmem + L::T_S + 128u * (uint32_t)(t & 1);  // dS(t) over S(t)
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk)
            mma_ts(tdQ, tdS + 64u * (kk >> 2) + 8u * (kk & 3), desc_mn<D>(sK(s), kk), kIdG,
                   (it > 0 || kk > 0));
          tc_commit(k_empty(s));  // K of this key tile no longer read
          // S(t+2) reuses S(t)'s buffer, after dQ(t) in the stream
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
  } else if (warp == kStoreWarp) {
    // ------------------------------------------------------------ dQ stores
    if (lane == 0) {
      tma_prefetch_desc(&tmdQ);
      int li = 0, gk = 0;  // items, key tiles so far
      for (int k_ = 0; k_ * dw < p.n_items; ++k_, ++li) {
        const int w = snake_item(k_, w0, dw, p.n_items);
        if (w < 0) break;  // past the last item: no later round has one either
        const DqItem I = dq_item(p, w);
        gk += I.n;
        const int s = (gk + li * PER_ITEM + E) % STK;  // the item's staging slot
        if (!wait_bounded(stg_full, li & 1, g, 10)) break;
        store_tile<D>(&tmdQ, sK(s), I.q0, I.bh);
        bulk_commit();
        bulk_wait_read_all();
        mbar_arrive(stg_free);
        mbar_arrive(k_empty(s));  // the slot goes back to the K ring
      }
      bulk_wait_all();
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
      const float nlse2 =
          (r < T) ? -ld_chk(p.lse, (size_t)I.bh * T + r, (size_t)p.BH * T) * kLog2e : -INFINITY;
      float ndlt;
      if (kDelta) {
        // delta of my row from the staged O tile and dO: each of the two warps on these lanes
        // sums half of the columns; both add the two halves in the same order
        const int eo = gk + li * PER_ITEM;  // the item's O element of the K ring
        if (!wait_bounded_warp(k_full(eo % STK), (eo / STK) & 1, g, 13) ||
            !wait_bounded_warp(qdo_full, li & 1, g, 13)) {
          ok = false;
          break;
        }
        dpart[cs * kRows + rl] = tile_half_row_dot<D>(gsm + L::K_OFF + (eo % STK) * Tl::BYTES,
                                                      gsm + L::DO_OFF, rl, cs);
        __syncwarp();
        if (lane == 0) mbar_arrive(dpart_full);
        if (!wait_bounded_warp(dpart_full, li & 1, g, 13)) { ok = false; break; }
        // every warp has read O and dO: O's slot goes back to the K ring, and dO may be
        // replaced once the MMAs are done with it as well
        if (warp == 0 && lane == 0) {
          mbar_arrive(k_empty(eo % STK));
          mbar_arrive(qdo_empty);
        }
        const float dlt = dpart[rl] + dpart[kRows + rl];
        if (cs == 0 && r < T) st_chk(p.delta_out, (size_t)I.bh * T + r, (size_t)p.BH * T, dlt);
        ndlt = (r < T) ? -dlt : 0.f;
      } else {
        ndlt = (r < T) ? -ld_chk(p.delta, (size_t)I.bh * T + r, (size_t)p.BH * T) : 0.f;
      }
      // first visible key of this row: its document start or the window's start
      int ds = p.doc ? ld_chk(p.doc, (size_t)I.b * T + (r < T ? r : T - 1),
                              (size_t)(p.BH / p.H) * T)
                     : 0;
      ds = ds > r - p.window + 1 ? ds : r - p.window + 1;
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
        // dP(t) is in registers: dP(t+1) may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dp_read);
        // dS = P * (dP - delta), bf16, over the first 32 of my columns of S(t)'s buffer
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
          tmem_st16(tS, lo);
          tmem_st16(tS + 16u, hi);
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full);
      }
      // ---------------------------------------------------------- epilogue
      // the two warps sharing these lanes split the columns: [cs*D/2, (cs+1)*D/2)
      if (ok && wait_bounded_warp(acc_done, li & 1, g, 8)) {
        tc_fence_after();
        uint32_t wq[D / 4];
        tmem_half_row_bf16<D>(tmem + lane_off + L::T_DQ, cs, p.scale, wq);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_free);
        // the K-ring slot after this item's key tiles stages the tile, once the
        // producer has handed it over and the previous item's store has been read
        const int ks = gk + li * PER_ITEM + E;
        if (!wait_bounded_warp(k_full(ks % STK), (ks / STK) & 1, g, 11) ||
            (li > 0 && !wait_bounded_warp(stg_free, (li - 1) & 1, g, 12))) {
          ok = false;
        } else {
          stage_row<D>(gsm + L::K_OFF + (ks % STK) * Tl::BYTES, rl, cs * (D / 2), wq);
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
