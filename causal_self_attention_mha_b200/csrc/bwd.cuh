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
  float scale;            // softmax scale (1/sqrt(d))
  float scale_log2;       // scale * log2(e)
  uint64_t wait_limit_ns;
};

// ------------------------------------------------------------------ dK/dV
template <int D>
struct DkdvLayout {
  static constexpr int ST = (D == 128) ? 2 : 3;   // Q/dO ring depth
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + Tile<D>::BYTES;
  static constexpr int Q_OFF = V_OFF + Tile<D>::BYTES;             // + s * BYTES
  static constexpr int DO_OFF = Q_OFF + ST * Tile<D>::BYTES;       // + s * BYTES
  static constexpr int VEC_OFF = DO_OFF + ST * Tile<D>::BYTES;     // per stage: lse2, delta, dsq
  static constexpr int VEC_STAGE = 3 * kRows * 4;
  static constexpr int BAR_OFF = VEC_OFF + ST * VEC_STAGE;
  // barriers: kv_full | q_full[ST] | q_empty[ST] | st_full | pds_full | acc_done | drain
  static constexpr int NBAR = 1 + 2 * ST + 4;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;   // tmem slot, abort flag, q-tile range
  static constexpr int BYTES = MISC_OFF + 32;
  static constexpr int SMEM = BYTES + 1024;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV,
                         const __grid_constant__ CUtensorMap tmdO, const BwdParams p) {
  using Tl = Tile<D>;
  using L = DkdvLayout<D>;
  constexpr int ST = L::ST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* gsm;
  const uint32_t sbase = aligned_smem_base(smem_raw, &gsm);
  const uint32_t sK = sbase + L::K_OFF, sV = sbase + L::V_OFF;
  auto sQ = [&](int s) { return sbase + L::Q_OFF + s * Tl::BYTES; };
  auto sdO = [&](int s) { return sbase + L::DO_OFF + s * Tl::BYTES; };
  float* vec = reinterpret_cast<float*>(gsm + L::VEC_OFF);   // [ST][3][128]
  const uint32_t bar0 = sbase + L::BAR_OFF;
  const uint32_t kv_full = bar0;
  auto q_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto q_empty = [&](int s) { return bar0 + 8u * (1 + ST + s); };
  const uint32_t st_full = bar0 + 8u * (1 + 2 * ST);
  const uint32_t pds_full = bar0 + 8u * (2 + 2 * ST);
  const uint32_t acc_done = bar0 + 8u * (3 + 2 * ST);
  const uint32_t drain = bar0 + 8u * (4 + 2 * ST);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gsm + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gsm + L::MISC_OFF + 4);
  int* range = reinterpret_cast<int*>(gsm + L::MISC_OFF + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  // Work item: key tiles near the start of the sequence see the most query tiles; launch them first.
  const int jt = (int)(blockIdx.x / p.BH);
  const int bh = (int)(blockIdx.x % p.BH);
  const int b = bh / p.H;
  const int k0 = jt * kRows;

  if (threadIdx.x == 0) {
    int i_hi = p.n_t - 1;
    if (p.doc) {
      // last query row that can see the last key row of this tile: end of its document - 1
      const int32_t* drow = p.doc + (size_t)b * T;
      const int c_last = (k0 + kRows - 1 < T) ? k0 + kRows - 1 : T - 1;
      int lo = c_last + 1, hi = T;  // first r in (c_last, T) with drow[r] > c_last, else T
      while (lo < hi) {
        const int mid = lo + ((hi - lo) >> 1);
        if (drow[mid] > c_last) hi = mid; else lo = mid + 1;
      }
      i_hi = (lo - 1) / kRows;
      i_hi = i_hi < jt ? jt : (i_hi > p.n_t - 1 ? p.n_t - 1 : i_hi);
    }
    range[0] = jt;
    range[1] = i_hi;
    mbar_init(kv_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(q_full(s), 32);
      mbar_init(q_empty(s), 1);
    }
    mbar_init(st_full, 1);
    mbar_init(pds_full, 4);
    mbar_init(acc_done, 1);
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
  const int i_lo = range[0];
  const int n = range[1] - i_lo + 1;
  const Guard g{abort_flag, p.wait_limit_ns};
  const uint32_t tST = tmem, tDPT = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      mbar_arrive_expect_tx(kv_full, 2 * Tl::BYTES);
      load_tile<D>(sK, &tmK, k0, bh, kv_full);
      load_tile<D>(sV, &tmV, k0, bh, kv_full);
    }
    int it = 0;
    for (; it < n; ++it) {
      const int s = it % ST, u = it / ST;
      if (u > 0 && !wait_bounded_warp(q_empty(s), (u - 1) & 1, g, 1)) break;
      const int r0 = (i_lo + it) * kRows;
      float* lse2 = vec + s * 3 * kRows;
      float* dl = lse2 + kRows;
      int* dsq = reinterpret_cast<int*>(dl + kRows);
#pragma unroll
      for (int k = 0; k < kRows / 32; ++k) {
        const int rl = lane + 32 * k, r = r0 + rl;
        if (r < T) {
          lse2[rl] = p.lse[(size_t)bh * T + r] * kLog2e;
          dl[rl] = p.delta[(size_t)bh * T + r];
          dsq[rl] = p.doc ? p.doc[(size_t)b * T + r] : 0;
        } else {  // rows past the end: no key is visible
          lse2[rl] = INFINITY;
          dl[rl] = 0.f;
          dsq[rl] = 0x7fffffff;
        }
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full(s), 2 * Tl::BYTES);
        load_tile<D>(sQ(s), &tmQ, r0, bh, q_full(s));
        load_tile<D>(sdO(s), &tmdO, r0, bh, q_full(s));
      } else {
        mbar_arrive(q_full(s));
      }
    }
    if (lane == 0 && *abort_flag) {
      drain_wait(kv_full, 0, p.wait_limit_ns);
      for (int s = 0; s < ST; ++s) {
        const int cnt = it > s ? (it - s + ST - 1) / ST : 0;
        if (cnt > 0) drain_wait(q_full(s), (cnt - 1) & 1, p.wait_limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false);  // S^T, dP^T: M = keys, N = queries
      constexpr uint32_t kIdG = idesc_bf16_f32(128, D, true);     // dV, dK: N = d, B is MN-major
      bool ok = wait_bounded(kv_full, 0, g, 2);
      for (int it = 0; ok && it < n; ++it) {
        const int s = it % ST;
        if (!wait_bounded(q_full(s), (it / ST) & 1, g, 3)) break;
        // S^T / dP^T overwrite the P^T / dS^T that the previous dV / dK MMAs read
        if (it > 0 && !wait_bounded(q_empty((it - 1) % ST), ((it - 1) / ST) & 1, g, 4)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tST, desc_k<D>(sK, kk), desc_k<D>(sQ(s), kk), kIdS, kk > 0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tDPT, desc_k<D>(sV, kk), desc_k<D>(sdO(s), kk), kIdS, kk > 0);
        tc_commit(st_full);
        if (!wait_bounded(pds_full, it & 1, g, 5)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          mma_ts(tdV, tST + 8u * kk, desc_mn<D>(sdO(s), kk), kIdG, (it > 0 || kk > 0));
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          mma_ts(tdK, tDPT + 8u * kk, desc_mn<D>(sQ(s), kk), kIdG, (it > 0 || kk > 0));
        tc_commit(q_empty(s));
      }
      tc_commit(acc_done);
      tc_commit(drain);
      drain_wait(drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------- P^T / dS^T (thread = key row)
    const int t = threadIdx.x;
    const int c = k0 + t;  // key position owned by this thread
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int it = 0; it < n; ++it) {
      const int s = it % ST;
      const int i = i_lo + it;
      const int r0 = i * kRows;
      if (!wait_bounded_warp(st_full, it & 1, g, 6)) { ok = false; break; }
      if (!wait_bounded_warp(q_full(s), (it / ST) & 1, g, 7)) { ok = false; break; }
      tc_fence_after();
      const float* lse2 = vec + s * 3 * kRows;
      const float* dl = lse2 + kRows;
      const int* dsq = reinterpret_cast<const int*>(dl + kRows);
      // no mask needed when every query row of the tile is strictly below this key
      // and its document starts at or before it
      const bool full = (i > jt) && (dsq[kRows - 1] <= c);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t sr[32], dr[32];
        tmem_ld32(tST + lane_off + 32u * cc, sr);
        tmem_ld32(tDPT + lane_off + 32u * cc, dr);
        tc_wait_ld();
        reg_fence(sr);
        reg_fence(dr);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float pv[2], dv[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int rl = 32 * cc + 2 * e + h;
            float pr = ex2(__uint_as_float(sr[2 * e + h]) * sl2 - lse2[rl]);
            if (!full) {
              const int r = r0 + rl;
              if (c > r || c < dsq[rl]) pr = 0.f;
            }
            pv[h] = pr;
            dv[h] = pr * (__uint_as_float(dr[2 * e + h]) - dl[rl]);
          }
          pk[e] = pack_bf16(pv[0], pv[1]);
          dk[e] = pack_bf16(dv[0], dv[1]);
        }
        tmem_st16(tST + lane_off + 16u * cc, pk);
        tmem_st16(tDPT + lane_off + 16u * cc, dk);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pds_full);
    }
    if (ok && wait_bounded_warp(acc_done, 0, g, 8)) {
      tc_fence_after();
      __nv_bfloat16* dk_row = p.g0 + ((size_t)bh * T + c) * D;
      __nv_bfloat16* dv_row = p.g1 + ((size_t)bh * T + c) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tdV + lane_off + 32u * cc, r);
        tc_wait_ld();
        reg_fence(r);
        if (c < T) store_row_chunk_bf16(dv_row + 32 * cc, r, 1.0f);
        tmem_ld32(tdK + lane_off + 32u * cc, r);
        tc_wait_ld();
        reg_fence(r);
        if (c < T) store_row_chunk_bf16(dk_row + 32 * cc, r, p.scale);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// --------------------------------------------------------------------- dQ
template <int D>
struct DqLayout {
  static constexpr int ST = (D == 128) ? 2 : 3;   // K/V ring depth
  static constexpr int Q_OFF = 0;
  static constexpr int DO_OFF = Q_OFF + Tile<D>::BYTES;
  static constexpr int K_OFF = DO_OFF + Tile<D>::BYTES;           // + s * BYTES
  static constexpr int V_OFF = K_OFF + ST * Tile<D>::BYTES;       // + s * BYTES
  static constexpr int BAR_OFF = V_OFF + ST * Tile<D>::BYTES;
  // barriers: qdo_full | kv_full[ST] | kv_empty[ST] | s_full | ds_full | acc_done | drain
  static constexpr int NBAR = 1 + 2 * ST + 4;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int SMEM = BYTES + 1024;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmdO, const BwdParams p) {
  using Tl = Tile<D>;
  using L = DqLayout<D>;
  constexpr int ST = L::ST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* gsm;
  const uint32_t sbase = aligned_smem_base(smem_raw, &gsm);
  const uint32_t sQ = sbase + L::Q_OFF, sdO = sbase + L::DO_OFF;
  auto sK = [&](int s) { return sbase + L::K_OFF + s * Tl::BYTES; };
  auto sV = [&](int s) { return sbase + L::V_OFF + s * Tl::BYTES; };
  const uint32_t bar0 = sbase + L::BAR_OFF;
  const uint32_t qdo_full = bar0;
  auto kv_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (1 + ST + s); };
  const uint32_t s_full = bar0 + 8u * (1 + 2 * ST);
  const uint32_t ds_full = bar0 + 8u * (2 + 2 * ST);
  const uint32_t acc_done = bar0 + 8u * (3 + 2 * ST);
  const uint32_t drain = bar0 + 8u * (4 + 2 * ST);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gsm + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gsm + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  const int qt = p.n_t - 1 - (int)(blockIdx.x / p.BH);
  const int bh = (int)(blockIdx.x % p.BH);
  const int b = bh / p.H;
  const int q0 = qt * kRows;
  int kv_lo = 0;
  if (p.doc) {
    kv_lo = p.doc[(size_t)b * T + q0] / kRows;
    kv_lo = kv_lo < 0 ? 0 : (kv_lo > qt ? qt : kv_lo);
  }
  const int n = qt - kv_lo + 1;

  if (threadIdx.x == 0) {
    mbar_init(qdo_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(ds_full, 4);
    mbar_init(acc_done, 1);
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
  const uint32_t tS = tmem, tDP = tmem + 128, tdQ = tmem + 256;

  if (warp == 4) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      mbar_arrive_expect_tx(qdo_full, 2 * Tl::BYTES);
      load_tile<D>(sQ, &tmQ, q0, bh, qdo_full);
      load_tile<D>(sdO, &tmdO, q0, bh, qdo_full);
      int it = 0;
      for (; it < n; ++it) {
        const int s = it % ST, u = it / ST;
        if (u > 0 && !wait_bounded(kv_empty(s), (u - 1) & 1, g, 1)) break;
        const int row = (kv_lo + it) * kRows;
        mbar_arrive_expect_tx(kv_full(s), 2 * Tl::BYTES);
        load_tile<D>(sK(s), &tmK, row, bh, kv_full(s));
        load_tile<D>(sV(s), &tmV, row, bh, kv_full(s));
      }
      if (*abort_flag) {
        drain_wait(qdo_full, 0, p.wait_limit_ns);
        for (int s = 0; s < ST; ++s) {
          const int cnt = it > s ? (it - s + ST - 1) / ST : 0;
          if (cnt > 0) drain_wait(kv_full(s), (cnt - 1) & 1, p.wait_limit_ns);
        }
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t kIdG = idesc_bf16_f32(128, D, true);
      bool ok = wait_bounded(qdo_full, 0, g, 2);
      for (int it = 0; ok && it < n; ++it) {
        const int s = it % ST;
        if (!wait_bounded(kv_full(s), (it / ST) & 1, g, 3)) break;
        // S / dP overwrite the dS that the previous dQ MMA read
        if (it > 0 && !wait_bounded(kv_empty((it - 1) % ST), ((it - 1) / ST) & 1, g, 4)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tS, desc_k<D>(sQ, kk), desc_k<D>(sK(s), kk), kIdS, kk > 0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tDP, desc_k<D>(sdO, kk), desc_k<D>(sV(s), kk), kIdS, kk > 0);
        tc_commit(s_full);
        if (!wait_bounded(ds_full, it & 1, g, 5)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          mma_ts(tdQ, tDP + 8u * kk, desc_mn<D>(sK(s), kk), kIdG, (it > 0 || kk > 0));
        tc_commit(kv_empty(s));
      }
      tc_commit(acc_done);
      tc_commit(drain);
      drain_wait(drain, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else {
    const int t = threadIdx.x;
    const int r = q0 + t;  // query position owned by this thread
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    const float lse2 = (r < T) ? p.lse[(size_t)bh * T + r] * kLog2e : INFINITY;
    const float dlt = (r < T) ? p.delta[(size_t)bh * T + r] : 0.f;
    const int ds = p.doc ? p.doc[(size_t)b * T + (r < T ? r : T - 1)] : 0;
    bool ok = true;
    for (int it = 0; it < n; ++it) {
      const int j = kv_lo + it;
      if (!wait_bounded_warp(s_full, it & 1, g, 6)) { ok = false; break; }
      tc_fence_after();
      const bool full = (j < qt) && (j * kRows >= ds);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t sr[32], dr[32];
        tmem_ld32(tS + lane_off + 32u * cc, sr);
        tmem_ld32(tDP + lane_off + 32u * cc, dr);
        tc_wait_ld();
        reg_fence(sr);
        reg_fence(dr);
        uint32_t dk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float dv[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float pr = ex2(__uint_as_float(sr[2 * e + h]) * sl2 - lse2);
            if (!full) {
              const int col = j * kRows + 32 * cc + 2 * e + h;
              if (col > r || col < ds) pr = 0.f;
            }
            dv[h] = pr * (__uint_as_float(dr[2 * e + h]) - dlt);
          }
          dk[e] = pack_bf16(dv[0], dv[1]);
        }
        tmem_st16(tDP + lane_off + 16u * cc, dk);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full);
    }
    if (ok && wait_bounded_warp(acc_done, 0, g, 8)) {
      tc_fence_after();
      __nv_bfloat16* dq_row = p.g0 + ((size_t)bh * T + r) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(tdQ + lane_off + 32u * cc, v);
        tc_wait_ld();
        reg_fence(v);
        if (r < T) store_row_chunk_bf16(dq_row + 32 * cc, v, p.scale);
      }
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
