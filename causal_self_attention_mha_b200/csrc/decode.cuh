// decode.cuh -- KV-cache decode attention on sm_100a.
//
// Generation appends Tq new tokens (1 in plain decoding, a few with
// speculative drafts) to a cache of L keys and values and attends from each new
// token to every cached position up to its own: query t sits at position
// L - Tq + t and sees keys 0 .. L - Tq + t (the causal rule of the training
// forward, restricted to the last Tq rows).  The pages' inference path
// ("How to build an LLM by hand", agmtopy.github.io, section 2: nanochat's
// engine keeps a KV cache and calls FlashAttention-3's kv-cache entry point on
// (B, T, H, D) tensors) is what this reproduces; the cache uses that layout.
//
// The work is one pass over the cache, so HBM bandwidth bounds it: each CTA
// takes one 128-key chunk of one (batch, head), brings the chunk's K and V
// rows in by TMA (128-byte swizzle), and computes, for every new token, the
// chunk's scores, their maximum, the sum of their exponentials and the
// unnormalised weighted sum of V rows.  With one new token that is a
// matrix-vector product, done on CUDA cores (one key row or one output column
// per thread, conflict-free shared-memory reads thanks to the swizzle); with
// two or more the arithmetic per cache byte outgrows the CUDA cores and the
// chunk kernel runs its two products on the tensor cores instead
// (attn_decode_chunk_tc_kernel).  A second kernel merges the chunks of each
// (batch, head, token) in chunk order -- deterministic, no atomics.
#pragma once

#include "tiles.cuh"

namespace ca {

constexpr int kDecChunk = 128;   // keys per CTA (one TMA box of rows)
constexpr int kDecThreads = 128; // CUDA-core chunk kernel: a thread per key row
constexpr int kDecMaxTq = 16;    // new tokens per call
constexpr int kDecTcMinTq = 2;   // from this many new tokens on, the tensor-core chunk kernel

struct DecParams {
  const __nv_bfloat16* q;  // [B, Tq, H, D]
  float* part_ml;          // [B, H, Tq, n_chunks, 2]: chunk max (base 2) and sum of 2^(s - max)
  float* part_o;           // [B, H, Tq, n_chunks, D]: unnormalised sum of weights x V rows
  int B, H, Tq, L, n_chunks;
  float scale_log2;        // scale * log2(e)
  uint64_t wait_limit_ns;
};

// Shared memory of the CUDA-core chunk kernel (one new token).
template <int D>
struct DecLayout {
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = Tile<D>::BYTES;
  static constexpr int Q_OFF = 2 * Tile<D>::BYTES;                 // fp32 [D], times scale*log2e
  static constexpr int P_OFF = Q_OFF + D * 4;                      // fp32 [128] weights
  static constexpr int RED_OFF = P_OFF + kDecChunk * 4;            // fp32 [2][4] warp partials
  static constexpr int G = kDecThreads / D;                        // key groups in the V pass
  static constexpr int ACC_OFF = RED_OFF + 2 * 4 * 4;              // fp32 [G][D] group sums
  static constexpr int BAR_OFF = ACC_OFF + (G > 1 ? G * D * 4 : 0);  // K landed, V landed
  static constexpr int MISC_OFF = BAR_OFF + 16;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int SMEM = BYTES + 1024;
};

// An L2 cache policy that marks the lines an access brings in as first to evict: for data
// read exactly once (a KV cache streamed past), so that it does not push out lines that will
// be read again soon.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 4-D tiled load with an L2 cache policy (from createpolicy), otherwise as tma_load_4d.
__device__ __forceinline__ void tma_load_4d_hint(uint32_t dst, const CUtensorMap* m, int c0,
                                                 int c1, int c2, int c3, uint32_t bar,
                                                 uint64_t policy) {
  if (!tma_coords_ok(c0, c1 | c3)) return;
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar),
      "l"(policy)
      : "memory");
}

// Element (row r, column col) of a staged 128-row tile (the layout load_tile produces).
template <int D>
__device__ __forceinline__ uint32_t tile_elem_offset(int r, int col) {
  using Tl = Tile<D>;
  const int ch = col / Tl::BOX_COLS, cu = (col % Tl::BOX_COLS) / 8;
  const int phys = (Tl::SW == 128) ? (cu ^ (r & 7)) : (cu ^ ((r >> 1) & 3));
  return (uint32_t)(ch * Tl::CHUNK_BYTES + r * Tl::SW + phys * 16 + (col % 8) * 2);
}

// Max or sum of v over the CTA's 4 warps (through `red`, 4 floats); every thread gets it.
__device__ __forceinline__ float dec_block_reduce(float v, bool is_max, float* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, v, off);
    v = is_max ? fmaxf(v, o) : v + o;
  }
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  const float4 r = *reinterpret_cast<const float4*>(red);
  return is_max ? fmaxf(fmaxf(r.x, r.y), fmaxf(r.z, r.w)) : (r.x + r.y) + (r.z + r.w);
}

// One new token, on CUDA cores.  One CTA: one 128-key chunk of one (batch, head); thread kr
// scores key row kr, then a thread per output column (in G groups of keys for d < 128)
// sums weights times V.
template <int D>
__global__ void __launch_bounds__(kDecThreads)
    attn_decode_chunk_kernel(const __grid_constant__ CUtensorMap tmK,
                             const __grid_constant__ CUtensorMap tmV, const DecParams p) {
  using Tl = Tile<D>;
  using L = DecLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* gsm;
  const uint32_t sbase = aligned_smem_base(smem_raw, &gsm);
  const uint8_t* sK = gsm + L::K_OFF;
  const uint8_t* sV = gsm + L::V_OFF;
  float* qs = reinterpret_cast<float*>(gsm + L::Q_OFF);
  float* ps = reinterpret_cast<float*>(gsm + L::P_OFF);
  float* red = reinterpret_cast<float*>(gsm + L::RED_OFF);
  float* acc_s = reinterpret_cast<float*>(gsm + L::ACC_OFF);
  const uint32_t bar_k = sbase + L::BAR_OFF, bar_v = bar_k + 8u;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gsm + L::MISC_OFF);

  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(bar_k, 1);
    mbar_init(bar_v, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {  // this chunk's 128 key and value rows of head h (rows past L read as zero)
    const uint64_t pol = l2_policy_evict_first();  // read once: first out of L2
    mbar_arrive_expect_tx(bar_k, Tl::BYTES);
    mbar_arrive_expect_tx(bar_v, Tl::BYTES);
#pragma unroll
    for (int ch = 0; ch < Tl::CHUNKS; ++ch)
      tma_load_4d_hint(sbase + L::K_OFF + ch * Tl::CHUNK_BYTES, &tmK, ch * Tl::BOX_COLS, h,
                       c * kDecChunk, b, bar_k, pol);
#pragma unroll
    for (int ch = 0; ch < Tl::CHUNKS; ++ch)
      tma_load_4d_hint(sbase + L::V_OFF + ch * Tl::CHUNK_BYTES, &tmV, ch * Tl::BOX_COLS, h,
                       c * kDecChunk, b, bar_v, pol);
  }
  // the query, times scale * log2(e), while the rows arrive (q is [B, 1, H, D])
  for (int i = tid; i < D; i += kDecThreads)
    qs[i] = __bfloat162float(p.q[((size_t)b * p.H + h) * D + i]) * p.scale_log2;
  const Guard g{abort_flag, p.wait_limit_ns};
  // the scores need only K: V keeps landing while they are computed
  const bool ok = wait_bounded(bar_k, 0, g, 1);
  __syncthreads();  // qs complete; the outcome of the wait is uniform after this point
  if (!ok || *abort_flag) {
    if (tid == 0) {
      drain_wait(bar_k, 0, p.wait_limit_ns);
      drain_wait(bar_v, 0, p.wait_limit_ns);
    }
    return;
  }

  // the score of my key row (base 2; -inf past the cache: the token sees keys 0 .. L - 1)
  const int kr = tid, j = c * kDecChunk + kr;
  float s = 0.f;
#pragma unroll
  for (int u = 0; u < D / 8; ++u) {
    const uint4 kv = *reinterpret_cast<const uint4*>(sK + tile_elem_offset<D>(kr, 8 * u));
    const float4 q0 = *reinterpret_cast<const float4*>(qs + 8 * u);
    const float4 q1 = *reinterpret_cast<const float4*>(qs + 8 * u + 4);
    s = fmaf(bf16_lo(kv.x), q0.x, s);
    s = fmaf(bf16_hi(kv.x), q0.y, s);
    s = fmaf(bf16_lo(kv.y), q0.z, s);
    s = fmaf(bf16_hi(kv.y), q0.w, s);
    s = fmaf(bf16_lo(kv.z), q1.x, s);
    s = fmaf(bf16_hi(kv.z), q1.y, s);
    s = fmaf(bf16_lo(kv.w), q1.z, s);
    s = fmaf(bf16_hi(kv.w), q1.w, s);
  }
  if (j > p.L - 1) s = -INFINITY;
  const float m = dec_block_reduce(s, true, red);
  const float w = (s == -INFINITY) ? 0.f : ex2(s - m);
  ps[kr] = w;
  const float lsum = dec_block_reduce(w, false, red + 4);  // the chunk's sum of weights
  // V must have landed before the weighted sums (ps is complete after the reduction's barrier)
  {
    const bool vok = wait_bounded(bar_v, 0, g, 2);
    __syncthreads();
    if (!vok || *abort_flag) {
      if (tid == 0) drain_wait(bar_v, 0, p.wait_limit_ns);
      return;
    }
  }
  // my column of V over my group's keys
  const int col = tid % D, grp = tid / D;
  constexpr int KPG = kDecChunk / L::G;
  float acc = 0.f;
#pragma unroll 4
  for (int k = grp * KPG; k < (grp + 1) * KPG; ++k) {
    const uint16_t bits = *reinterpret_cast<const uint16_t*>(sV + tile_elem_offset<D>(k, col));
    acc = fmaf(ps[k], __uint_as_float((uint32_t)bits << 16), acc);
  }
  if (L::G > 1) {
    acc_s[grp * D + col] = acc;
    __syncthreads();
    if (grp == 0)
      for (int gg = 1; gg < L::G; ++gg) acc += acc_s[gg * D + col];
  }
  const size_t row = (((size_t)b * p.H + h) * p.Tq) * p.n_chunks + c;  // Tq = 1
  if (grp == 0) p.part_o[row * D + col] = acc;
  if (tid == 0) {  // the chunk maximum and sum
    p.part_ml[row * 2] = m;
    p.part_ml[row * 2 + 1] = lsum;
  }
}

// Tensor-core form of the chunk kernel for two or more new tokens.  With Tq tokens a cached
// key row (2d bytes of K and of V) feeds 4 d Tq flops, so from Tq = 4 or so the CUDA-core
// form runs out of arithmetic before HBM runs out of bandwidth (~16 flops per cache byte at
// Tq = 16, above the fp32 rate per byte the B200 can stream).  Here the chunk's scores
// S = Q K^T and its weighted sum P V are two chains of tcgen05 MMAs with M = 128 whose rows
// 0 .. 15 are the new tokens (rows past Tq are zero queries; the A-operand rows past the 32
// stored query rows or the 16 stored weight rows are whatever lies behind them in shared
// memory, and their results are never read).  Warp 0 does the rest: lane 0 issues the
// MMAs; the query rows are stored twice
// (rows 16 .. 31 repeat rows 0 .. 15), so token t's scores are in TMEM lanes t and t + 16,
// and lane t takes keys 0 .. 63, lane t + 16 keys 64 .. 127 (row maximum and sums combined
// with one shuffle).  Each lane writes its 64 weights, packed bf16, into row t of the P
// operand in shared memory (over the query tile and the K tile, both read by then), so P V
// is a single shared-memory MMA chain with N = d, accumulating over S's TMEM columns.  The
// partial output is scaled by (sum of the fp32 weights) / (sum of the bf16-rounded weights
// the MMA multiplied), so that the merge, which weighs chunks by the fp32 sums, normalises
// each chunk by the weights actually used, as the training forward does.  A CTA needs 128
// TMEM columns and, at d = 128, 73 KB of shared memory: three CTAs share an SM and overlap
// one another's loads and chains.
template <int D>
struct DecTcLayout {
  static constexpr int QROWS = 32;                      // tokens 0 .. 15, twice
  static constexpr int QCH = QROWS * Tile<D>::SW;       // one swizzle chunk of the query rows
  static constexpr int PCH = 16 * 128;                  // one 64-key chunk of the P rows
  static constexpr int Q_OFF = 0;                       // bf16 [32][D], rows of tokens >= Tq zero
  static constexpr int P_OFF = 0;                       // bf16 [16][128 keys], after S is done
  static constexpr int K_OFF = Tile<D>::CHUNKS * QCH;   // 1024-byte multiple
  static constexpr int V_OFF = K_OFF + Tile<D>::BYTES;
  static constexpr int BAR_OFF = V_OFF + Tile<D>::BYTES;  // K landed, V landed, S done, PV done
  static constexpr int MISC_OFF = BAR_OFF + 32;           // TMEM base slot, abort flag
  static constexpr int BYTES = MISC_OFF + 16;
  // below d = 128 the dynamic shared memory is padded so that at most four CTAs share an SM:
  // four TMEM allocations of 128 columns fill its 512
  static constexpr int SMEM = (D == 128) ? BYTES + 1024 : (BYTES + 1024 > 56 * 1024 ? BYTES + 1024 : 56 * 1024);
  static constexpr int THREADS = 128;
  static constexpr uint32_t TMEM_COLS = 128u;           // S, then O over its first d columns
  // what the 128-row operands read stays inside this CTA's shared memory, and P stays clear
  // of V (still needed when P is written)
  static_assert((Tile<D>::CHUNKS - 1) * QCH + kRows * Tile<D>::SW <= BAR_OFF, "query operand");
  static_assert(PCH + kRows * 128 <= BAR_OFF && 2 * PCH <= V_OFF, "weight operand");
};

// Byte offset of element (r, col), r < 32, of the query operand.
template <int D>
__device__ __forceinline__ uint32_t qtile_elem_offset(int r, int col) {
  using Tl = Tile<D>;
  const int ch = col / Tl::BOX_COLS, cu = (col % Tl::BOX_COLS) / 8;
  const int phys = (Tl::SW == 128) ? (cu ^ (r & 7)) : (cu ^ ((r >> 1) & 3));
  return (uint32_t)(ch * DecTcLayout<D>::QCH + r * Tl::SW + phys * 16 + (col % 8) * 2);
}

// K-major descriptor of the query operand for MMA-K step kk (16 columns of d).
template <int D>
__device__ __forceinline__ uint64_t qdesc_k(uint32_t tile, int kk) {
  using Tl = Tile<D>;
  const uint32_t byte = (uint32_t)kk * 32u;
  const uint32_t addr = tile + (byte / Tl::SW) * DecTcLayout<D>::QCH + (byte % Tl::SW);
  return sdesc(addr, 16u, 8u * Tl::SW, Tl::LAYOUT);
}

// K-major descriptor of the weight operand (keys along K, 64-key chunks of 128-byte rows,
// 128-byte swizzle) for MMA-K step kk (16 keys).
template <int D>
__device__ __forceinline__ uint64_t pdesc_k(uint32_t tile, int kk) {
  const uint32_t byte = (uint32_t)kk * 32u;
  const uint32_t addr = tile + (byte / 128u) * DecTcLayout<D>::PCH + (byte % 128u);
  return sdesc(addr, 16u, 8u * 128u, 2u);
}

template <int D>
__global__ void __launch_bounds__(128)
    attn_decode_chunk_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                                const __grid_constant__ CUtensorMap tmV, const DecParams p) {
  using Tl = Tile<D>;
  using L = DecTcLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* gsm;
  const uint32_t sbase = aligned_smem_base(smem_raw, &gsm);
  if (sbase - smem_u32(smem_raw) + L::BYTES > dynamic_smem_bytes()) {
    if (threadIdx.x == 0) report_smem_shortfall();
    return;
  }
  const uint32_t sK = sbase + L::K_OFF, sV = sbase + L::V_OFF, sQ = sbase + L::Q_OFF,
                 sP = sbase + L::P_OFF;
  const uint32_t bar_k = sbase + L::BAR_OFF, bar_v = bar_k + 8u, bar_s = bar_k + 16u,
                 bar_o = bar_k + 24u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gsm + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gsm + L::MISC_OFF + 4);

  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Tq = p.Tq;
  if (tid == 0) {
    mbar_init(bar_k, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    *abort_flag = 0;
    fence_barrier_init();
    // this chunk's 128 key and value rows of head h (rows past L read as zero), read once:
    // first out of L2, so that the chunk partials stay there for the merge
    const uint64_t pol = l2_policy_evict_first();
    mbar_arrive_expect_tx(bar_k, Tl::BYTES);
    mbar_arrive_expect_tx(bar_v, Tl::BYTES);
#pragma unroll
    for (int ch = 0; ch < Tl::CHUNKS; ++ch)
      tma_load_4d_hint(sK + ch * Tl::CHUNK_BYTES, &tmK, ch * Tl::BOX_COLS, h, c * kDecChunk, b,
                       bar_k, pol);
#pragma unroll
    for (int ch = 0; ch < Tl::CHUNKS; ++ch)
      tma_load_4d_hint(sV + ch * Tl::CHUNK_BYTES, &tmV, ch * Tl::BOX_COLS, h, c * kDecChunk, b,
                       bar_v, pol);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  // the query rows: rows t and t + 16 hold new token t's query (bf16, as given), zero past Tq
  for (int i = tid; i < L::QROWS * (D / 8); i += L::THREADS) {
    const int r = i / (D / 8), u = i % (D / 8), t = r & 15;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (t < Tq)
      v = *reinterpret_cast<const uint4*>(p.q + (((size_t)b * Tq + t) * p.H + h) * D + 8 * u);
    *reinterpret_cast<uint4*>(gsm + L::Q_OFF + qtile_elem_offset<D>(r, 8 * u)) = v;
  }
  fence_proxy_async_smem();  // the MMA reads the tile through the async proxy
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Guard g{abort_flag, p.wait_limit_ns};

  if (warp == 0) {
    bool issued_s = false, issued_o = false;
    bool ok = true;
    if (lane == 0) {
      ok = wait_bounded(bar_k, 0, g, 1);
      if (ok) {
        tc_fence_after();
        constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem, qdesc_k<D>(sQ, kk), desc_k<D>(sK, kk), kIdS, kk > 0);
        tc_commit(bar_s);
        issued_s = true;
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0) && wait_bounded_warp(bar_s, 0, g, 2);
    const int t = lane & 15, hh = lane >> 4;  // my token, my half of the chunk's keys
    float m = -INFINITY, l = 0.f, lr = 0.f;
    if (ok) {
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(tmem + 32u * q4, sr[q4]);
      tc_wait_ld();
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) reg_fence(sr[q4]);
      // keys e (in my half: 64 hh + e) <= vis are visible to token t
      const int vis = p.L - Tq + t - c * kDecChunk - 64 * hh;
      uint32_t s64[64];
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < 64; ++e) {
        const uint32_t v = hh ? sr[2 + (e >> 5)][e & 31] : sr[e >> 5][e & 31];
        s64[e] = (e > vis) ? 0xFF800000u : v;  // -inf past the token's position
        mx = fmaxf(mx, __uint_as_float(s64[e]));
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      m = mx * p.scale_log2;
      const float mu = (m == -INFINITY) ? 0.f : m;
      const uint64_t sl2x2 = f2(p.scale_log2, p.scale_log2), nmu2 = f2(-mu, -mu);
      uint64_t acc_l = f2(0.f, 0.f), acc_lr = f2(0.f, 0.f);
      uint32_t pk[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float2 xx = f2split(ffma2(f2u(s64[2 * e], s64[2 * e + 1]), sl2x2, nmu2));
        const float w0 = ex2(xx.x), w1 = ex2(xx.y);
        const uint32_t v = pack_bf16(w0, w1);
        acc_l = fadd2(acc_l, f2(w0, w1));
        acc_lr = fadd2(acc_lr, bf16x2_to_f2(v));
        pk[e] = v;
      }
      const float2 a = f2split(acc_l), ar = f2split(acc_lr);
      l = a.x + a.y;
      lr = ar.x + ar.y;
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      lr += __shfl_xor_sync(0xffffffffu, lr, 16);
      // my 64 weights: row t of the weight operand, 64-key chunk hh (16-byte units swizzled
      // with the row); S has been read into registers, so the query tile may be overwritten
      uint8_t* prow = gsm + L::P_OFF + hh * L::PCH + t * 128;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        *reinterpret_cast<uint4*>(prow + ((u ^ (t & 7)) * 16)) =
            make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
    }
    __syncwarp();
    if (lane == 0 && ok) {
      ok = wait_bounded(bar_v, 0, g, 3);
      if (ok) {
        tc_fence_after();
        constexpr uint32_t kIdO = idesc_bf16_f32(128, D, true);
#pragma unroll
        for (int kk = 0; kk < kDecChunk / 16; ++kk)
          mma_ss(tmem, pdesc_k<D>(sP, kk), desc_mn<D>(sV, kk), kIdO, kk > 0);
        tc_commit(bar_o);
        issued_o = true;
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0) && wait_bounded_warp(bar_o, 0, g, 4);
    if (ok) {
      tc_fence_after();
      const float fix = lr > 0.f ? l / lr : 0.f;  // fp32 over rounded weight sum (0: no key)
      const bool mine = lane < Tq;                // lanes 0 .. Tq-1 hold the tokens' O rows
      const size_t row = (((size_t)b * p.H + h) * Tq + (mine ? lane : 0)) * p.n_chunks + c;
#pragma unroll
      for (int w2 = 0; w2 < D / 32; ++w2) {
        uint32_t r[32];
        tmem_ld32(tmem + 32u * w2, r);
        tc_wait_ld();
        reg_fence(r);
        if (mine) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(p.part_o + row * D + 32 * w2 + e) =
                make_float4(__uint_as_float(r[e]) * fix, __uint_as_float(r[e + 1]) * fix,
                            __uint_as_float(r[e + 2]) * fix, __uint_as_float(r[e + 3]) * fix);
        }
      }
      if (mine) {
        p.part_ml[row * 2] = m;
        p.part_ml[row * 2 + 1] = l;
      }
    }
    if (lane == 0) {  // after a failed wait: no copy or MMA of this CTA may still be in flight
      if (!ok) {
        drain_wait(bar_k, 0, p.wait_limit_ns);
        drain_wait(bar_v, 0, p.wait_limit_ns);
        if (issued_s) drain_wait(bar_s, 0, p.wait_limit_ns);
        if (issued_o) drain_wait(bar_o, 0, p.wait_limit_ns);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// Merges the chunks of one (batch, head, token).  kCombWarps warps each fold a fixed
// slice of the chunks (chunk order within the slice), lane l holding columns
// l*VEC .. l*VEC + VEC - 1; the warps' results are then folded in warp order.  The
// order is fixed, so the result is deterministic.  Every chunk's partial output is
// finite (zero for a chunk without visible keys), so weight-zero chunks add nothing.
constexpr int kCombWarps = 8;

template <int D>
__global__ void __launch_bounds__(kCombWarps * 32)
    attn_decode_combine_kernel(const float* __restrict__ part_ml, const float* __restrict__ part_o,
                               __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int H,
                               int Tq, int n_chunks) {
  constexpr int VEC = D / 32;  // columns per lane
  __shared__ float sm_m[kCombWarps], sm_l[kCombWarps];
  __shared__ float sm_o[kCombWarps][D];
  const int idx = blockIdx.x;  // ((b * H) + h) * Tq + t
  const int t = idx % Tq, bh = idx / Tq, h = bh % H, b = bh / H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* ml = part_ml + (size_t)idx * n_chunks * 2;
  const float* po = part_o + (size_t)idx * n_chunks * D;
  const int per = (n_chunks + kCombWarps - 1) / kCombWarps;
  const int c0 = warp * per, c1 = min(n_chunks, c0 + per);
  // The slice is taken 32 chunks at a time: lane j loads chunk j's (m, l), the group's
  // maximum and weights follow from shuffles, then the group's partial outputs are loaded
  // without waiting on one another and summed in chunk order.
  float M = -INFINITY, l = 0.f, acc[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
  for (int g0 = c0; g0 < c1; g0 += 32) {
    const int c = g0 + lane;
    const float mc = c < c1 ? ml[2 * c] : -INFINITY;
    const float lc = c < c1 ? ml[2 * c + 1] : 0.f;
    float mg = mc;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mg = fmaxf(mg, __shfl_xor_sync(0xffffffffu, mg, off));
    if (mg == -INFINITY) continue;  // no visible key in the whole group (warp-uniform)
    const float mn = fmaxf(M, mg);
    const float fo = ex2(M - mn);  // ex2(-inf) = 0 before the first group
    const float fc = (mc == -INFINITY) ? 0.f : ex2(mc - mn);
    float lg = lc * fc;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lg += __shfl_xor_sync(0xffffffffu, lg, off);
    l = l * fo + lg;
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] *= fo;
    const int n = min(32, c1 - g0);
#pragma unroll 8
    for (int j = 0; j < n; ++j) {
      const float fj = __shfl_sync(0xffffffffu, fc, j);
      const float* src = po + (size_t)(g0 + j) * D + lane * VEC;
      float x[VEC];
      if constexpr (VEC == 4) {
        const float4 t4 = *reinterpret_cast<const float4*>(src);
        x[0] = t4.x; x[1] = t4.y; x[2] = t4.z; x[3] = t4.w;
      } else if constexpr (VEC == 2) {
        const float2 t2 = *reinterpret_cast<const float2*>(src);
        x[0] = t2.x; x[1] = t2.y;
      } else {
        x[0] = src[0];
      }
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[v] = fmaf(x[v], fj, acc[v]);
    }
    M = mn;
  }
  if (lane == 0) {
    sm_m[warp] = M;
    sm_l[warp] = l;
  }
#pragma unroll
  for (int v = 0; v < VEC; ++v) sm_o[warp][lane * VEC + v] = acc[v];
  __syncthreads();
  if (warp == 0) {
    float Mt = -INFINITY;
#pragma unroll
    for (int w = 0; w < kCombWarps; ++w) Mt = fmaxf(Mt, sm_m[w]);
    float lt = 0.f, ot[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) ot[v] = 0.f;
#pragma unroll
    for (int w = 0; w < kCombWarps; ++w) {
      if (sm_m[w] == -INFINITY) continue;
      const float f = ex2(sm_m[w] - Mt);
      lt = fmaf(sm_l[w], f, lt);
#pragma unroll
      for (int v = 0; v < VEC; ++v) ot[v] = fmaf(sm_o[w][lane * VEC + v], f, ot[v]);
    }
    const float inv = 1.0f / lt;
    __nv_bfloat16* orow = o + (((size_t)b * Tq + t) * H + h) * D;
#pragma unroll
    for (int v = 0; v < VEC; ++v) orow[lane * VEC + v] = __float2bfloat16_rn(ot[v] * inv);
    if (lane == 0) lse[idx] = (Mt + lg2(lt)) * kLn2;
  }
}

}  // namespace ca
