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
// The work is one pass over the cache, so the kernel is bound by HBM
// bandwidth, not by arithmetic: each CTA takes one 128-key chunk of one
// (batch, head), brings the chunk's K and V rows in by TMA (128-byte swizzle,
// so that a thread per key row and a thread per column both read shared
// memory without bank conflicts), and computes, for every new token, the
// chunk's scores, their maximum, the sum of their exponentials and the
// unnormalised weighted sum of V rows on CUDA cores (one key row or one
// output column per thread).  A second kernel merges the chunks of each
// (batch, head, token) in chunk order -- deterministic, no atomics.
#pragma once

#include "tiles.cuh"

namespace ca {

constexpr int kDecChunk = 128;   // keys per CTA (one TMA box of rows)
constexpr int kDecThreads = 128;
// Threads of a chunk CTA: one token, a thread per key row; several tokens, two threads per key
// row (each taking half of the tokens in the score pass) -- the multi-token path is bound by
// shared-memory and L1 latency, and twice the warps hide twice as much of it.
template <int TQM>
constexpr int dec_threads() { return TQM > 1 ? 2 * kDecThreads : kDecThreads; }
constexpr int kDecMaxTq = 16;    // new tokens per call

struct DecParams {
  const __nv_bfloat16* q;  // [B, Tq, H, D]
  float* part_ml;          // [B, H, Tq, n_chunks, 2]: chunk max (base 2) and sum of 2^(s - max)
  float* part_o;           // [B, H, Tq, n_chunks, D]: unnormalised sum of weights x V rows
  int B, H, Tq, L, n_chunks;
  float scale_log2;        // scale * log2(e)
  uint64_t wait_limit_ns;
};

template <int D, int TQM>
struct DecLayout {
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = Tile<D>::BYTES;
  static constexpr int Q_OFF = 2 * Tile<D>::BYTES;                 // fp32 [TQM][D], times scale*log2e
  static constexpr int P_OFF = Q_OFF + TQM * D * 4;                // fp32 [TQM][128] weights
  static constexpr int NT = dec_threads<TQM>();
  static constexpr int RED_OFF = P_OFF + TQM * kDecChunk * 4;      // fp32 [2][TQM][4] warp partials
  static constexpr int G = NT / D;                                 // key groups in the V pass
  static constexpr int ACC_OFF = RED_OFF + 2 * TQM * 4 * 4;        // fp32 [G][TQM][D] group sums
  static constexpr int BAR_OFF = ACC_OFF + (G > 1 ? G * TQM * D * 4 : 0);  // K landed, V landed
  static constexpr int MISC_OFF = BAR_OFF + 16;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int SMEM = BYTES + 1024;
};

// Element (row r, column col) of a staged 128-row tile (the layout load_tile produces).
template <int D>
__device__ __forceinline__ uint32_t tile_elem_offset(int r, int col) {
  using Tl = Tile<D>;
  const int ch = col / Tl::BOX_COLS, cu = (col % Tl::BOX_COLS) / 8;
  const int phys = (Tl::SW == 128) ? (cu ^ (r & 7)) : (cu ^ ((r >> 1) & 3));
  return (uint32_t)(ch * Tl::CHUNK_BYTES + r * Tl::SW + phys * 16 + (col % 8) * 2);
}

// Max or sum of v[t] (t < TQM) over the 4 warps of this thread's group of 128 threads (the
// group's own slice of `red`); every thread of the group gets the results.
template <int TQM>
__device__ __forceinline__ void dec_block_reduce(float (&v)[TQM], bool is_max, float* red) {
#pragma unroll
  for (int t = 0; t < TQM; ++t)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float o = __shfl_xor_sync(0xffffffffu, v[t], off);
      v[t] = is_max ? fmaxf(v[t], o) : v[t] + o;
    }
  const int warp = (threadIdx.x >> 5) & 3;
  if ((threadIdx.x & 31) == 0) {
#pragma unroll
    for (int t = 0; t < TQM; ++t) red[t * 4 + warp] = v[t];
  }
  __syncthreads();
#pragma unroll
  for (int t = 0; t < TQM; ++t) {
    const float4 r = *reinterpret_cast<const float4*>(red + t * 4);
    v[t] = is_max ? fmaxf(fmaxf(r.x, r.y), fmaxf(r.z, r.w)) : (r.x + r.y) + (r.z + r.w);
  }
}

// One CTA: one 128-key chunk of one (batch, head), every new token at once: each key row
// and each V element is read from shared memory once for all Tq tokens.
template <int D, int TQM>
__global__ void __launch_bounds__(dec_threads<TQM>())
    attn_decode_chunk_kernel(const __grid_constant__ CUtensorMap tmK,
                             const __grid_constant__ CUtensorMap tmV, const DecParams p) {
  using Tl = Tile<D>;
  using L = DecLayout<D, TQM>;
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
  const int Tq = p.Tq;
  if (tid == 0) {
    mbar_init(bar_k, 1);
    mbar_init(bar_v, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {  // this chunk's 128 key and value rows of head h (rows past L read as zero)
    mbar_arrive_expect_tx(bar_k, Tl::BYTES);
    mbar_arrive_expect_tx(bar_v, Tl::BYTES);
#pragma unroll
    for (int ch = 0; ch < Tl::CHUNKS; ++ch)
      tma_load_4d(sbase + L::K_OFF + ch * Tl::CHUNK_BYTES, &tmK, ch * Tl::BOX_COLS, h,
                  c * kDecChunk, b, bar_k);
#pragma unroll
    for (int ch = 0; ch < Tl::CHUNKS; ++ch)
      tma_load_4d(sbase + L::V_OFF + ch * Tl::CHUNK_BYTES, &tmV, ch * Tl::BOX_COLS, h,
                  c * kDecChunk, b, bar_v);
  }
  // the new tokens' queries, times scale * log2(e), while the rows arrive (zero past Tq)
  for (int i = tid; i < TQM * D; i += L::NT) {
    const int t = i / D, col = i % D;
    qs[i] = t < Tq ? __bfloat162float(p.q[(((size_t)b * Tq + t) * p.H + h) * D + col]) * p.scale_log2
                   : 0.f;
  }
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

  // scores of my key row against my half of the new tokens (base 2; -inf where not visible)
  constexpr int TH = TQM / (L::NT / kDecChunk);  // tokens per score thread
  const int kr = tid % kDecChunk, th = tid / kDecChunk;
  const int j = c * kDecChunk + kr;
  float s[TH];
#pragma unroll
  for (int i = 0; i < TH; ++i) s[i] = 0.f;
#pragma unroll
  for (int u = 0; u < D / 8; ++u) {
    const uint4 kv = *reinterpret_cast<const uint4*>(sK + tile_elem_offset<D>(kr, 8 * u));
    const float k8[8] = {bf16_lo(kv.x), bf16_hi(kv.x), bf16_lo(kv.y), bf16_hi(kv.y),
                         bf16_lo(kv.z), bf16_hi(kv.z), bf16_lo(kv.w), bf16_hi(kv.w)};
#pragma unroll
    for (int i = 0; i < TH; ++i) {
      const int t = th * TH + i;
      const float4 q0 = *reinterpret_cast<const float4*>(qs + t * D + 8 * u);
      const float4 q1 = *reinterpret_cast<const float4*>(qs + t * D + 8 * u + 4);
      float a = s[i];
      a = fmaf(k8[0], q0.x, a);
      a = fmaf(k8[1], q0.y, a);
      a = fmaf(k8[2], q0.z, a);
      a = fmaf(k8[3], q0.w, a);
      a = fmaf(k8[4], q1.x, a);
      a = fmaf(k8[5], q1.y, a);
      a = fmaf(k8[6], q1.z, a);
      a = fmaf(k8[7], q1.w, a);
      s[i] = a;
    }
  }
#pragma unroll
  for (int i = 0; i < TH; ++i) {  // query t sees keys 0 .. L - Tq + t
    const int t = th * TH + i;
    if (t >= Tq || j > p.L - Tq + t) s[i] = -INFINITY;
  }
  float m[TH], w[TH];
#pragma unroll
  for (int i = 0; i < TH; ++i) m[i] = s[i];
  dec_block_reduce<TH>(m, true, red + th * TH * 4);
#pragma unroll
  for (int i = 0; i < TH; ++i) {
    w[i] = (s[i] == -INFINITY) ? 0.f : ex2(s[i] - m[i]);
    ps[(th * TH + i) * kDecChunk + kr] = w[i];
  }
  // w[i] now holds the chunk's sum for token th * TH + i
  dec_block_reduce<TH>(w, false, red + TQM * 4 + th * TH * 4);
  // V must have landed before the weighted sums (ps is complete after the reduction's barrier)
  {
    const bool vok = wait_bounded(bar_v, 0, g, 2);
    __syncthreads();
    if (!vok || *abort_flag) {
      if (tid == 0) drain_wait(bar_v, 0, p.wait_limit_ns);
      return;
    }
  }
  // my column of V over my group's keys, for every token
  const int col = tid % D, grp = tid / D;
  constexpr int KPG = kDecChunk / L::G;
  float acc[TQM];
#pragma unroll
  for (int t = 0; t < TQM; ++t) acc[t] = 0.f;
#pragma unroll 4
  for (int k = grp * KPG; k < (grp + 1) * KPG; ++k) {
    const uint16_t bits = *reinterpret_cast<const uint16_t*>(sV + tile_elem_offset<D>(k, col));
    const float v = __uint_as_float((uint32_t)bits << 16);
#pragma unroll
    for (int t = 0; t < TQM; ++t) acc[t] = fmaf(ps[t * kDecChunk + k], v, acc[t]);
  }
  if (L::G > 1) {
#pragma unroll
    for (int t = 0; t < TQM; ++t) acc_s[(grp * TQM + t) * D + col] = acc[t];
    __syncthreads();
    if (grp == 0) {
      for (int gg = 1; gg < L::G; ++gg)
#pragma unroll
        for (int t = 0; t < TQM; ++t) acc[t] += acc_s[(gg * TQM + t) * D + col];
    }
  }
#pragma unroll
  for (int t = 0; t < TQM; ++t) {
    if (t >= Tq) break;
    const size_t row = (((size_t)b * p.H + h) * Tq + t) * p.n_chunks + c;
    if (grp == 0) p.part_o[row * D + col] = acc[t];
  }
  if (kr == 0) {  // the chunk maximum and sum of this half's tokens
#pragma unroll
    for (int i = 0; i < TH; ++i) {
      const int t = th * TH + i;
      if (t >= Tq) break;
      const size_t row = (((size_t)b * p.H + h) * Tq + t) * p.n_chunks + c;
      p.part_ml[row * 2] = m[i];
      p.part_ml[row * 2 + 1] = w[i];
    }
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
