// tiles.cuh -- tile geometry shared by the attention kernels.
//
// Every operand tile is 128 rows of one head's [T, d] slice, brought into
// shared memory by TMA with the hardware swizzle: the d columns are split into
// chunks of SW bytes (128 for d >= 64, 64 for d = 32); chunk c of all 128 rows
// occupies one contiguous region of 128 * SW bytes, rows SW bytes apart, with
// 8-row swizzle atoms (8 * SW bytes).  The same smem image serves as
//   * a K-major operand (rows = M or N, contraction over d), and
//   * an MN-major operand (rows = the contraction dimension, N = d),
// depending on which descriptor is built for it.
#pragma once

#include "sm100.cuh"

namespace ca {

constexpr int kRows = 128;          // rows per tile (queries or keys)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D>
struct Tile {
  static_assert(D == 32 || D == 64 || D == 128, "head dim");
  static constexpr int SW = (D >= 64) ? 128 : 64;       // swizzle span = bytes per row per chunk
  static constexpr int CHUNKS = (D * 2) / SW;           // 2 (d=128) or 1
  static constexpr int CHUNK_BYTES = kRows * SW;        // 16 KB or 8 KB
  static constexpr int BYTES = kRows * D * 2;           // whole tile
  static constexpr int BOX_COLS = SW / 2;               // bf16 elements per TMA box row
  static constexpr uint32_t LAYOUT = (SW == 128) ? 2u : 4u;  // descriptor swizzle code
};

// Descriptor of a K-major operand for MMA-K step kk (16 bf16 = 32 bytes of d).
template <int D>
__device__ __forceinline__ uint64_t desc_k(uint32_t tile, int kk) {
  using Tl = Tile<D>;
  const uint32_t byte = (uint32_t)kk * 32u;
  const uint32_t addr = tile + (byte / Tl::SW) * Tl::CHUNK_BYTES + (byte % Tl::SW);
  return sdesc(addr, 16u, 8u * Tl::SW, Tl::LAYOUT);
}

// Descriptor of an MN-major operand (contraction over the tile's rows) for
// MMA-K step kk (16 rows).  N runs along d: chunks of SW/2 elements, CHUNK_BYTES apart.
template <int D>
__device__ __forceinline__ uint64_t desc_mn(uint32_t tile, int kk) {
  using Tl = Tile<D>;
  const uint32_t addr = tile + (uint32_t)kk * 16u * Tl::SW;
  return sdesc(addr, (uint32_t)Tl::CHUNK_BYTES, 8u * Tl::SW, Tl::LAYOUT);
}

// TMA: one 128-row tile of head `bh` starting at row `row0` (rows >= T read as zero).
template <int D>
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* m, int row0, int bh,
                                          uint32_t bar) {
#pragma unroll
  for (int c = 0; c < Tile<D>::CHUNKS; ++c)
    tma_load_3d(dst + c * Tile<D>::CHUNK_BYTES, m, c * Tile<D>::BOX_COLS, row0, bh, bar);
}

// Writes packed bf16 pairs w (columns col0 .. col0 + 2*NW - 1 of tile row r)
// into a staged tile with the layout load_tile produces (16-byte units XORed
// with the row inside each swizzle atom), ready for store_tile.  A warp writing
// 32 consecutive rows at the same columns hits every bank once per 8 rows.
template <int D, int NW>
__device__ __forceinline__ void stage_row(uint8_t* stage, int r, int col0, const uint32_t (&w)[NW]) {
  using Tl = Tile<D>;
  static_assert(NW % 4 == 0, "whole 16-byte units");
#pragma unroll
  for (int u = 0; u < NW / 4; ++u) {
    const int col = col0 + 8 * u;
    const int ch = col / Tl::BOX_COLS, cu = (col % Tl::BOX_COLS) / 8;
    const int phys = (Tl::SW == 128) ? (cu ^ (r & 7)) : (cu ^ ((r >> 1) & 3));
    *reinterpret_cast<uint4*>(stage + ch * Tl::CHUNK_BYTES + r * Tl::SW + phys * 16) =
        make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
  }
}

// TMA store of a staged tile to rows row0 .. row0 + 127 of head bh (rows past T are dropped).
template <int D>
__device__ __forceinline__ void store_tile(const CUtensorMap* m, uint32_t src, int row0, int bh) {
#pragma unroll
  for (int c = 0; c < Tile<D>::CHUNKS; ++c)
    tma_store_3d(m, src + c * Tile<D>::CHUNK_BYTES, c * Tile<D>::BOX_COLS, row0, bh);
}

// Keeps the compiler from using TMEM-load destination registers before
// tcgen05.wait::ld has been executed.
__device__ __forceinline__ void reg_fence(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31]));
}

__device__ __forceinline__ void reg_fence16(uint32_t (&r)[16]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]));
}

// Bounded wait that ignores the abort flag: used only while draining work
// already in flight (TMA copies and MMAs always finish on their own).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      report_timeout(15);
      return;
    }
  }
}

// Persistent work distribution: items are numbered heaviest first; CTA c of G
// takes, in round k, item k*G + c for even k and k*G + (G-1-c) for odd k, so a
// CTA that got one of the heavier items of a round gets one of the lighter
// items of the next.  Returns -1 past the end.
__device__ __forceinline__ int snake_item(int k, int c, int G, int n_items) {
  const int w = k * G + ((k & 1) ? (G - 1 - c) : c);
  return w < n_items ? w : -1;
}

// Shared-memory carve-up helper: 1024-byte aligned base inside dynamic smem.
__device__ __forceinline__ uint32_t aligned_smem_base(const void* raw, uint8_t** generic) {
  const uint32_t a = smem_u32(raw);
  const uint32_t b = (a + 1023u) & ~1023u;
  *generic = (uint8_t*)raw + (b - a);
  return b;
}

}  // namespace ca
