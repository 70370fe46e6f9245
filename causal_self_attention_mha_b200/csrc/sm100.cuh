// sm100.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) features the
// attention kernels use: mbarriers with bounded waits, TMA tile loads,
// tcgen05 UMMA (shared-memory and tensor-memory operands), TMEM allocation and
// TMEM <-> register copies.  Written against the PTX ISA descriptions of these
// instructions; the descriptor bit layouts follow the public tcgen05 matrix and
// instruction descriptor tables.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace ca {

// ------------------------------------------------------------------ status
// Device-side error word (bit flags), read by the host through
// gpt_attn_device_status().  A kernel that gives up on a wait ORs
// kStatusTimeout plus a site code in; it never traps.
enum : unsigned {
  kStatusTimeout = 1u << 31,
  kStatusSmem = 1u << 30,  // a kernel's shared-memory layout did not fit what it was given
  kStatusBounds = 1u << 29,  // (debug builds) a checked index or TMA coordinate was out of range
};

__device__ unsigned int g_status;

__device__ __forceinline__ void report_timeout(unsigned site) {
  atomicOr(&g_status, kStatusTimeout | (1u << (site & 15)));
}

__device__ __forceinline__ void report_smem_shortfall() { atomicOr(&g_status, kStatusSmem); }

// Debug builds (compiled with CA_DEBUG_CHECKS): the kernels check every TMA coordinate and
// every global index they compute on the device; a failed check sets kStatusBounds and the
// access is skipped (a load reads 0, a TMA copy is not issued, so its waiter times out and
// reports) instead of trapping.  In release builds the checks compile to nothing.
#ifdef CA_DEBUG_CHECKS
__device__ __forceinline__ bool dbg_ok(bool ok) {
  if (!ok) atomicOr(&g_status, kStatusBounds);
  return ok;
}
#else
__device__ __forceinline__ constexpr bool dbg_ok(bool) { return true; }
#endif

// a[i] of an array of n elements (i computed by the kernel), checked in debug builds.
template <class T>
__device__ __forceinline__ T ld_chk(const T* a, size_t i, size_t n) {
  return dbg_ok(i < n) ? a[i] : T(0);
}
template <class T>
__device__ __forceinline__ T ldg_chk(const T* a, size_t i, size_t n) {
  return dbg_ok(i < n) ? __ldg(a + i) : T(0);
}
template <class T>
__device__ __forceinline__ void st_chk(T* a, size_t i, size_t n, T v) {
  if (dbg_ok(i < n)) a[i] = v;
}

// The innermost coordinate of a tiled TMA copy must start on a 16-byte boundary: every copy
// here moves 16-bit (bf16) or 8-bit (e4m3, at x = 0) elements, so x is a multiple of 8; a
// store never starts at a negative coordinate.
__device__ __forceinline__ bool tma_coords_ok(int c0, int c_outer) {
  return dbg_ok(c0 >= 0 && (c0 & 7) == 0 && c_outer >= 0);
}

// Opt-in limit of dynamic shared memory per block (227 KB).
constexpr int kMaxDynSmem = 232448;

__device__ __forceinline__ uint32_t dynamic_smem_bytes() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// One try_wait: the thread may sleep in hardware (up to the hint, 0.1 ms) until
// the phase completes, instead of spinning and taking issue slots from its
// sub-partition's other warps.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2, %3;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(100000u)
      : "memory");
  return ok != 0;
}

// One non-blocking test of a phase: cheaper than try_wait when the phase has completed (about 60
// against 90 cycles measured), which is what the MMA-issuing threads mostly find.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Per-CTA wait guard.  Every wait is bounded by limit_ns of wall time; on
// expiry the waiter raises the CTA-wide abort flag (shared memory), records
// the site in g_status and returns false.  A waiter that sees the abort flag
// raised by another thread also returns false.  Callers then skip the rest of
// their work, drain what they have in flight and leave.
struct Guard {
  volatile int* abort_flag;
  uint64_t limit_ns;
};

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, const Guard& g,
                                             unsigned site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*g.abort_flag) return false;
    if (globaltimer_ns() - t0 > g.limit_ns) {
      *g.abort_flag = 1;
      report_timeout(site);
      return false;
    }
  }
}

// The MMA-issuing threads' wait: every cycle it spends leaves the tensor pipe idle, so the
// phase is tested once before the (sleeping) bounded wait.
__device__ __forceinline__ bool wait_bounded_fast(uint32_t bar, uint32_t parity, const Guard& g,
                                                  unsigned site) {
  return mbar_test(bar, parity) || wait_bounded(bar, parity, g, site);
}

// Same, with the outcome made uniform across the warp (needed before any
// warp-collective tcgen05.ld/st that follows the wait).
__device__ __forceinline__ bool wait_bounded_warp(uint32_t bar, uint32_t parity, const Guard& g,
                                                  unsigned site) {
  bool ok = wait_bounded(bar, parity, g, site);
  return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 3-D tiled load (coordinates innermost first) into shared memory, completing
// `bytes` of transaction count on `bar`.  c0 * 2 bytes is always a multiple of
// 16 here (c0 is 0 or a multiple of the 32/64-element swizzle width).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* m, int c0, int c1,
                                            int c2, uint32_t bar) {
  if (!tma_coords_ok(c0, c2)) return;
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// 4-D tiled load, as above (c0 * 2 bytes a multiple of 16).
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* m, int c0, int c1,
                                            int c2, int c3, uint32_t bar) {
  if (!tma_coords_ok(c0, c1 | c3)) return;
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

// 3-D tiled store from shared memory (rows past the tensor's extent are not
// written).  Completion is tracked per thread with bulk groups.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* m, uint32_t src, int c0, int c1,
                                             int c2) {
  if (!tma_coords_ok(c0, c1 | c2)) return;
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Until every committed bulk store of this thread has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Until every committed bulk store of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Orders this thread's shared-memory writes before later async-proxy (TMA) reads.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------ tcgen05 / TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// Arrive once on `bar` when every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], 8-bit floating-point operands (K = 32 per instruction)
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], 8-bit floating-point operands
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor for kind::f8f6f4 with e4m3 A/B (format code 0) and fp32 accumulate;
// same fields as idesc_bf16_f32.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, bool b_mn_major) {
  return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 accumulate.
//   bits 4-5 D format (1 = f32), 7-9 A format (1 = bf16), 10-12 B format (1 = bf16),
//   bit 15 A major (0 = K), bit 16 B major (0 = K, 1 = MN), 17-22 N>>3, 24-28 M>>4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor.
//   bits 0-13 start >> 4, 16-29 leading-dim byte offset >> 4, 32-45 stride-dim
//   byte offset >> 4, 46-47 version (1), 61-63 layout (2 = 128B swizzle, 4 = 64B).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                          uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)layout << 61;
  return d;
}

// TMEM -> registers: 32 lanes x 32 consecutive 32-bit columns; thread i of the
// warp receives lane (quadrant base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// TMEM -> registers: 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Per-warpgroup register budget changes (all four warps of a warpgroup execute
// them).  The launch budget must cover the sum of the new per-warpgroup counts.
template <uint32_t N>
__device__ __forceinline__ void regs_grow() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_shrink() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// registers -> TMEM: 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// registers -> TMEM: 32 lanes x 8 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

// ------------------------------------------------------------- arithmetic
// Hardware base-2 exponential / logarithm (MUFU), flush-to-zero.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (Blackwell f32x2 arithmetic: one instruction, two lanes of math).
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ uint64_t f2u(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ float2 f2split(uint64_t v) {
  float2 f;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(v));
  return f;
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// 2^x for a pair of x < 126 on the FMA pipe: x = n + f with n = round(x) (clamped at -125) and
// f in [-1/2, 1/2]; 2^f from a cubic fitted for least maximum relative error on that interval
// (Lawson's iteratively reweighted least squares; max relative error 7.5e-5, far below the
// 2^-9 of the bf16 weights it feeds), and n added into the exponent field.  Below 2^-125 the
// result is 2^-125 times 2^f instead of the exact value (or 0 for -inf): weights that small
// change no sum, and no output, by more than 1e-37.
__device__ __forceinline__ uint64_t exp2_fma2(uint64_t x2) {
  const float2 x = f2split(x2);
  const uint64_t xc = f2(fmaxf(x.x, -125.f), fmaxf(x.y, -125.f));
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23: adding it rounds to an integer
  const uint64_t t = fadd2(xc, f2(kRound, kRound));
  const uint64_t n = fadd2(t, f2(-kRound, -kRound));
  const uint64_t fr = ffma2(n, f2(-1.f, -1.f), xc);
  uint64_t q = ffma2(f2(0.05517166f, 0.05517166f), fr, f2(0.24261112f, 0.24261112f));
  q = ffma2(q, fr, f2(0.69326099f, 0.69326099f));
  q = ffma2(q, fr, f2(0.99992807f, 0.99992807f));
  const float2 qf = f2split(q), tf = f2split(t);
  // the low bits of t hold n in two's complement: shifted into the exponent field they add n
  return f2(__uint_as_float(__float_as_uint(qf.x) + (__float_as_uint(tf.x) << 23)),
            __uint_as_float(__float_as_uint(qf.y) + (__float_as_uint(tf.y) << 23)));
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Two floats -> packed bf16x2 (round to nearest even); `lo` lands in bits 0-15.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Four floats -> four e4m3 codes in one 32-bit word, a in bits 0-7 ... d in bits 24-31 (round to
// nearest even, saturating to +-448).
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(r)
      : "f"(a), "f"(b), "f"(c), "f"(d));
  return r;
}

// acc0 += value of byte 0 of w, acc1 += byte 1, acc2 += byte 2, acc3 += byte 3 (e4m3 codes,
// exact: every e4m3 value is an f16 value).
__device__ __forceinline__ void add_e4m3x4(uint32_t w, float& acc0, float& acc1, float& acc2,
                                           float& acc3) {
  asm("{\n\t.reg .b16 lo, hi, a, b, c, d;\n\t.reg .b32 hlo, hhi;\n\t"
      "mov.b32 {lo, hi}, %4;\n\t"
      "cvt.rn.f16x2.e4m3x2 hlo, lo;\n\t"
      "cvt.rn.f16x2.e4m3x2 hhi, hi;\n\t"
      "mov.b32 {a, b}, hlo;\n\t"
      "mov.b32 {c, d}, hhi;\n\t"
      "add.rn.f32.f16 %0, a, %0;\n\t"
      "add.rn.f32.f16 %1, b, %1;\n\t"
      "add.rn.f32.f16 %2, c, %2;\n\t"
      "add.rn.f32.f16 %3, d, %3;\n\t}"
      : "+f"(acc0), "+f"(acc1), "+f"(acc2), "+f"(acc3)
      : "r"(w));
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
// packed bf16x2 -> fp32 pair (exact)
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t v) { return f2u(v << 16, v & 0xFFFF0000u); }

}  // namespace ca
