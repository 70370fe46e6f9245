// causalattn.cu -- host side of libcausalattn: the C ABI declared in
// include/causalattn.h (argument validation, TMA descriptor encoding,
// per-device setup, kernel launches, status reporting) plus the small
// utility kernels (document-offset validator, wait-timeout self-test).
// The attention kernels themselves live in fwd.cuh and bwd.cuh.

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdint>
#include <mutex>

#include "../../include/causalattn.h"
#include "bwd.cuh"
#include "decode.cuh"
#include "fwd.cuh"
#include "fwd8.cuh"
#include "fwd_pair.cuh"
#include "prologue.cuh"

namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far above any legitimate wait
constexpr int kMaxDevices = 64;

// An NVTX range around each kernel launch, named after the kernel, for timelines taken with
// nsys or `ncu --nvtx`; with no tool attached a push and a pop cost a few nanoseconds.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// ------------------------------------------------------------ validation
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_shape(int B, int H, int T, int d) {
  if (B < 1 || H < 1 || T < 1) return GPT_ATTN_ERR_BAD_SHAPE;
  if (d != 32 && d != 64 && d != 128) return GPT_ATTN_ERR_UNSUPPORTED_HEAD_DIM;
  const int64_t elems = (int64_t)B * H * T * d;
  if (elems > (int64_t)INT32_MAX) return GPT_ATTN_ERR_TOO_LARGE;
  return GPT_ATTN_OK;
}

int check_scale(float scale) {
  if (!std::isfinite(scale) || !(scale > 0.f)) return GPT_ATTN_ERR_BAD_SCALE;
  return GPT_ATTN_OK;
}

// ----------------------------------------------------------- device setup
std::mutex g_mu;
std::atomic<int> g_dev_state[kMaxDevices];  // 0 unknown, 1 ready, 2 wrong arch, 3 setup failed
int g_sm_count[kMaxDevices];                // multiprocessors per device (persistent grids)
int g_pair_clusters[kMaxDevices];           // co-resident CTA pairs of the pair forward kernel

// Shared-memory opt-in of the CTA-pair forward kernel and how many of its pairs fit at once.
cudaError_t setup_pair_kernel(int dev) {
  cudaError_t e = cudaFuncSetAttribute(ca::attn_fwd_pair_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       ca::PairLayout::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (unsigned)(g_sm_count[dev] / 2));
  cfg.blockDim = dim3(ca::PairLayout::THREADS);
  cfg.dynamicSmemBytes = ca::PairLayout::SMEM;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, (void*)ca::attn_fwd_pair_kernel, &cfg) != cudaSuccess ||
      n < 1) {
    cudaGetLastError();
    n = g_sm_count[dev] / 2;
  }
  g_pair_clusters[dev] = n;
  return cudaSuccess;
}

template <int D>
cudaError_t set_smem_attrs() {
  cudaError_t e;
  e = cudaFuncSetAttribute(ca::attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           ca::FwdLayout<D>::SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(ca::attn_bwd_dkdv_kernel<D>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, ca::DkdvLayout<D>::SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(ca::attn_fwd_fp8_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           ca::Fwd8Layout<D>::SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(ca::attn_decode_chunk_kernel<D>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, ca::DecLayout<D>::SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(ca::attn_decode_chunk_tc_kernel<D>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, ca::DecTcLayout<D>::SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(ca::attn_bwd_dq_kernel<D, true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, ca::DqLayout<D>::SMEM);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(ca::attn_bwd_dq_kernel<D, false>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, ca::DqLayout<D>::SMEM);
}

int ensure_device() {
  int count = 0;
  if (cudaGetDeviceCount(&count) != cudaSuccess || count < 1) {
    cudaGetLastError();
    return GPT_ATTN_ERR_NO_DEVICE;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return GPT_ATTN_ERR_NO_DEVICE;
  }
  // The runtime binds a device's primary context to a host thread lazily; descriptor encoding
  // (a driver call) needs it bound, and the first library call on a thread (torch's autograd
  // engine calls the backward from a worker thread of its own) may come before anything else
  // has bound it.  cudaSetDevice binds it; once per thread and device.
  thread_local int t_bound_dev = -1;
  if (t_bound_dev != dev) {
    if (cudaSetDevice(dev) != cudaSuccess) {
      cudaGetLastError();
      return GPT_ATTN_ERR_NO_DEVICE;
    }
    t_bound_dev = dev;
  }
  int st = g_dev_state[dev].load(std::memory_order_acquire);
  if (st == 0) {
    std::lock_guard<std::mutex> lock(g_mu);
    st = g_dev_state[dev].load(std::memory_order_relaxed);
    if (st == 0) {
      int major = 0, minor = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return GPT_ATTN_ERR_NO_DEVICE;
      }
      int sms = 0;
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      g_sm_count[dev] = sms > 0 ? sms : 148;
      if (major != 10 || minor != 0) {
        st = 2;
      } else if (set_smem_attrs<32>() != cudaSuccess || set_smem_attrs<64>() != cudaSuccess ||
                 set_smem_attrs<128>() != cudaSuccess || setup_pair_kernel(dev) != cudaSuccess) {
        cudaGetLastError();
        st = 3;
      } else {
        st = 1;
      }
      g_dev_state[dev].store(st, std::memory_order_release);
    }
  }
  if (st == 1) return GPT_ATTN_OK;
  if (st == 2) return GPT_ATTN_ERR_UNSUPPORTED_ARCH;
  return GPT_ATTN_ERR_LAUNCH;
}

// ------------------------------------------------------ TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// Encoded descriptors are cached: a descriptor is a pure function of its kind, head dim, base
// address and extents, which together form the key, so a hit is always valid (also after the
// memory was freed and reallocated).  Small and round-robin (a training step touches about a
// dozen distinct tensors); one cache for all host threads, under a mutex.
struct MapKey {
  const void* base;
  int kind, d, e0, e1, e2;
  bool operator==(const MapKey& o) const {
    return base == o.base && kind == o.kind && d == o.d && e0 == o.e0 && e1 == o.e1 && e2 == o.e2;
  }
};
constexpr int kMapCache = 32;
struct MapCache {
  MapKey key[kMapCache];
  CUtensorMap map[kMapCache];
  bool used[kMapCache];
  int next;
};
MapCache g_maps;  // zero-initialised: no entry used
std::mutex g_maps_mu;

thread_local const char* t_last_cuda_error = "no error";
thread_local char t_encode_error[96];

template <class F>
bool cached_map(CUtensorMap* m, const MapKey& k, F encode) {
  std::lock_guard<std::mutex> lock(g_maps_mu);
  MapCache& c = g_maps;
  for (int i = 0; i < kMapCache; ++i)
    if (c.used[i] && c.key[i] == k) {
      *m = c.map[i];
      return true;
    }
  if (!encode(m)) return false;
  const int i = c.next;
  c.next = (c.next + 1) % kMapCache;
  c.key[i] = k;
  c.map[i] = *m;
  c.used[i] = true;
  return true;
}

enum MapKind { kMapBf16 = 1, kMapE4m3 = 2, kMapCacheKV = 3, kMapBf16Half = 4 };

// True on success; otherwise records the driver's code for gpt_attn_last_cuda_error.
bool encode_ok(CUresult r) {
  if (r == CUDA_SUCCESS) return true;
  snprintf(t_encode_error, sizeof(t_encode_error), "cuTensorMapEncodeTiled failed with CUresult %d",
           (int)r);
  t_last_cuda_error = t_encode_error;
  return false;
}

// A [B*H, T, d] bf16 tensor viewed as 3-D (d innermost), boxes of
// (swizzle width, 128 rows, 1 head); rows past T read as zero.
template <int D>
bool encode_map(CUtensorMap* m, const void* base, int BH, int T, int box_rows = ca::kRows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    t_last_cuda_error = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  using Tl = ca::Tile<D>;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)T * D * 2};
  cuuint32_t box[3] = {(cuuint32_t)Tl::BOX_COLS, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   Tl::SW == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return encode_ok(r);
}

template <int D>
bool make_map(CUtensorMap* m, const void* base, int BH, int T) {
  return cached_map(m, MapKey{base, kMapBf16, D, BH, T, 0},
                    [&](CUtensorMap* out) { return encode_map<D>(out, base, BH, T); });
}

// The same view with boxes of 64 rows: each CTA of a pair loads half of a 128-row tile.
template <int D>
bool make_half_map(CUtensorMap* m, const void* base, int BH, int T) {
  return cached_map(m, MapKey{base, kMapBf16Half, D, BH, T, 0},
                    [&](CUtensorMap* out) { return encode_map<D>(out, base, BH, T, 64); });
}

// A [B*H, T, d] tensor of e4m3 codes viewed as 3-D bytes (d innermost), boxes of (d, 128 rows,
// 1 head) with a d-byte swizzle; rows past T read as zero.
template <int D>
bool encode_map8(CUtensorMap* m, const void* base, int BH, int T) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D, (cuuint64_t)T * D};
  cuuint32_t box[3] = {(cuuint32_t)D, (cuuint32_t)ca::kRows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw = D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : (D == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return encode_ok(r);
}

template <int D>
bool make_map8(CUtensorMap* m, const void* base, int BH, int T) {
  return cached_map(m, MapKey{base, kMapE4m3, D, BH, T, 0},
                    [&](CUtensorMap* out) { return encode_map8<D>(out, base, BH, T); });
}

// A [B, L, H, d] bf16 KV cache (the layout of the pages' kv-cache call) viewed as 4-D
// (d, H, L, B) with boxes of (swizzle width, 1 head, 128 rows, 1 batch); rows past L read
// as zero.  The staged box has the same shared-memory image as make_map's tiles.
template <int D>
bool encode_cache_map(CUtensorMap* m, const void* base, int B, int L, int H) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  using Tl = ca::Tile<D>;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)L * H * D * 2};
  cuuint32_t box[4] = {(cuuint32_t)Tl::BOX_COLS, 1, (cuuint32_t)ca::kDecChunk, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   Tl::SW == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return encode_ok(r);
}

template <int D>
bool make_cache_map(CUtensorMap* m, const void* base, int B, int L, int H) {
  return cached_map(m, MapKey{base, kMapCacheKV, D, B, L, H},
                    [&](CUtensorMap* out) { return encode_cache_map<D>(out, base, B, L, H); });
}

int sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  return (dev >= 0 && dev < kMaxDevices && g_sm_count[dev] > 0) ? g_sm_count[dev] : 148;
}

int pair_clusters() {
  int dev = 0;
  cudaGetDevice(&dev);
  return (dev >= 0 && dev < kMaxDevices && g_pair_clusters[dev] > 0) ? g_pair_clusters[dev] : 74;
}

int launch_status() {
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return GPT_ATTN_OK;
  t_last_cuda_error = cudaGetErrorString(e);
  return GPT_ATTN_ERR_LAUNCH;
}

// ------------------------------------------------------------- launchers
// A window of w keys (the query's own included); w <= 0 or w >= T is no window,
// which the kernels express as w = T (the band then covers every causal key).
int effective_window(int window, int T) { return (window <= 0 || window > T) ? T : window; }

template <int D>
int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int T,
             float scale, const int32_t* doc, int window, cudaStream_t st) {
  const int BH = B * H;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map<D>(&mq, q, BH, T) || !make_map<D>(&mk, k, BH, T) || !make_map<D>(&mv, v, BH, T) ||
      !make_map<D>(&mo, o, BH, T))
    return GPT_ATTN_ERR_LAUNCH;
  ca::FwdParams p;
  p.doc = doc;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.H = H;
  p.T = T;
  p.BH = BH;
  p.n_qt = (T + ca::kRows - 1) / ca::kRows;
  p.n_pairs = (p.n_qt + 1) / 2;
  p.n_items = p.n_pairs * BH;
  p.scale_log2 = scale * ca::kLog2e;
  p.window = effective_window(window, T);
  p.wait_limit_ns = kWaitLimitNs;
  if (D == 128 && p.window >= T) {
    // CTA pairs: each pair walks items, each CTA of it one query tile of the item.  Both CTAs
    // walk the union of the two tiles' key ranges, so with a sliding window (ranges offset by
    // a tile) the single-CTA kernel, whose two tiles each walk their own range, is faster.
    CUtensorMap mkh;
    if (!make_half_map<D>(&mkh, k, BH, T)) return GPT_ATTN_ERR_LAUNCH;
    const int pairs = pair_clusters();
    const unsigned grid = 2u * (unsigned)(p.n_items < pairs ? p.n_items : pairs);
    NvtxRange nvtx("attn_fwd_pair");
    ca::attn_fwd_pair_kernel<<<grid, ca::PairLayout::THREADS, ca::PairLayout::SMEM, st>>>(
        mq, mkh, mv, mo, p);
    return launch_status();
  }
  // persistent: one CTA per SM, each walking items blockIdx.x, blockIdx.x + gridDim.x, ...
  const int sms = sm_count();
  const unsigned grid = (unsigned)(p.n_items < sms ? p.n_items : sms);
  NvtxRange nvtx("attn_fwd");
  ca::attn_fwd_kernel<D><<<grid, ca::FwdLayout<D>::THREADS, ca::FwdLayout<D>::SMEM, st>>>(
      mq, mk, mv, mo, p);
  return launch_status();
}

template <int D>
int fwd8_impl(const void* q8, const void* k8, const void* v8, float dsq, float dsk, float dsv,
              void* o, float* lse, int B, int H, int T, float scale, const int32_t* doc,
              cudaStream_t st) {
  const int BH = B * H;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map8<D>(&mq, q8, BH, T) || !make_map8<D>(&mk, k8, BH, T) ||
      !make_map8<D>(&mv, v8, BH, T) || !make_map<D>(&mo, o, BH, T))
    return GPT_ATTN_ERR_LAUNCH;
  ca::Fwd8Params p8;
  ca::FwdParams& p = p8.f;
  p.doc = doc;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.H = H;
  p.T = T;
  p.BH = BH;
  p.n_qt = (T + ca::kRows - 1) / ca::kRows;
  p.n_pairs = (p.n_qt + 1) / 2;
  p.n_items = p.n_pairs * BH;
  p.scale_log2 = (float)((double)scale * dsq * dsk * 1.4426950408889634);
  p.window = T;
  p.wait_limit_ns = kWaitLimitNs;
  p8.descale_v = dsv;
  const int sms = sm_count();
  const unsigned grid = (unsigned)(p.n_items < sms ? p.n_items : sms);
  NvtxRange nvtx("attn_fwd_fp8");
  ca::attn_fwd_fp8_kernel<D><<<grid, ca::Fwd8Layout<D>::THREADS, ca::Fwd8Layout<D>::SMEM, st>>>(
      mq, mk, mv, mo, p8);
  return launch_status();
}

template <int D>
int delta_impl(const void* o, const void* dout, float* delta, int B, int H, int T,
               cudaStream_t st) {
  const long rows = (long)B * H * T;
  const long threads = rows * (D / 8);
  long blocks = (threads + 255) / 256;
  if (blocks > 148L * 16) blocks = 148L * 16;
  NvtxRange nvtx("attn_bwd_delta");
  ca::attn_bwd_delta_kernel<D><<<(unsigned)blocks, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), delta, rows);
  return launch_status();
}

// dkdv: the dK/dV kernel (g0 = dK, g1 = dV); otherwise the dQ kernel (g0 = dQ), which with
// o != nullptr also computes delta from o and dout and writes it to delta_out.
template <int D>
int bwd_tiled_impl(bool dkdv, const void* q, const void* k, const void* v, const void* dout,
                   const float* lse, const float* delta, void* g0, void* g1, int B, int H, int T,
                   float scale, const int32_t* doc, int window, cudaStream_t st,
                   const void* o = nullptr, float* delta_out = nullptr) {
  const int BH = B * H;
  CUtensorMap mq, mk, mv, mdo;
  if (!make_map<D>(&mq, q, BH, T) || !make_map<D>(&mk, k, BH, T) || !make_map<D>(&mv, v, BH, T) ||
      !make_map<D>(&mdo, dout, BH, T))
    return GPT_ATTN_ERR_LAUNCH;
  ca::BwdParams p;
  p.doc = doc;
  p.lse = lse;
  p.delta = delta;
  p.delta_out = delta_out;
  p.g0 = static_cast<__nv_bfloat16*>(g0);
  p.g1 = static_cast<__nv_bfloat16*>(g1);
  p.H = H;
  p.T = T;
  p.BH = BH;
  p.n_t = (T + ca::kRows - 1) / ca::kRows;
  p.n_items = p.n_t * BH;
  p.scale = scale;
  p.scale_log2 = scale * ca::kLog2e;
  p.window = effective_window(window, T);
  p.wait_limit_ns = kWaitLimitNs;
  // persistent: one CTA per SM, each walking items blockIdx.x, blockIdx.x + gridDim.x, ...
  const int sms = sm_count();
  const unsigned grid = (unsigned)(p.n_items < sms ? p.n_items : sms);
  // outputs leave through TMA stores of whole tiles (rows past T are dropped)
  CUtensorMap mg0, mg1, mo;
  if (!make_map<D>(&mg0, g0, BH, T) || (dkdv && !make_map<D>(&mg1, g1, BH, T)) ||
      (o && !make_map<D>(&mo, o, BH, T)))
    return GPT_ATTN_ERR_LAUNCH;
  NvtxRange nvtx(dkdv ? "attn_bwd_dkdv" : (o ? "attn_bwd_dq_delta" : "attn_bwd_dq"));
  if (dkdv)
    ca::attn_bwd_dkdv_kernel<D><<<grid, ca::DkdvLayout<D>::THREADS, ca::DkdvLayout<D>::SMEM, st>>>(
        mq, mk, mv, mdo, mg0, mg1, p);
  else if (o)
    ca::attn_bwd_dq_kernel<D, true><<<grid, ca::DqLayout<D>::THREADS, ca::DqLayout<D>::SMEM, st>>>(
        mq, mk, mv, mdo, mg0, mo, p);
  else  // the O map is not read without the fused delta: any valid map will do
    ca::attn_bwd_dq_kernel<D, false><<<grid, ca::DqLayout<D>::THREADS, ca::DqLayout<D>::SMEM, st>>>(
        mq, mk, mv, mdo, mg0, mq, p);
  return launch_status();
}

template <int D>
int decode_impl(const void* q, const void* kc, const void* vc, void* o, float* lse, float* ws,
                int B, int H, int Tq, int L, float scale, cudaStream_t st) {
  CUtensorMap mk, mv;
  if (!make_cache_map<D>(&mk, kc, B, L, H) || !make_cache_map<D>(&mv, vc, B, L, H))
    return GPT_ATTN_ERR_LAUNCH;
  ca::DecParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.B = B;
  p.H = H;
  p.Tq = Tq;
  p.L = L;
  p.n_chunks = (L + ca::kDecChunk - 1) / ca::kDecChunk;
  const size_t rows = (size_t)B * H * Tq * p.n_chunks;
  // partial outputs first: every (row, chunk) slice of them starts on a 16-byte boundary
  // (the merge kernel reads them as float4 / float2 vectors)
  p.part_o = ws;
  p.part_ml = ws + rows * D;
  p.scale_log2 = scale * ca::kLog2e;
  p.wait_limit_ns = kWaitLimitNs;
  dim3 grid((unsigned)p.n_chunks, (unsigned)H, (unsigned)B);
  // one new token: CUDA cores, a thread per key row; two or more: tensor cores
  {
  NvtxRange nvtx("attn_decode_chunk");
  if (Tq >= ca::kDecTcMinTq)
    ca::attn_decode_chunk_tc_kernel<D><<<grid, ca::DecTcLayout<D>::THREADS, ca::DecTcLayout<D>::SMEM,
                                         st>>>(mk, mv, p);
  else
    ca::attn_decode_chunk_kernel<D><<<grid, ca::kDecThreads, ca::DecLayout<D>::SMEM, st>>>(mk, mv, p);
  }
  int s = launch_status();
  if (s) return s;
  NvtxRange nvtx("attn_decode_combine");
  ca::attn_decode_combine_kernel<D><<<(unsigned)(B * H * Tq), ca::kCombWarps * 32, 0, st>>>(
      p.part_ml, p.part_o, static_cast<__nv_bfloat16*>(o), lse, H, Tq, p.n_chunks);
  return launch_status();
}

// Workspace of gpt_attn_decode in bytes (0 for arguments it would reject).
size_t decode_ws_bytes(int B, int H, int Tq, int L, int d) {
  if (B < 1 || H < 1 || Tq < 1 || Tq > ca::kDecMaxTq || L < Tq) return 0;
  if (d != 32 && d != 64 && d != 128) return 0;
  const size_t chunks = ((size_t)L + ca::kDecChunk - 1) / ca::kDecChunk;
  return (size_t)B * H * Tq * chunks * (2 + (size_t)d) * sizeof(float);
}

// -------------------------------------------------------- utility kernels
// Verdict word of gpt_attn_check_doc_offsets.  One per device; every call clears it, runs the
// checker and reads it back before returning, all under g_doc_mu, so calls from several host
// threads (on any streams) never see one another's verdict.
__device__ int g_doc_bad;
std::mutex g_doc_mu;

__global__ void check_doc_kernel(const int32_t* doc, int B, int T) {
  const long n = (long)B * T;
  for (long e = (long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long)gridDim.x * blockDim.x) {
    const int i = (int)(e % T);
    const int v = doc[e];
    const bool ok = (i == 0) ? (v == 0) : (v == i || v == doc[e - 1]);
    if (!ok) atomicOr(&g_doc_bad, 1);
  }
}

__global__ void wait_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    ca::mbar_init(ca::smem_u32(&bar), 1);
    ca::fence_barrier_init();
    const ca::Guard g{&abort_flag, limit_ns};
    // nothing ever arrives on `bar`: the wait must give up and report
    ca::wait_bounded(ca::smem_u32(&bar), 0, g, 14);
  }
}

int common_checks(int B, int H, int T, int d) { return check_shape(B, H, T, d); }

// Persistent grid: the resident blocks per SM times the SMs, or fewer when the work is small.
template <int D>
int prologue_impl(bool bwd, const ca::ProParams& p, cudaStream_t st) {
  static std::atomic<int> resident[2] = {0, 0};
  const void* fn = bwd ? reinterpret_cast<const void*>(ca::rope_qknorm_bwd_kernel<D>)
                       : reinterpret_cast<const void*>(ca::rope_qknorm_fwd_kernel<D>);
  int per_sm = resident[bwd].load(std::memory_order_relaxed);
  if (per_sm == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, ca::kProThreads, 0) !=
            cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    resident[bwd].store(per_sm, std::memory_order_relaxed);
  }
  const int hg = bwd ? ca::kProBwdHeads : ca::kProFwdHeads;
  const long items = (long)p.B * ((p.H + hg - 1) / hg) * p.T * (D / 16);
  long blocks = (items + ca::kProThreads - 1) / ca::kProThreads;
  if (blocks > (long)sm_count() * per_sm) blocks = (long)sm_count() * per_sm;
  NvtxRange nvtx(bwd ? "rope_qknorm_bwd" : "rope_qknorm_fwd");
  if (bwd)
    ca::rope_qknorm_bwd_kernel<D><<<(unsigned)blocks, ca::kProThreads, 0, st>>>(p);
  else
    ca::rope_qknorm_fwd_kernel<D><<<(unsigned)blocks, ca::kProThreads, 0, st>>>(p);
  return launch_status();
}

}  // namespace

// ======================================================================== ABI
extern "C" {

int gpt_attn_version(void) { return GPT_ATTN_ABI_VERSION; }

const char* gpt_attn_last_cuda_error(void) { return t_last_cuda_error; }

const char* gpt_attn_strerror(int s) {
  switch (s) {
    case GPT_ATTN_OK: return "ok";
    case GPT_ATTN_ERR_NULL_PTR: return "a required pointer is NULL";
    case GPT_ATTN_ERR_BAD_SHAPE: return "B, H and T must be >= 1";
    case GPT_ATTN_ERR_UNSUPPORTED_HEAD_DIM: return "head dim d must be 32, 64 or 128";
    case GPT_ATTN_ERR_MISALIGNED: return "bf16 tensors need 16-byte alignment, fp32/int32 arrays 4-byte";
    case GPT_ATTN_ERR_BAD_DOC_OFFSETS: return "doc_offsets is not a valid document-start array";
    case GPT_ATTN_ERR_NO_DEVICE: return "no usable CUDA device";
    case GPT_ATTN_ERR_UNSUPPORTED_ARCH: return "current device is not sm_100 (B200)";
    case GPT_ATTN_ERR_LAUNCH: return "CUDA launch or setup failed";
    case GPT_ATTN_ERR_DEVICE_TIMEOUT: return "a kernel gave up on a bounded wait";
    case GPT_ATTN_ERR_NOT_IMPLEMENTED: return "not implemented";
    case GPT_ATTN_ERR_BAD_SCALE: return "scale must be finite and > 0";
    case GPT_ATTN_ERR_TOO_LARGE: return "tensor too large (B*H*T*d must be < 2^31)";
    case GPT_ATTN_ERR_BAD_PARAM:
      return "bad parameter: rope_base must be finite and > 0, gain finite, eps finite and >= 0; "
             "FP8 descale factors finite and > 0";
    default: return "unknown status";
  }
}

static int fwd_entry(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int T, int d, float scale, const int32_t* doc_offsets, int window,
                     void* stream) {
  if (!q || !k || !v || !o || !lse) return GPT_ATTN_ERR_NULL_PTR;
  int s = common_checks(B, H, T, d);
  if (s) return s;
  if ((s = check_scale(scale))) return s;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(doc_offsets, 4))
    return GPT_ATTN_ERR_MISALIGNED;
  if ((s = ensure_device())) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 32: return fwd_impl<32>(q, k, v, o, lse, B, H, T, scale, doc_offsets, window, st);
    case 64: return fwd_impl<64>(q, k, v, o, lse, B, H, T, scale, doc_offsets, window, st);
    default: return fwd_impl<128>(q, k, v, o, lse, B, H, T, scale, doc_offsets, window, st);
  }
}

int gpt_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int T, int d, float scale, const int32_t* doc_offsets, void* stream) {
  return fwd_entry(q, k, v, o, lse, B, H, T, d, scale, doc_offsets, 0, stream);
}

int gpt_attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int H, int T, int d, float scale, const int32_t* doc_offsets, int window,
                        void* stream) {
  return fwd_entry(q, k, v, o, lse, B, H, T, d, scale, doc_offsets, window, stream);
}

int gpt_attn_fwd_fp8(const void* q8, const void* k8, const void* v8, float descale_q,
                     float descale_k, float descale_v, void* o, float* lse, int B, int H, int T,
                     int d, float scale, const int32_t* doc_offsets, void* stream) {
  if (!q8 || !k8 || !v8 || !o || !lse) return GPT_ATTN_ERR_NULL_PTR;
  int s = common_checks(B, H, T, d);
  if (s) return s;
  if ((s = check_scale(scale))) return s;
  for (float ds : {descale_q, descale_k, descale_v})
    if (!std::isfinite(ds) || !(ds > 0.f)) return GPT_ATTN_ERR_BAD_PARAM;
  // the combined score scale must stay a finite, non-zero fp32 number
  const double sl = (double)scale * descale_q * descale_k;
  if (!(sl > 1e-30) || !(sl < 1e30)) return GPT_ATTN_ERR_BAD_PARAM;
  if (!aligned(q8, 16) || !aligned(k8, 16) || !aligned(v8, 16) || !aligned(o, 16) ||
      !aligned(lse, 4) || !aligned(doc_offsets, 4))
    return GPT_ATTN_ERR_MISALIGNED;
  if ((s = ensure_device())) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 32:
      return fwd8_impl<32>(q8, k8, v8, descale_q, descale_k, descale_v, o, lse, B, H, T, scale,
                           doc_offsets, st);
    case 64:
      return fwd8_impl<64>(q8, k8, v8, descale_q, descale_k, descale_v, o, lse, B, H, T, scale,
                           doc_offsets, st);
    default:
      return fwd8_impl<128>(q8, k8, v8, descale_q, descale_k, descale_v, o, lse, B, H, T, scale,
                            doc_offsets, st);
  }
}

int gpt_attn_bwd_preprocess(const void* o, const void* dout, float* delta, int B, int H, int T,
                            int d, void* stream) {
  if (!o || !dout || !delta) return GPT_ATTN_ERR_NULL_PTR;
  int s = common_checks(B, H, T, d);
  if (s) return s;
  if (!aligned(o, 16) || !aligned(dout, 16) || !aligned(delta, 4)) return GPT_ATTN_ERR_MISALIGNED;
  if ((s = ensure_device())) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 32: return delta_impl<32>(o, dout, delta, B, H, T, st);
    case 64: return delta_impl<64>(o, dout, delta, B, H, T, st);
    default: return delta_impl<128>(o, dout, delta, B, H, T, st);
  }
}

// With o != nullptr (dQ step only) delta is not read but computed from o and dout and written
// to delta_out; otherwise delta is an input.
static int bwd_step(bool dkdv, const void* q, const void* k, const void* v, const void* dout,
                    const float* lse, const float* delta, void* g0, void* g1, int B, int H, int T,
                    int d, float scale, const int32_t* doc, int window, void* stream,
                    const void* o = nullptr, float* delta_out = nullptr) {
  if (!q || !k || !v || !dout || !lse || !g0 || (dkdv && !g1) || (o ? !delta_out : !delta))
    return GPT_ATTN_ERR_NULL_PTR;
  int s = common_checks(B, H, T, d);
  if (s) return s;
  if ((s = check_scale(scale))) return s;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(dout, 16) ||
      !aligned(g0, 16) || (dkdv && !aligned(g1, 16)) || !aligned(lse, 4) || !aligned(delta, 4) ||
      !aligned(doc, 4) || !aligned(o, 16) || !aligned(delta_out, 4))
    return GPT_ATTN_ERR_MISALIGNED;
  if ((s = ensure_device())) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 32:
      return bwd_tiled_impl<32>(dkdv, q, k, v, dout, lse, delta, g0, g1, B, H, T, scale, doc,
                                window, st, o, delta_out);
    case 64:
      return bwd_tiled_impl<64>(dkdv, q, k, v, dout, lse, delta, g0, g1, B, H, T, scale, doc,
                                window, st, o, delta_out);
    default:
      return bwd_tiled_impl<128>(dkdv, q, k, v, dout, lse, delta, g0, g1, B, H, T, scale, doc,
                                 window, st, o, delta_out);
  }
}

int gpt_attn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dout,
                      const float* lse, const float* delta, void* dk, void* dv, int B, int H,
                      int T, int d, float scale, const int32_t* doc_offsets, void* stream) {
  return bwd_step(true, q, k, v, dout, lse, delta, dk, dv, B, H, T, d, scale, doc_offsets, 0, stream);
}

int gpt_attn_bwd_dq(const void* q, const void* k, const void* v, const void* dout,
                    const float* lse, const float* delta, void* dq, int B, int H, int T, int d,
                    float scale, const int32_t* doc_offsets, void* stream) {
  return bwd_step(false, q, k, v, dout, lse, delta, dq, nullptr, B, H, T, d, scale, doc_offsets, 0,
                  stream);
}

int gpt_attn_bwd_dq_delta(const void* q, const void* k, const void* v, const void* o,
                          const void* dout, const float* lse, float* delta_out, void* dq, int B,
                          int H, int T, int d, float scale, const int32_t* doc_offsets,
                          void* stream) {
  if (!o) return GPT_ATTN_ERR_NULL_PTR;
  return bwd_step(false, q, k, v, dout, lse, nullptr, dq, nullptr, B, H, T, d, scale, doc_offsets,
                  0, stream, o, delta_out);
}

static int bwd_entry(const void* q, const void* k, const void* v, const void* o, const void* dout,
                     const float* lse, void* dq, void* dk, void* dv, float* delta_ws, int B, int H,
                     int T, int d, float scale, const int32_t* doc_offsets, int window,
                     void* stream) {
  // validate everything before the first launch, so an error never leaves a partial backward
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !delta_ws)
    return GPT_ATTN_ERR_NULL_PTR;
  int s = common_checks(B, H, T, d);
  if (s) return s;
  if ((s = check_scale(scale))) return s;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
      !aligned(lse, 4) || !aligned(delta_ws, 4) || !aligned(doc_offsets, 4))
    return GPT_ATTN_ERR_MISALIGNED;
  if ((s = ensure_device())) return s;
  // dQ first: it also computes delta (into delta_ws), which dK/dV then reads
  if ((s = bwd_step(false, q, k, v, dout, lse, nullptr, dq, nullptr, B, H, T, d, scale,
                    doc_offsets, window, stream, o, delta_ws)))
    return s;
  return bwd_step(true, q, k, v, dout, lse, delta_ws, dk, dv, B, H, T, d, scale, doc_offsets,
                  window, stream);
}

int gpt_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, float* delta_ws, int B, int H,
                 int T, int d, float scale, const int32_t* doc_offsets, void* stream) {
  return bwd_entry(q, k, v, o, dout, lse, dq, dk, dv, delta_ws, B, H, T, d, scale, doc_offsets, 0,
                   stream);
}

int gpt_attn_bwd_window(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        float* delta_ws, int B, int H, int T, int d, float scale,
                        const int32_t* doc_offsets, int window, void* stream) {
  return bwd_entry(q, k, v, o, dout, lse, dq, dk, dv, delta_ws, B, H, T, d, scale, doc_offsets,
                   window, stream);
}

size_t gpt_attn_decode_workspace_size(int B, int H, int Tq, int L, int d) {
  return decode_ws_bytes(B, H, Tq, L, d);
}

int gpt_attn_decode(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                    void* workspace, size_t workspace_bytes, int B, int H, int Tq, int L, int d,
                    float scale, void* stream) {
  if (!q || !k_cache || !v_cache || !o || !lse || !workspace) return GPT_ATTN_ERR_NULL_PTR;
  if (B < 1 || H < 1 || Tq < 1 || L < 1 || Tq > L || Tq > ca::kDecMaxTq || H > 65535 || B > 65535)
    return GPT_ATTN_ERR_BAD_SHAPE;
  if (d != 32 && d != 64 && d != 128) return GPT_ATTN_ERR_UNSUPPORTED_HEAD_DIM;
  if ((int64_t)B * L * H * d >= ((int64_t)1 << 31) || (int64_t)B * Tq * H * d >= ((int64_t)1 << 31))
    return GPT_ATTN_ERR_TOO_LARGE;
  int s;
  if ((s = check_scale(scale))) return s;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) ||
      !aligned(lse, 4) || !aligned(workspace, 16))
    return GPT_ATTN_ERR_MISALIGNED;
  if (workspace_bytes < decode_ws_bytes(B, H, Tq, L, d)) return GPT_ATTN_ERR_BAD_SHAPE;
  if ((s = ensure_device())) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* ws = static_cast<float*>(workspace);
  switch (d) {
    case 32: return decode_impl<32>(q, k_cache, v_cache, o, lse, ws, B, H, Tq, L, scale, st);
    case 64: return decode_impl<64>(q, k_cache, v_cache, o, lse, ws, B, H, Tq, L, scale, st);
    default: return decode_impl<128>(q, k_cache, v_cache, o, lse, ws, B, H, Tq, L, scale, st);
  }
}

static int prologue_entry(bool bwd, const void* x0, const void* x1, const void* g0, const void* g1,
                          void* y0, void* y1, int B, int H, int T, int d, float rope_base,
                          float gain, float eps, void* stream) {
  if (!x0 || !x1 || !y0 || !y1 || (bwd && (!g0 || !g1))) return GPT_ATTN_ERR_NULL_PTR;
  int s = common_checks(B, H, T, d);
  if (s) return s;
  if (!std::isfinite(rope_base) || !(rope_base > 0.f) || !std::isfinite(gain) ||
      !std::isfinite(eps) || !(eps >= 0.f))
    return GPT_ATTN_ERR_BAD_PARAM;
  if (!aligned(x0, 16) || !aligned(x1, 16) || !aligned(g0, 16) || !aligned(g1, 16) ||
      !aligned(y0, 16) || !aligned(y1, 16))
    return GPT_ATTN_ERR_MISALIGNED;
  if ((s = ensure_device())) return s;
  ca::ProParams p;
  p.x0 = static_cast<const __nv_bfloat16*>(x0);
  p.x1 = static_cast<const __nv_bfloat16*>(x1);
  p.g0 = static_cast<const __nv_bfloat16*>(g0);
  p.g1 = static_cast<const __nv_bfloat16*>(g1);
  p.y0 = static_cast<__nv_bfloat16*>(y0);
  p.y1 = static_cast<__nv_bfloat16*>(y1);
  p.B = B;
  p.H = H;
  p.T = T;
  p.log2_base = std::log2((double)rope_base);
  p.gain = gain;
  p.eps = eps;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 32: return prologue_impl<32>(bwd, p, st);
    case 64: return prologue_impl<64>(bwd, p, st);
    default: return prologue_impl<128>(bwd, p, st);
  }
}

int gpt_attn_rope_qknorm_fwd(const void* q, const void* k, void* q_out, void* k_out, int B, int H,
                             int T, int d, float rope_base, float gain, float eps, void* stream) {
  return prologue_entry(false, q, k, nullptr, nullptr, q_out, k_out, B, H, T, d, rope_base, gain,
                        eps, stream);
}

int gpt_attn_rope_qknorm_bwd(const void* q, const void* k, const void* dq_out, const void* dk_out,
                             void* dq, void* dk, int B, int H, int T, int d, float rope_base,
                             float gain, float eps, void* stream) {
  return prologue_entry(true, q, k, dq_out, dk_out, dq, dk, B, H, T, d, rope_base, gain, eps,
                        stream);
}

int gpt_attn_check_doc_offsets(const int32_t* doc_offsets, int B, int T, void* stream) {
  if (!doc_offsets) return GPT_ATTN_ERR_NULL_PTR;
  if (B < 1 || T < 1) return GPT_ATTN_ERR_BAD_SHAPE;
  if ((int64_t)B * T > (int64_t)INT32_MAX) return GPT_ATTN_ERR_TOO_LARGE;
  if (!aligned(doc_offsets, 4)) return GPT_ATTN_ERR_MISALIGNED;
  int s = ensure_device();
  if (s) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_doc_mu);  // clear, check, read back: one call at a time
  const int zero = 0;
  if (cudaMemcpyToSymbolAsync(g_doc_bad, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) !=
      cudaSuccess) {
    cudaGetLastError();
    return GPT_ATTN_ERR_LAUNCH;
  }
  long blocks = ((long)B * T + 255) / 256;
  if (blocks > 148L * 8) blocks = 148L * 8;
  check_doc_kernel<<<(unsigned)blocks, 256, 0, st>>>(doc_offsets, B, T);
  if ((s = launch_status())) return s;
  int bad = 0;
  if (cudaMemcpyFromSymbolAsync(&bad, g_doc_bad, sizeof(int), 0, cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return GPT_ATTN_ERR_LAUNCH;
  }
  return bad ? GPT_ATTN_ERR_BAD_DOC_OFFSETS : GPT_ATTN_OK;
}

int gpt_attn_device_status(unsigned int* out, int clear) {
  if (!out) return GPT_ATTN_ERR_NULL_PTR;
  int s = ensure_device();
  if (s) return s;
  if (cudaDeviceSynchronize() != cudaSuccess ||
      cudaMemcpyFromSymbol(out, ca::g_status, sizeof(unsigned)) != cudaSuccess) {
    cudaGetLastError();
    return GPT_ATTN_ERR_LAUNCH;
  }
  if (clear) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(ca::g_status, &zero, sizeof(unsigned)) != cudaSuccess) {
      cudaGetLastError();
      return GPT_ATTN_ERR_LAUNCH;
    }
  }
  return GPT_ATTN_OK;
}

int gpt_attn_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  int s = ensure_device();
  if (s) return s;
  unsigned before = 0;
  if ((s = gpt_attn_device_status(&before, 1))) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  wait_selftest_kernel<<<1, 32, 0, st>>>(limit_ns);
  if ((s = launch_status())) return s;
  if (cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return GPT_ATTN_ERR_LAUNCH;
  }
  unsigned after = 0;
  if ((s = gpt_attn_device_status(&after, 1))) return s;
  return (after & ca::kStatusTimeout) ? GPT_ATTN_ERR_DEVICE_TIMEOUT : GPT_ATTN_OK;
}

}  // extern "C"

// ============================================ backward without caller scratch
// For callers that cannot allocate device memory (see gpt_attn_bwd_static_ws in
// include/causalattn.h): the delta workspace lives in this file-scope device
// array instead of a caller buffer.  Every GPU that loads the library holds it
// (4 MiB) until the process exits.

namespace {

constexpr long kStaticWsRows = 1L << 20;  // == GPT_ATTN_STATIC_WS_MAX_ROWS

static __device__ __align__(256) float g_static_delta[kStaticWsRows];

std::mutex g_static_mu;
float* g_static_delta_ptr[kMaxDevices];  // device address per device, set once

// Device address of g_static_delta on the current device.  In host code the
// symbol's name is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress, once per device, with that device current.
int static_delta_ptr(float** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return GPT_ATTN_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (g_static_delta_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_delta) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return GPT_ATTN_ERR_LAUNCH;
    }
    g_static_delta_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_static_delta_ptr[dev];
  return GPT_ATTN_OK;
}

}  // namespace

extern "C" int gpt_attn_bwd_static_ws(const void* q, const void* k, const void* v, const void* o,
                                      const void* dout, const float* lse, void* dq, void* dk,
                                      void* dv, int B, int H, int T, int d, float scale,
                                      const int32_t* doc_offsets, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return GPT_ATTN_ERR_NULL_PTR;
  int s = common_checks(B, H, T, d);
  if (s) return s;
  if ((int64_t)B * H * T > (int64_t)kStaticWsRows) return GPT_ATTN_ERR_TOO_LARGE;
  if ((s = check_scale(scale))) return s;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
      !aligned(lse, 4) || !aligned(doc_offsets, 4))
    return GPT_ATTN_ERR_MISALIGNED;
  if ((s = ensure_device())) return s;
  float* delta = nullptr;
  if ((s = static_delta_ptr(&delta))) return s;
  // delta is fully rewritten by the first step (dQ, which computes it), so nothing needs
  // clearing first
  if ((s = gpt_attn_bwd_dq_delta(q, k, v, o, dout, lse, delta, dq, B, H, T, d, scale, doc_offsets,
                                 stream)))
    return s;
  return gpt_attn_bwd_dkdv(q, k, v, dout, lse, delta, dk, dv, B, H, T, d, scale, doc_offsets,
                           stream);
}
