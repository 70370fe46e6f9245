// prologue.cuh -- RoPE + QK RMS-norm on the queries and keys, forward and backward, sm_100a.
//
// "How to build an LLM by hand" (agmtopy.github.io), section 9 (the gpt.py walkthrough): the
// attention block applies RoPE and then QK Norm ("x1.2") to Q and K before the causal
// attention.  Per row x (one head, one position t, d elements):
//   u = RoPE_t(x):  element p (p < d/2) is paired with p + d/2 and the pair is rotated by
//                   angle t * theta_p, theta_p = base^(-2p/d):
//                   u_p = x_p cos + x_{p+d/2} sin,  u_{p+d/2} = -x_p sin + x_{p+d/2} cos
//   z = gain * u / sqrt(mean(u^2) + eps)
// Backward, with r = sqrt(mean(u^2) + eps):
//   du = (gain / r) * (dz - u * <u, dz> / (d r^2)),   dx = RoPE_t^T(du)
//
// Both kernels are HBM bound: one read of each input row and one write of each output row,
// Q and K in the same launch.  A thread owns 8 rotation pairs of a row (two 16-byte
// chunks, elements 8c..8c+7 and d/2+8c..d/2+8c+7), so d/16 neighbouring lanes hold a row
// and the row sums are a shuffle over those lanes.  The angles depend on t and p only: a
// thread computes its 8 (cos, sin) once and applies them to several heads of Q and
// of K.  The angle t * theta_p is formed and reduced to [-pi, pi] in fp64 (so positions in
// the tens of thousands keep full fp32 phase accuracy), then __sincosf runs on the small
// reduced argument.  Output rows may be the input rows (in place): a row is read in full
// by its lanes before the shuffle that precedes any store to it (plain loads, not the
// read-only path, for that reason).
#pragma once

#include "sm100.cuh"

namespace ca {

constexpr int kProFwdHeads = 4;  // heads per work item (sharing one set of angles)
constexpr int kProBwdHeads = 2;
constexpr int kProThreads = 256;

struct ProParams {
  const __nv_bfloat16* x0;   // Q      [B, H, T, D]
  const __nv_bfloat16* x1;   // K
  const __nv_bfloat16* g0;   // backward: dL/dQ' (incoming), else unused
  const __nv_bfloat16* g1;   // backward: dL/dK'
  __nv_bfloat16* y0;         // forward Q' / backward dL/dQ
  __nv_bfloat16* y1;         // forward K' / backward dL/dK
  int B, H, T;
  double log2_base;
  float gain, eps;
};

// theta_p = base^(-2p/D) for p < D/2, fp64, into shared memory (one per block).
template <int D>
__device__ __forceinline__ void rope_theta_table(double* th, double log2_base) {
  for (int p = threadIdx.x; p < D / 2; p += blockDim.x)
    th[p] = exp2(-(2.0 * p / D) * log2_base);
  __syncthreads();
}

// cos / sin of t * theta_p for the 8 pairs p = 8c .. 8c+7.
template <int D>
__device__ __forceinline__ void rope_angles(const double* th, int t, int c, float (&cs)[8],
                                            float (&sn)[8]) {
  constexpr double kTwoPi = 6.283185307179586476925286766559;
  constexpr double kInvTwoPi = 0.15915494309189533576888376337251;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const double a = (double)t * th[8 * c + j];
    const double r = fma(-rint(a * kInvTwoPi), kTwoPi, a);  // a mod 2pi, in [-pi, pi]
    __sincosf((float)r, &sn[j], &cs[j]);
  }
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                    pack_bf16(f[6], f[7]));
}

// Sum over the D/16 lanes that share a row (aligned groups of consecutive lanes).
template <int D>
__device__ __forceinline__ float row_sum(float v) {
#pragma unroll
  for (int off = D / 32; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Work item = (b, group of HG heads, t, c); consecutive items take consecutive c, then t,
// so a warp reads 32 / (D/16) whole consecutive rows of a head.  The grid is persistent
// (a few blocks per SM) and each warp strides over the items 32 at a time, so the angle
// table is built once per block and there are no waves of short-lived blocks.
template <int D, int HG>
struct ProItems {
  long n;   // number of items (a multiple of D/16, so every row's lane group is whole)
  int hgs;  // head groups
  __device__ __forceinline__ explicit ProItems(const ProParams& p)
      : n((long)p.B * ((p.H + HG - 1) / HG) * p.T * (D / 16)), hgs((p.H + HG - 1) / HG) {}
  __device__ __forceinline__ void decompose(const ProParams& p, long g, int& b, int& h0, int& t,
                                            int& c) const {
    constexpr int TPR = D / 16;
    c = (int)(g % TPR);
    long rest = g / TPR;
    t = (int)(rest % p.T);
    rest /= p.T;
    h0 = (int)(rest % hgs) * HG;
    b = (int)(rest / hgs);
  }
};

__device__ __forceinline__ long warp_first_item() {
  return (long)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
}

template <int D>
__global__ void __launch_bounds__(kProThreads, 2) rope_qknorm_fwd_kernel(ProParams p) {
  constexpr int HG = kProFwdHeads;
  __shared__ double th[D / 2];
  rope_theta_table<D>(th, p.log2_base);
  const ProItems<D, HG> items(p);
  const int lane = threadIdx.x & 31;
  const long stride = (long)gridDim.x * blockDim.x;
  const float inv_d = 1.0f / D;
  // the loop bound is warp-uniform: every lane joins every row shuffle
  for (long base = warp_first_item(); base < items.n; base += stride) {
    const long g = base + lane;
    const bool ok = g < items.n;
    int b = 0, h0 = 0, t = 0, c = 0;
    if (ok) items.decompose(p, g, b, h0, t, c);
    uint4 raw[HG][2][2];  // [head][Q,K][first half, second half]
#pragma unroll
    for (int i = 0; i < HG; ++i) {
      const bool live = ok && h0 + i < p.H;
      const long row = (((long)b * p.H + h0 + i) * p.T + t) * D;
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const __nv_bfloat16* x = s ? p.x1 : p.x0;
        raw[i][s][0] = live ? *reinterpret_cast<const uint4*>(x + row + 8 * c)
                            : make_uint4(0, 0, 0, 0);
        raw[i][s][1] = live ? *reinterpret_cast<const uint4*>(x + row + D / 2 + 8 * c)
                            : make_uint4(0, 0, 0, 0);
      }
    }
    float cs[8], sn[8];
    rope_angles<D>(th, t, c, cs, sn);  // while the loads are in flight
#pragma unroll
    for (int i = 0; i < HG; ++i) {
      const bool live = ok && h0 + i < p.H;
      const long row = (((long)b * p.H + h0 + i) * p.T + t) * D;
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        float a[8], z[8], u1[8], u2[8];
        unpack8(raw[i][s][0], a);
        unpack8(raw[i][s][1], z);
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          u1[j] = a[j] * cs[j] + z[j] * sn[j];
          u2[j] = z[j] * cs[j] - a[j] * sn[j];
          ss += u1[j] * u1[j] + u2[j] * u2[j];
        }
        ss = row_sum<D>(ss);
        const float k = p.gain / sqrtf(ss * inv_d + p.eps);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          u1[j] *= k;
          u2[j] *= k;
        }
        if (live) {
          __nv_bfloat16* y = s ? p.y1 : p.y0;
          *reinterpret_cast<uint4*>(y + row + 8 * c) = pack8(u1);
          *reinterpret_cast<uint4*>(y + row + D / 2 + 8 * c) = pack8(u2);
        }
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kProThreads, 2) rope_qknorm_bwd_kernel(ProParams p) {
  constexpr int HG = kProBwdHeads;
  __shared__ double th[D / 2];
  rope_theta_table<D>(th, p.log2_base);
  const ProItems<D, HG> items(p);
  const int lane = threadIdx.x & 31;
  const long stride = (long)gridDim.x * blockDim.x;
  const float inv_d = 1.0f / D;
  for (long base = warp_first_item(); base < items.n; base += stride) {
    const long g = base + lane;
    const bool ok = g < items.n;
    int b = 0, h0 = 0, t = 0, c = 0;
    if (ok) items.decompose(p, g, b, h0, t, c);
    uint4 raw[HG][2][4];  // [head][Q,K][x lo, x hi, dz lo, dz hi]
#pragma unroll
    for (int i = 0; i < HG; ++i) {
      const bool live = ok && h0 + i < p.H;
      const long row = (((long)b * p.H + h0 + i) * p.T + t) * D;
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const __nv_bfloat16* x = s ? p.x1 : p.x0;
        const __nv_bfloat16* gz = s ? p.g1 : p.g0;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const long e = row + hh * (D / 2) + 8 * c;
          raw[i][s][hh] = live ? *reinterpret_cast<const uint4*>(x + e) : make_uint4(0, 0, 0, 0);
          raw[i][s][2 + hh] = live ? *reinterpret_cast<const uint4*>(gz + e) : make_uint4(0, 0, 0, 0);
        }
      }
    }
    float cs[8], sn[8];
    rope_angles<D>(th, t, c, cs, sn);
#pragma unroll
    for (int i = 0; i < HG; ++i) {
      const bool live = ok && h0 + i < p.H;
      const long row = (((long)b * p.H + h0 + i) * p.T + t) * D;
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        float a[8], z[8], g1[8], g2[8], u1[8], u2[8];
        unpack8(raw[i][s][0], a);
        unpack8(raw[i][s][1], z);
        unpack8(raw[i][s][2], g1);
        unpack8(raw[i][s][3], g2);
        float ss = 0.f, sd = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          u1[j] = a[j] * cs[j] + z[j] * sn[j];
          u2[j] = z[j] * cs[j] - a[j] * sn[j];
          ss += u1[j] * u1[j] + u2[j] * u2[j];
          sd += u1[j] * g1[j] + u2[j] * g2[j];
        }
        ss = row_sum<D>(ss);
        sd = row_sum<D>(sd);
        const float r2 = ss * inv_d + p.eps;
        const float k = p.gain / sqrtf(r2);
        const float m = sd * inv_d / r2;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float d1 = k * (g1[j] - u1[j] * m), d2 = k * (g2[j] - u2[j] * m);
          a[j] = d1 * cs[j] - d2 * sn[j];  // RoPE^T: rotate back
          z[j] = d1 * sn[j] + d2 * cs[j];
        }
        if (live) {
          __nv_bfloat16* y = s ? p.y1 : p.y0;
          *reinterpret_cast<uint4*>(y + row + 8 * c) = pack8(a);
          *reinterpret_cast<uint4*>(y + row + D / 2 + 8 * c) = pack8(z);
        }
      }
    }
  }
}

}  // namespace ca
