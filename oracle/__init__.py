"""CPU fp64 oracle for multi-head causal self-attention -- TEST INFRASTRUCTURE.

Only the tests, the smoke check in ``__graft_entry__`` and the CPU-baseline
leg of ``bench.py`` may import this package.  The CUDA library never touches
it, and it imports nothing from the CUDA package: the two share only the
seeded input generators, which hold none of the method's arithmetic.

The arithmetic lives in ``attn_oracle.c`` (plain C, double precision,
OpenMP over the independent (batch, head) pairs).  This module compiles it
with gcc on first use and marshals numpy float64 arrays through ctypes.

What is computed (see the C file header for the passages it follows):
  forward:   S = scale * Q K^T, S_ij = -inf for j > i (and, with a document
             mask, for j < doc_start[i]; with a sliding window of w keys, for
             j <= i - w), P = softmax_rows(S), O = P V,
             LSE_i = log sum_j exp(S_ij)  (natural log, scaled scores)
  backward:  dV = P^T dO, dP = dO V^T, dS_i = (diag(p_i) - p_i p_i^T) dP_i
             with the Jacobian formed explicitly, dQ = scale dS K,
             dK = scale dS^T Q.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "_attn_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into _attn_oracle.so (gcc, -O2, OpenMP).  Returns the path."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        lib.oracle_attn_fwd.argtypes = [dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_double, ip, dp, dp, dp]
        lib.oracle_attn_fwd.restype = ctypes.c_int
        lib.oracle_attn_bwd.argtypes = [dp, dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_double, ip, dp, dp, dp]
        lib.oracle_attn_bwd.restype = ctypes.c_int
        lib.oracle_attn_fwd_window.argtypes = [dp, dp, dp, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_double, ip,
                                               ctypes.c_int, dp, dp, dp]
        lib.oracle_attn_fwd_window.restype = ctypes.c_int
        lib.oracle_attn_bwd_window.argtypes = [dp, dp, dp, dp, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_double, ip,
                                               ctypes.c_int, dp, dp, dp]
        lib.oracle_attn_bwd_window.restype = ctypes.c_int
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact upcast to a C-contiguous float64 array (bf16/fp32 values are exact in fp64)."""
    if hasattr(x, "detach"):  # torch tensor (CPU)
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: Optional[np.ndarray], ctype):
    if a is None:
        return ctypes.cast(None, ctypes.POINTER(ctype))
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _doc(doc_start, B, T) -> Optional[np.ndarray]:
    if doc_start is None:
        return None
    if hasattr(doc_start, "detach"):
        doc_start = doc_start.detach().cpu().numpy()
    a = np.ascontiguousarray(np.asarray(doc_start, dtype=np.int32))
    if a.shape != (B, T):
        raise ValueError(f"doc_start must be [B,T]=({B},{T}), got {a.shape}")
    return a


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _window(window) -> int:
    """None or <= 0: no window; otherwise the number of keys a query sees, itself included."""
    return 0 if window is None or int(window) <= 0 else int(window)


def attention_forward(q, k, v, scale: float, doc_start=None, return_probs: bool = False,
                      window=None):
    """O [B,H,T,d], LSE [B,H,T] (float64); with return_probs also P [B,H,T,T].
    window: i sees j iff i - window < j <= i (None: plain causal)."""
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, T, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [B,H,T,d] shape")
    doc = _doc(doc_start, B, T)
    o = np.empty_like(q)
    lse = np.empty((B, H, T), dtype=np.float64)
    probs = np.empty((B, H, T, T), dtype=np.float64) if return_probs else None
    rc = lib.oracle_attn_fwd_window(_ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double),
                                    _ptr(v, ctypes.c_double), B, H, T, d, float(scale),
                                    _ptr(doc, ctypes.c_int32), _window(window),
                                    _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double),
                                    _ptr(probs, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd failed with code {rc}")
    return (o, lse, probs) if return_probs else (o, lse)


def attention_backward(q, k, v, dout, scale: float, doc_start=None,
                       window=None) -> Tuple[np.ndarray, ...]:
    """dQ, dK, dV [B,H,T,d] float64, by the explicit softmax Jacobian."""
    lib = _load()
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, T, d = q.shape
    for t in (k, v, dout):
        if t.shape != q.shape:
            raise ValueError("q, k, v, dout must share one [B,H,T,d] shape")
    doc = _doc(doc_start, B, T)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    rc = lib.oracle_attn_bwd_window(_ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double),
                                    _ptr(v, ctypes.c_double), _ptr(dout, ctypes.c_double),
                                    B, H, T, d, float(scale), _ptr(doc, ctypes.c_int32),
                                    _window(window), _ptr(dq, ctypes.c_double),
                                    _ptr(dk, ctypes.c_double), _ptr(dv, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_bwd failed with code {rc}")
    return dq, dk, dv


def decode_forward(q, k_cache, v_cache, scale: float):
    """KV-cache decode, written out in numpy float64: new token t of Tq sits at position
    L - Tq + t and attends to cache positions 0 .. L - Tq + t.  q: [B,Tq,H,d];
    k_cache, v_cache: [B,L,H,d].  Returns O [B,Tq,H,d] and LSE [B,H,Tq] (natural log)."""
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    B, Tq, H, d = q.shape
    L = kc.shape[1]
    if kc.shape != (B, L, H, d) or vc.shape != kc.shape or Tq > L:
        raise ValueError("q [B,Tq,H,d], k_cache / v_cache [B,L,H,d], Tq <= L")
    o = np.empty((B, Tq, H, d))
    lse = np.empty((B, H, Tq))
    for b in range(B):
        for h in range(H):
            for t in range(Tq):
                n = L - Tq + t + 1                       # visible cache positions
                s = scale * (kc[b, :n, h, :] @ q[b, t, h, :])
                m = s.max()
                w = np.exp(s - m)
                z = w.sum()
                o[b, t, h] = (w / z) @ vc[b, :n, h, :]
                lse[b, h, t] = m + np.log(z)
    return o, lse


# ------------------------------------------------------- RoPE + QK-norm prologue
# "How to build an LLM by hand" (agmtopy.github.io), section 9 (gpt.py walkthrough):
# the attention applies RoPE and then QK Norm ("x1.2") to the queries and keys.  The page
# gives no formulas; the readings: RoPE in the rotate-half form (element i is paired with
# i + d/2, angle = position * base^(-2i/d), base 10000), QK Norm an RMS normalisation over
# d without learned weights (eps 1e-6) followed by the constant gain 1.2.

def _rope_angles(T: int, d: int, base: float):
    i = np.arange(d // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / d)
    ang = np.arange(T, dtype=np.float64)[:, None] * theta[None, :]  # [T, d/2]
    return np.cos(ang), np.sin(ang)


def _rope(x, cos, sin, inverse=False):
    h = x.shape[-1] // 2
    x1, x2 = x[..., :h], x[..., h:]
    s = -sin if inverse else sin
    return np.concatenate([x1 * cos + x2 * s, -x1 * s + x2 * cos], axis=-1)


def qk_prologue_forward(x, base: float = 10000.0, gain: float = 1.2, eps: float = 1e-6):
    """z = gain * u / sqrt(mean(u^2) + eps), u = RoPE(x) at positions 0..T-1.  x: [B,H,T,d]."""
    x = _f64(x)
    T, d = x.shape[2], x.shape[3]
    cos, sin = _rope_angles(T, d, base)
    u = _rope(x, cos, sin)
    r = np.sqrt(np.mean(u * u, axis=-1, keepdims=True) + eps)
    return gain * u / r


def qk_prologue_backward(x, dz, base: float = 10000.0, gain: float = 1.2, eps: float = 1e-6):
    """dL/dx for z = qk_prologue_forward(x): through the norm, dL/du = (gain / r) *
    (dz - u (u . dz) / (d r^2)); through the rotation, dL/dx = RoPE^T(dL/du) (the inverse
    rotation)."""
    x, dz = _f64(x), _f64(dz)
    T, d = x.shape[2], x.shape[3]
    cos, sin = _rope_angles(T, d, base)
    u = _rope(x, cos, sin)
    r = np.sqrt(np.mean(u * u, axis=-1, keepdims=True) + eps)
    s = np.sum(u * dz, axis=-1, keepdims=True)
    du = (gain / r) * (dz - u * s / (d * r * r))
    return _rope(du, cos, sin, inverse=True)


# ------------------------------------------------------ FP8 (e4m3) attention forward
# "How to build an LLM by hand" (agmtopy.github.io), section 5, item 4: the in-house FP8
# training runs the forward matmuls with e4m3 operands through torch._scaled_mm (per-tensor
# scales, higher-precision accumulation); the page lists the missing dynamic scaling as a
# shortcoming, so scales are fixed per tensor.  Reading for the attention forward: Q, K and
# V arrive as e4m3 codes with one fp32 descale factor each (x = descale * x8); the scores
# are scale * (dq * dk) * Q8 K8^T, the softmax is exact, and the left operand of the second
# product -- the attention weights -- is itself quantised to e4m3.  The weights are taken
# relative to the row maximum (so they lie in (0, 1]) and multiplied by 2^8 before rounding,
# so that the largest weight sits well inside e4m3's range (max 448) and weights down to
# 2^-14 of the maximum stay normal numbers; the weighted sum is normalised by the sum of the
# quantised weights.  The e4m3 format is the OCP 8-bit floating point "E4M3" (bias 7, no
# infinities, S.1111.111 is NaN, largest finite 448, smallest subnormal 2^-9); rounding to it
# is round-to-nearest-even with saturation at +-448.
#
# The reference output is the exact attention of the dequantised inputs (fp64).  What the
# quantised weights may change is bounded row by row: with r_j = exp(s_j - max_k s_k) and a
# weight error |q_j - r_j| <= e_j,
#     O - o = sum_j (q_j - r_j)(v_j - o) / sum_j q_j,
# so |O_c - o_c| <= sum_j e_j |v_jc - o_c| / (sum_j r_j - sum_j e_j).  Rounding 2^8 r_j c
# (c >= 1 when the weights are taken relative to a running maximum that later grew) to e4m3
# leaves e_j = 2^-4 r_j (normal range, half an ulp of 3 mantissa bits) or 2^-10 / 2^8 / c
# <= 2^-18 (subnormal range, half the 2^-9 spacing); the bound uses their sum plus 2^-14 r_j
# for the fp32 evaluation of the exponential before rounding.

E4M3_MAX = 448.0
FP8_P_SCALE = 256.0  # weights relative to the row maximum are multiplied by 2^8 before rounding


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of e4m3 codes (uint8): sign, 4 exponent bits (bias 7), 3 mantissa bits;
    exponent field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


_E4M3_POS = None  # the 127 finite non-negative e4m3 values, ascending, and their codes


def _e4m3_table():
    global _E4M3_POS
    if _E4M3_POS is None:
        codes = np.arange(0x7F, dtype=np.uint8)  # 0x00 .. 0x7E: +0 .. 448
        _E4M3_POS = (e4m3_decode(codes), codes)
    return _E4M3_POS


def e4m3_encode(x) -> np.ndarray:
    """Nearest e4m3 code to each float (ties to the even code, i.e. the even mantissa),
    saturating to +-448; NaN -> 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    vals, codes = _e4m3_table()
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(vals, a, side="left"), 0, len(vals) - 1)  # first value >= a
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - vals[lo], vals[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (codes[hi] % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    out = codes[idx].astype(np.uint8)
    out = np.where((x < 0) & (out != 0), out | 0x80, out)
    out = np.where(np.signbit(x) & (out == 0), 0x80, out)  # -0 keeps its sign
    return np.where(np.isnan(x), 0x7F, out).astype(np.uint8)


def e4m3_round(x) -> np.ndarray:
    """x rounded to the nearest e4m3 value (float64)."""
    return e4m3_decode(e4m3_encode(x))


def _codes(x) -> np.ndarray:
    if hasattr(x, "detach"):
        import torch
        x = x.detach().cpu()
        if x.dtype != torch.uint8:
            x = x.view(torch.uint8)
        x = x.numpy()
    return np.asarray(x, dtype=np.uint8)


def fp8_dequantize(x8, descale: float) -> np.ndarray:
    """descale * value of each e4m3 code (exact in fp64)."""
    return float(descale) * e4m3_decode(_codes(x8))


def fp8_weight_error_bound(r: np.ndarray) -> np.ndarray:
    """Largest |q - r| of a weight r in (0, 1] (relative to the row maximum) after rounding
    2^8 r c to e4m3 and dividing by 2^8 c, for any c >= 1."""
    return (2.0 ** -4 + 2.0 ** -14) * r + 2.0 ** -18


def fp8_attention_forward(q8, k8, v8, descale_q: float, descale_k: float, descale_v: float,
                          scale: float, doc_start=None, window=None):
    """Reference of the FP8 attention forward: O [B,H,T,d] and LSE [B,H,T] (exact attention of
    the dequantised e4m3 inputs, float64) and BOUND [B,H,T,d], the largest change that
    quantising the weights to e4m3 can make to each element of O."""
    q = fp8_dequantize(q8, descale_q)
    k = fp8_dequantize(k8, descale_k)
    v = fp8_dequantize(v8, descale_v)
    B, H, T, d = q.shape
    doc = _doc(doc_start, B, T)
    o = np.empty_like(q)
    lse = np.empty((B, H, T))
    bound = np.empty_like(q)
    for b in range(B):
        for h in range(H):
            ds = doc[b:b + 1] if doc is not None else None
            ob, lb, pb = attention_forward(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1],
                                           v[b:b + 1, h:h + 1], scale, ds, return_probs=True,
                                           window=window)
            o[b, h], lse[b, h] = ob[0, 0], lb[0, 0]
            p = pb[0, 0]                               # [T, T], rows sum to 1, zeros masked
            r = p / p.max(axis=1, keepdims=True)       # weights relative to the row maximum
            e = np.where(p > 0, fp8_weight_error_bound(r), 0.0)
            den = r.sum(axis=1) - e.sum(axis=1)        # lower bound on the quantised sum
            vb = v[b, h]
            for i0 in range(0, T, 256):                # sum_j e_ij |v_jc - o_ic|, row blocks
                i1 = min(T, i0 + 256)
                dev = np.abs(vb[None, :, :] - o[b, h, i0:i1, None, :])   # [rows, T, d]
                bound[b, h, i0:i1] = np.einsum("ij,ijc->ic", e[i0:i1], dev)
            bound[b, h] /= den[:, None]
    return o, lse, bound


def fp8_attention_simulated(q8, k8, v8, descale_q: float, descale_k: float, descale_v: float,
                            scale: float, doc_start=None, window=None, p_scale=FP8_P_SCALE):
    """The quantised-weight forward of the reading above, evaluated in float64 with the weights
    taken relative to the final row maximum: q_j = e4m3(p_scale * r_j) / p_scale,
    O = sum_j q_j v_j / sum_j q_j.  (A device kernel that takes the weights relative to a
    running maximum rounds at other points; its result obeys the same bound.)"""
    q = fp8_dequantize(q8, descale_q)
    k = fp8_dequantize(k8, descale_k)
    v = fp8_dequantize(v8, descale_v)
    B, H, T, d = q.shape
    doc = _doc(doc_start, B, T)
    o = np.empty_like(q)
    for b in range(B):
        for h in range(H):
            ds = doc[b:b + 1] if doc is not None else None
            _, _, pb = attention_forward(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1],
                                         v[b:b + 1, h:h + 1], scale, ds, return_probs=True,
                                         window=window)
            p = pb[0, 0]
            r = p / p.max(axis=1, keepdims=True)
            qw = e4m3_round(p_scale * r) / p_scale
            o[b, h] = (qw @ v[b, h]) / qw.sum(axis=1, keepdims=True)
    return o
