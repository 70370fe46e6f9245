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
