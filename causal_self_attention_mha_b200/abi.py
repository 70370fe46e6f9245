"""ctypes binding of libcausalattn (include/causalattn.h).

Argument marshalling only: every function here checks that the torch tensors
it is given have the layout the C ABI documents (contiguous bf16 [B,H,T,d] on
the current CUDA device, fp32/int32 side arrays), passes their device
pointers, sizes and the current CUDA stream through the C ABI, and turns a
non-zero status into an exception.  All arithmetic happens in the library's
CUDA kernels.  There is no CPU fallback: if the library is missing or cannot
be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# CAUSALATTN_LIBRARY selects another build of the same library (e.g. libcausalattn_debug.so,
# whose kernels check every TMA coordinate and computed global index on the device).
LIB_PATH = os.environ.get("CAUSALATTN_LIBRARY") or os.path.join(_HERE, "libcausalattn.so")

GPT_ATTN_OK = 0
GPT_ATTN_ERR_NULL_PTR = 1
GPT_ATTN_ERR_BAD_SHAPE = 2
GPT_ATTN_ERR_UNSUPPORTED_HEAD_DIM = 3
GPT_ATTN_ERR_MISALIGNED = 4
GPT_ATTN_ERR_BAD_DOC_OFFSETS = 5
GPT_ATTN_ERR_NO_DEVICE = 6
GPT_ATTN_ERR_UNSUPPORTED_ARCH = 7
GPT_ATTN_ERR_LAUNCH = 8
GPT_ATTN_ERR_DEVICE_TIMEOUT = 9
GPT_ATTN_ERR_NOT_IMPLEMENTED = 10
GPT_ATTN_ERR_BAD_SCALE = 11
GPT_ATTN_ERR_TOO_LARGE = 12
GPT_ATTN_ERR_BAD_PARAM = 13

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float

# name -> (argtypes, restype); mirrors include/causalattn.h
SIGNATURES = {
    "gpt_attn_fwd": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _vp], _i),
    "gpt_attn_bwd": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _vp], _i),
    "gpt_attn_fwd_fp8": ([_vp, _vp, _vp, _f, _f, _f, _vp, _vp, _i, _i, _i, _i, _f, _vp, _vp], _i),
    "gpt_attn_fwd_window": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _i, _vp], _i),
    "gpt_attn_bwd_window": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f,
                             _vp, _i, _vp], _i),
    "gpt_attn_decode_workspace_size": ([_i, _i, _i, _i, _i], ctypes.c_size_t),
    "gpt_attn_decode": ([_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _i, _i, _i, _i, _i, _f, _vp],
                        _i),
    "gpt_attn_rope_qknorm_fwd": ([_vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _f, _f, _vp], _i),
    "gpt_attn_rope_qknorm_bwd": ([_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _f, _f, _vp], _i),
    "gpt_attn_bwd_preprocess": ([_vp, _vp, _vp, _i, _i, _i, _i, _vp], _i),
    "gpt_attn_bwd_dkdv": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _vp], _i),
    "gpt_attn_bwd_dq": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _vp], _i),
    "gpt_attn_bwd_dq_delta": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _vp],
                              _i),
    "gpt_attn_bwd_static_ws": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _vp], _i),
    "gpt_attn_check_doc_offsets": ([_vp, _i, _i, _vp], _i),
    "gpt_attn_device_status": ([ctypes.POINTER(ctypes.c_uint), _i], _i),
    "gpt_attn_selftest_wait_timeout": ([ctypes.c_uint64, _vp], _i),
    "gpt_attn_strerror": ([_i], ctypes.c_char_p),
    "gpt_attn_version": ([], _i),
    "gpt_attn_last_cuda_error": ([], ctypes.c_char_p),
}

_lib = None


class AttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        detail = ""
        if status == GPT_ATTN_ERR_LAUNCH:
            try:
                detail = ": " + load().gpt_attn_last_cuda_error().decode()
            except Exception:
                pass
        super().__init__(f"{fn} failed: status {status} ({strerror(status)}{detail})")


_tls = threading.local()  # prepare(): a per-thread recorder that stands in for the library


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libcausalattn.so (raises if it is missing: there is no fallback)."""
    global _lib
    rec = getattr(_tls, "recorder", None)
    if rec is not None and path is None:
        return rec
    if _lib is None or path is not None:
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(
                f"libcausalattn.so not found at {p}; build it with "
                "`python -m causal_self_attention_mha_b200.build`")
        lib = ctypes.CDLL(p)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        if path is not None:
            return lib
        _lib = lib
    return _lib


def strerror(status: int) -> str:
    try:
        return load().gpt_attn_strerror(int(status)).decode()
    except Exception:  # the library itself may be what failed to load
        return "unknown"


def version() -> int:
    return int(load().gpt_attn_version())


def _stream(stream, device: Optional[torch.device] = None) -> Optional[int]:
    """The cudaStream_t handle to launch on.  The library launches on the CURRENT CUDA device,
    so the tensors' device (`device`) must be the current one, and a torch stream passed in must
    belong to it: otherwise one device's pointers would reach kernels and TMA descriptors on
    another."""
    if device is not None and device.index != torch.cuda.current_device():
        raise ValueError(f"tensors are on {device} but the current CUDA device is "
                         f"cuda:{torch.cuda.current_device()}; call under torch.cuda.device({device})")
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if hasattr(stream, "cuda_stream"):  # torch.cuda.Stream / ExternalStream
        if device is not None and stream.device != device:
            raise ValueError(f"stream belongs to {stream.device}, tensors are on {device}")
        return stream.cuda_stream
    return int(stream)


def _check(fn: str, status: int) -> None:
    if status != GPT_ATTN_OK:
        raise AttnError(fn, status)


def _bhtd(name: str, t: torch.Tensor, ref: Optional[torch.Tensor] = None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be bfloat16, got {t.dtype}")
    if t.dim() != 4 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous [B,H,T,d] tensor")
    if ref is not None and (t.shape != ref.shape or t.device != ref.device):
        raise ValueError(f"{name} must match q: {tuple(ref.shape)} on {ref.device}")
    return tuple(t.shape)


def _side(name: str, t: torch.Tensor, shape, dtype, ref: Optional[torch.Tensor] = None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}")
    if ref is not None and t.device != ref.device:
        raise ValueError(f"{name} is on {t.device}, q is on {ref.device}")


def _doc_ptr(doc, B, T, ref=None):
    if doc is None:
        return None
    _side("doc_offsets", doc, (B, T), torch.int32, ref)
    return doc.data_ptr()


def gpt_attn_fwd(q, k, v, o, lse, scale: float, doc_offsets=None, stream=None) -> None:
    B, H, T, d = _bhtd("q", q)
    _bhtd("k", k, q)
    _bhtd("v", v, q)
    _bhtd("o", o, q)
    _side("lse", lse, (B, H, T), torch.float32, q)
    _check("gpt_attn_fwd", load().gpt_attn_fwd(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, T, d,
        float(scale), _doc_ptr(doc_offsets, B, T, q), _stream(stream, q.device)))


def _e4m3(name: str, t: torch.Tensor, ref: Optional[torch.Tensor] = None):
    """A contiguous [B,H,T,d] CUDA tensor of e4m3 codes (torch.float8_e4m3fn or uint8)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in (torch.float8_e4m3fn, torch.uint8):
        raise ValueError(f"{name} must hold e4m3 codes (float8_e4m3fn or uint8), got {t.dtype}")
    if t.dim() != 4 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous [B,H,T,d] tensor")
    if ref is not None and (t.shape != ref.shape or t.device != ref.device):
        raise ValueError(f"{name} must match q8: {tuple(ref.shape)} on {ref.device}")
    return tuple(t.shape)


def gpt_attn_fwd_fp8(q8, k8, v8, descale_q: float, descale_k: float, descale_v: float, o, lse,
                     scale: float, doc_offsets=None, stream=None) -> None:
    """FP8 forward: q8, k8, v8 e4m3 codes [B,H,T,d] standing for descale * code; o bf16
    [B,H,T,d], lse fp32 [B,H,T]."""
    B, H, T, d = _e4m3("q8", q8)
    _e4m3("k8", k8, q8)
    _e4m3("v8", v8, q8)
    _bhtd("o", o)
    if tuple(o.shape) != (B, H, T, d) or o.device != q8.device:
        raise ValueError(f"o must be bf16 {(B, H, T, d)} on {q8.device}")
    _side("lse", lse, (B, H, T), torch.float32, q8)
    _check("gpt_attn_fwd_fp8", load().gpt_attn_fwd_fp8(
        q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), float(descale_q), float(descale_k),
        float(descale_v), o.data_ptr(), lse.data_ptr(), B, H, T, d, float(scale),
        _doc_ptr(doc_offsets, B, T, q8), _stream(stream, q8.device)))


def attention_forward_fp8(q8, k8, v8, descale_q: float, descale_k: float, descale_v: float,
                          scale: Optional[float] = None, doc_offsets=None, stream=None):
    """Allocates O [B,H,T,d] bf16 and LSE [B,H,T] fp32 and runs gpt_attn_fwd_fp8."""
    B, H, T, d = _e4m3("q8", q8)
    if scale is None:
        scale = d ** -0.5
    o = torch.empty(B, H, T, d, device=q8.device, dtype=torch.bfloat16)
    lse = torch.empty(B, H, T, device=q8.device, dtype=torch.float32)
    gpt_attn_fwd_fp8(q8, k8, v8, descale_q, descale_k, descale_v, o, lse, scale, doc_offsets,
                     stream)
    return o, lse


def gpt_attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, delta_ws, scale: float, doc_offsets=None,
                 stream=None) -> None:
    B, H, T, d = _bhtd("q", q)
    for name, t in (("k", k), ("v", v), ("o", o), ("dout", dout), ("dq", dq), ("dk", dk), ("dv", dv)):
        _bhtd(name, t, q)
    _side("lse", lse, (B, H, T), torch.float32, q)
    _side("delta_ws", delta_ws, (B, H, T), torch.float32, q)
    _check("gpt_attn_bwd", load().gpt_attn_bwd(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), delta_ws.data_ptr(), B, H, T, d, float(scale),
        _doc_ptr(doc_offsets, B, T, q), _stream(stream, q.device)))


def gpt_attn_fwd_window(q, k, v, o, lse, scale: float, window: int, doc_offsets=None,
                        stream=None) -> None:
    """gpt_attn_fwd with a sliding window: i attends to j iff i - window < j <= i."""
    B, H, T, d = _bhtd("q", q)
    _bhtd("k", k, q)
    _bhtd("v", v, q)
    _bhtd("o", o, q)
    _side("lse", lse, (B, H, T), torch.float32, q)
    _check("gpt_attn_fwd_window", load().gpt_attn_fwd_window(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, T, d,
        float(scale), _doc_ptr(doc_offsets, B, T, q), int(window), _stream(stream, q.device)))


def gpt_attn_bwd_window(q, k, v, o, dout, lse, dq, dk, dv, delta_ws, scale: float, window: int,
                        doc_offsets=None, stream=None) -> None:
    """gpt_attn_bwd with a sliding window (the one the forward used)."""
    B, H, T, d = _bhtd("q", q)
    for name, t in (("k", k), ("v", v), ("o", o), ("dout", dout), ("dq", dq), ("dk", dk), ("dv", dv)):
        _bhtd(name, t, q)
    _side("lse", lse, (B, H, T), torch.float32, q)
    _side("delta_ws", delta_ws, (B, H, T), torch.float32, q)
    _check("gpt_attn_bwd_window", load().gpt_attn_bwd_window(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), delta_ws.data_ptr(), B, H, T, d, float(scale),
        _doc_ptr(doc_offsets, B, T, q), int(window), _stream(stream, q.device)))


def gpt_attn_bwd_static_ws(q, k, v, o, dout, lse, dq, dk, dv, scale: float, doc_offsets=None,
                           stream=None) -> None:
    """gpt_attn_bwd without a caller workspace: for callers that cannot allocate device memory
    (the delta scratch is a fixed 2^20-row array inside the library; calls share it)."""
    B, H, T, d = _bhtd("q", q)
    for name, t in (("k", k), ("v", v), ("o", o), ("dout", dout), ("dq", dq), ("dk", dk), ("dv", dv)):
        _bhtd(name, t, q)
    _side("lse", lse, (B, H, T), torch.float32, q)
    _check("gpt_attn_bwd_static_ws", load().gpt_attn_bwd_static_ws(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, T, d, float(scale),
        _doc_ptr(doc_offsets, B, T, q), _stream(stream, q.device)))


def gpt_attn_bwd_preprocess(o, dout, delta, stream=None) -> None:
    B, H, T, d = _bhtd("o", o)
    _bhtd("dout", dout, o)
    _side("delta", delta, (B, H, T), torch.float32, o)
    _check("gpt_attn_bwd_preprocess", load().gpt_attn_bwd_preprocess(
        o.data_ptr(), dout.data_ptr(), delta.data_ptr(), B, H, T, d, _stream(stream, o.device)))


def gpt_attn_bwd_dkdv(q, k, v, dout, lse, delta, dk, dv, scale: float, doc_offsets=None,
                      stream=None) -> None:
    B, H, T, d = _bhtd("q", q)
    for name, t in (("k", k), ("v", v), ("dout", dout), ("dk", dk), ("dv", dv)):
        _bhtd(name, t, q)
    _side("lse", lse, (B, H, T), torch.float32, q)
    _side("delta", delta, (B, H, T), torch.float32, q)
    _check("gpt_attn_bwd_dkdv", load().gpt_attn_bwd_dkdv(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(), lse.data_ptr(), delta.data_ptr(),
        dk.data_ptr(), dv.data_ptr(), B, H, T, d, float(scale), _doc_ptr(doc_offsets, B, T, q),
        _stream(stream, q.device)))


def gpt_attn_bwd_dq(q, k, v, dout, lse, delta, dq, scale: float, doc_offsets=None,
                    stream=None) -> None:
    B, H, T, d = _bhtd("q", q)
    for name, t in (("k", k), ("v", v), ("dout", dout), ("dq", dq)):
        _bhtd(name, t, q)
    _side("lse", lse, (B, H, T), torch.float32, q)
    _side("delta", delta, (B, H, T), torch.float32, q)
    _check("gpt_attn_bwd_dq", load().gpt_attn_bwd_dq(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(), lse.data_ptr(), delta.data_ptr(),
        dq.data_ptr(), B, H, T, d, float(scale), _doc_ptr(doc_offsets, B, T, q), _stream(stream, q.device)))


def gpt_attn_bwd_dq_delta(q, k, v, o, dout, lse, delta_out, dq, scale: float, doc_offsets=None,
                          stream=None) -> None:
    """dQ, computing delta = rowsum(dout * o) on the way into delta_out (for gpt_attn_bwd_dkdv)."""
    B, H, T, d = _bhtd("q", q)
    for name, t in (("k", k), ("v", v), ("o", o), ("dout", dout), ("dq", dq)):
        _bhtd(name, t, q)
    _side("lse", lse, (B, H, T), torch.float32, q)
    _side("delta_out", delta_out, (B, H, T), torch.float32, q)
    _check("gpt_attn_bwd_dq_delta", load().gpt_attn_bwd_dq_delta(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
        delta_out.data_ptr(), dq.data_ptr(), B, H, T, d, float(scale),
        _doc_ptr(doc_offsets, B, T, q), _stream(stream, q.device)))


def gpt_attn_decode_workspace_size(B: int, H: int, Tq: int, L: int, d: int) -> int:
    return int(load().gpt_attn_decode_workspace_size(B, H, Tq, L, d))


def gpt_attn_decode(q, k_cache, v_cache, o, lse, workspace, scale: float, stream=None) -> None:
    """q, o: bf16 [B,Tq,H,d]; k_cache, v_cache: bf16 [B,L,H,d]; lse fp32 [B,H,Tq];
    workspace: a CUDA tensor of at least gpt_attn_decode_workspace_size bytes."""
    B, Tq, H, d = _bhtd("q", q)
    Bk, L, Hk, dk = _bhtd("k_cache", k_cache)
    if (Bk, Hk, dk) != (B, H, d):
        raise ValueError("k_cache must be [B, L, H, d] with q's B, H, d")
    _bhtd("v_cache", v_cache, k_cache)
    _bhtd("o", o, q)
    _side("lse", lse, (B, H, Tq), torch.float32, q)
    if (not isinstance(workspace, torch.Tensor) or not workspace.is_cuda
            or not workspace.is_contiguous() or workspace.device != q.device):
        raise ValueError("workspace must be a contiguous CUDA tensor on q's device")
    nbytes = workspace.numel() * workspace.element_size()
    _check("gpt_attn_decode", load().gpt_attn_decode(
        q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), o.data_ptr(), lse.data_ptr(),
        workspace.data_ptr(), nbytes, B, H, Tq, L, d, float(scale), _stream(stream, q.device)))


def gpt_attn_check_doc_offsets(doc_offsets, stream=None) -> bool:
    """True when the [B,T] int32 device array is a valid document-start array."""
    if not isinstance(doc_offsets, torch.Tensor) or doc_offsets.dim() != 2:
        raise ValueError("doc_offsets must be a [B,T] tensor")
    B, T = doc_offsets.shape
    _side("doc_offsets", doc_offsets, (B, T), torch.int32)
    s = load().gpt_attn_check_doc_offsets(doc_offsets.data_ptr(), B, T,
                                             _stream(stream, doc_offsets.device))
    if s == GPT_ATTN_ERR_BAD_DOC_OFFSETS:
        return False
    _check("gpt_attn_check_doc_offsets", s)
    return True


def gpt_attn_device_status(clear: bool = False) -> int:
    out = ctypes.c_uint(0)
    _check("gpt_attn_device_status", load().gpt_attn_device_status(ctypes.byref(out), int(clear)))
    return int(out.value)


def gpt_attn_selftest_wait_timeout(limit_ns: int, stream=None) -> int:
    """Runs the bounded-wait self-test; returns the raw status (DEVICE_TIMEOUT expected)."""
    return int(load().gpt_attn_selftest_wait_timeout(int(limit_ns), _stream(stream)))


# ------------------------------------------------------------ prepared calls

class PreparedCall:
    """One library call whose arguments were checked and marshalled once: calling it re-issues
    the C call with the same device pointers, sizes and stream (a few microseconds of host time
    instead of the binding's per-call checks).  The tensors must stay alive and unmoved (they
    are referenced here); their contents may change between calls."""

    def __init__(self, name: str, args, keep):
        self._fn = getattr(load(), name)
        self._name = name
        # converted to ctypes values once, so a call does not convert Python numbers again
        self._args = tuple(t(a) if a is not None else None
                           for t, a in zip(SIGNATURES[name][0], args))
        self._keep = keep  # the tensors whose pointers are in _args

    def __call__(self) -> None:
        st = self._fn(*self._args)
        if st:
            raise AttnError(self._name, st)


def _capture(fn, *a, **kw):
    """Runs fn's checks and argument marshalling without calling the library: returns the
    (name, args) it would pass to the C function."""
    captured = {}

    class _Recorder:
        def __getattr__(self, name):
            def rec(*args):
                if "call" in captured:
                    raise ValueError("prepare() needs a function that makes one library call")
                captured["call"] = (name, args)
                return GPT_ATTN_OK
            return rec
    load()  # the real library must be there: a prepared call will use it
    _tls.recorder = _Recorder()
    try:
        fn(*a, **kw)
    finally:
        _tls.recorder = None
    if "call" not in captured:
        raise ValueError("prepare() needs a function that makes one library call")
    return captured["call"]


def prepare(fn, *args, **kwargs) -> PreparedCall:
    """prepare(gpt_attn_fwd, q, k, v, o, lse, scale, ...) -> a PreparedCall re-issuing that call.
    Works for every binding function that makes exactly one library call."""
    name, cargs = _capture(fn, *args, **kwargs)
    keep = [x for x in args if isinstance(x, torch.Tensor)]
    keep += [x for x in kwargs.values() if isinstance(x, torch.Tensor)]
    return PreparedCall(name, cargs, keep)


# ------------------------------------------------------------ conveniences

def attention_forward(q, k, v, scale: Optional[float] = None, doc_offsets=None, stream=None,
                      window: Optional[int] = None):
    """Allocates O [B,H,T,d] bf16 and LSE [B,H,T] fp32 and runs gpt_attn_fwd (or, with a
    window, gpt_attn_fwd_window)."""
    B, H, T, d = _bhtd("q", q)
    if scale is None:
        scale = d ** -0.5
    o = torch.empty_like(q)
    lse = torch.empty(B, H, T, device=q.device, dtype=torch.float32)
    if window is None:
        gpt_attn_fwd(q, k, v, o, lse, scale, doc_offsets, stream)
    else:
        gpt_attn_fwd_window(q, k, v, o, lse, scale, window, doc_offsets, stream)
    return o, lse


def attention_backward(q, k, v, o, lse, dout, scale: Optional[float] = None, doc_offsets=None,
                       stream=None, window: Optional[int] = None):
    """Allocates dQ, dK, dV and the delta workspace and runs gpt_attn_bwd (or, with a
    window, gpt_attn_bwd_window)."""
    B, H, T, d = _bhtd("q", q)
    if scale is None:
        scale = d ** -0.5
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    delta = torch.empty(B, H, T, device=q.device, dtype=torch.float32)
    if window is None:
        gpt_attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, delta, scale, doc_offsets, stream)
    else:
        gpt_attn_bwd_window(q, k, v, o, dout, lse, dq, dk, dv, delta, scale, window, doc_offsets,
                            stream)
    return dq, dk, dv


def attention_decode(q, k_cache, v_cache, scale: Optional[float] = None, stream=None):
    """Allocates O [B,Tq,H,d] bf16, LSE [B,H,Tq] fp32 and the workspace; runs gpt_attn_decode."""
    B, Tq, H, d = _bhtd("q", q)
    L = k_cache.shape[1]
    if scale is None:
        scale = d ** -0.5
    o = torch.empty_like(q)
    lse = torch.empty(B, H, Tq, device=q.device, dtype=torch.float32)
    ws = torch.empty(max(gpt_attn_decode_workspace_size(B, H, Tq, L, d), 16), device=q.device,
                     dtype=torch.uint8)
    gpt_attn_decode(q, k_cache, v_cache, o, lse, ws, scale, stream)
    return o, lse


def _span(t: torch.Tensor):
    return t.data_ptr(), t.data_ptr() + t.numel() * t.element_size()


def _same_or_disjoint(name: str, out: torch.Tensor, allowed: torch.Tensor, others) -> None:
    """out may be exactly `allowed` (in place) but must not otherwise overlap it or `others`."""
    lo, hi = _span(out)
    if _span(allowed) != (lo, hi):
        others = (allowed, *others)
    for t in others:
        a, b = _span(t)
        if a < hi and lo < b:
            raise ValueError(f"{name} overlaps another argument")


def gpt_attn_rope_qknorm_fwd(q, k, q_out, k_out, rope_base: float = 10000.0, gain: float = 1.2,
                             eps: float = 1e-6, stream=None) -> None:
    """RoPE (positions 0..T-1) then RMS norm times `gain`, on q and k [B,H,T,d] in one launch.
    q_out may be q and k_out may be k (in place)."""
    B, H, T, d = _bhtd("q", q)
    _bhtd("k", k, q)
    _bhtd("q_out", q_out, q)
    _bhtd("k_out", k_out, q)
    _same_or_disjoint("q_out", q_out, q, (k, k_out))
    _same_or_disjoint("k_out", k_out, k, (q, q_out))
    _check("gpt_attn_rope_qknorm_fwd", load().gpt_attn_rope_qknorm_fwd(
        q.data_ptr(), k.data_ptr(), q_out.data_ptr(), k_out.data_ptr(), B, H, T, d,
        float(rope_base), float(gain), float(eps), _stream(stream, q.device)))


def gpt_attn_rope_qknorm_bwd(q, k, dq_out, dk_out, dq, dk, rope_base: float = 10000.0,
                             gain: float = 1.2, eps: float = 1e-6, stream=None) -> None:
    """Gradients with respect to the prologue's inputs q, k from those with respect to its
    outputs.  dq may be dq_out and dk may be dk_out (in place)."""
    B, H, T, d = _bhtd("q", q)
    for name, t in (("k", k), ("dq_out", dq_out), ("dk_out", dk_out), ("dq", dq), ("dk", dk)):
        _bhtd(name, t, q)
    _same_or_disjoint("dq", dq, dq_out, (q, k, dk_out, dk))
    _same_or_disjoint("dk", dk, dk_out, (q, k, dq_out, dq))
    _check("gpt_attn_rope_qknorm_bwd", load().gpt_attn_rope_qknorm_bwd(
        q.data_ptr(), k.data_ptr(), dq_out.data_ptr(), dk_out.data_ptr(), dq.data_ptr(),
        dk.data_ptr(), B, H, T, d, float(rope_base), float(gain), float(eps), _stream(stream, q.device)))


def rope_qknorm(q, k, rope_base: float = 10000.0, gain: float = 1.2, eps: float = 1e-6,
                stream=None):
    """Allocates and returns (q', k') = the prologue of q and k."""
    q_out, k_out = torch.empty_like(q), torch.empty_like(k)
    gpt_attn_rope_qknorm_fwd(q, k, q_out, k_out, rope_base, gain, eps, stream)
    return q_out, k_out


class RopeQKNormFunction(torch.autograd.Function):
    """torch.autograd wrapper of the prologue; the backward recomputes from the saved inputs."""

    @staticmethod
    def forward(ctx, q, k, rope_base, gain, eps):
        ctx.save_for_backward(q, k)
        ctx.args = (rope_base, gain, eps)
        return rope_qknorm(q, k, rope_base, gain, eps)

    @staticmethod
    def backward(ctx, dq_out, dk_out):
        q, k = ctx.saved_tensors
        dq_out, dk_out = dq_out.contiguous(), dk_out.contiguous()
        dq, dk = torch.empty_like(q), torch.empty_like(k)
        gpt_attn_rope_qknorm_bwd(q, k, dq_out, dk_out, dq, dk, *ctx.args)
        return dq, dk, None, None, None


def rope_qk_norm(q, k, rope_base: float = 10000.0, gain: float = 1.2, eps: float = 1e-6):
    """Autograd form: (q', k') with gradients through the library's backward kernel."""
    return RopeQKNormFunction.apply(q, k, rope_base, gain, eps)


class CausalSelfAttentionFunction(torch.autograd.Function):
    """torch.autograd wrapper: y = attention(q, k, v) with the library's fwd/bwd kernels."""

    @staticmethod
    def forward(ctx, q, k, v, scale, doc_offsets):
        o, lse = attention_forward(q, k, v, scale, doc_offsets)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.scale, ctx.doc = scale, doc_offsets
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = attention_backward(q, k, v, o, lse, dout.contiguous(), ctx.scale, ctx.doc)
        return dq, dk, dv, None, None


def causal_attention(q, k, v, scale: Optional[float] = None, doc_offsets=None):
    if scale is None:
        scale = q.shape[-1] ** -0.5
    return CausalSelfAttentionFunction.apply(q, k, v, scale, doc_offsets)


class HostStep:
    """Forward + backward on pinned HOST tensors: copies the step's inputs to the
    device, runs gpt_attn_fwd and gpt_attn_bwd, and copies O, LSE, dQ, dK, dV back
    into caller-provided pinned host tensors, all on one stream.  The device
    buffers are allocated once, here, by torch."""

    def __init__(self, B: int, H: int, T: int, d: int, device="cuda"):
        dev = torch.device(device)
        bf = dict(device=dev, dtype=torch.bfloat16)
        self.q, self.k, self.v, self.do, self.o, self.dq, self.dk, self.dv = (
            torch.empty(B, H, T, d, **bf) for _ in range(8))
        self.lse = torch.empty(B, H, T, device=dev, dtype=torch.float32)
        self.delta = torch.empty(B, H, T, device=dev, dtype=torch.float32)
        self.doc = None
        self.shape = (B, H, T, d)

    def set_doc_offsets(self, doc_host):
        self.doc = None if doc_host is None else doc_host.to(self.q.device).contiguous()

    def h2d_bytes(self) -> int:
        return 4 * self.q.numel() * 2

    def d2h_bytes(self) -> int:
        return 4 * self.q.numel() * 2 + self.lse.numel() * 4

    def run(self, q_h, k_h, v_h, do_h, out_h, scale: float, stream=None) -> None:
        """out_h: dict with pinned host tensors 'o', 'lse', 'dq', 'dk', 'dv'.  Asynchronous."""
        s = stream or torch.cuda.current_stream()
        with torch.cuda.stream(s):
            for dst, src in ((self.q, q_h), (self.k, k_h), (self.v, v_h), (self.do, do_h)):
                dst.copy_(src, non_blocking=True)
            gpt_attn_fwd(self.q, self.k, self.v, self.o, self.lse, scale, self.doc, s)
            gpt_attn_bwd(self.q, self.k, self.v, self.o, self.do, self.lse, self.dq, self.dk,
                         self.dv, self.delta, scale, self.doc, s)
            for name in ("o", "lse", "dq", "dk", "dv"):
                out_h[name].copy_(getattr(self, name), non_blocking=True)


class HostStream:
    """Forward + backward over a sequence of steps whose inputs and outputs all
    live in pinned HOST memory, with neighbouring steps overlapped: while step k
    computes, step k+1's inputs are copied in and step k-1's outputs copied out
    (host-to-device and device-to-host copies use opposite directions of the bus,
    so they run at the same time).  Two sets of device buffers alternate between
    steps; three CUDA streams carry the copies in, the kernels and the copies
    out, ordered by events.  Every step still moves all of its inputs to the
    device and all of its outputs (O, LSE, dQ, dK, dV) back."""

    def __init__(self, B: int, H: int, T: int, d: int, device="cuda"):
        dev = torch.device(device)
        self.sets = [HostStep(B, H, T, d, dev) for _ in range(2)]
        self.s_in, self.s_comp, self.s_out = (torch.cuda.Stream(dev) for _ in range(3))
        self.device = dev

    def set_doc_offsets(self, doc_host):
        for st in self.sets:
            st.set_doc_offsets(doc_host)

    def h2d_bytes(self) -> int:
        return self.sets[0].h2d_bytes()

    def d2h_bytes(self) -> int:
        return self.sets[0].d2h_bytes()

    def run(self, steps, scale: float, after=None):
        """steps: sequence of (q_h, k_h, v_h, do_h, out_h); out_h is a dict of pinned host
        tensors 'o', 'lse', 'dq', 'dk', 'dv'.  `after`: an optional CUDA event the first copy
        waits for.  Enqueues everything and returns the event recorded after the last copy
        out (asynchronous: synchronise on it before reading the outputs)."""
        ev_comp, ev_out = [], []
        for k, (q_h, k_h, v_h, do_h, out_h) in enumerate(steps):
            st = self.sets[k % 2]
            if k == 0 and after is not None:
                self.s_in.wait_event(after)
            if k >= 2:  # set k % 2 holds step k-2's inputs until its kernels have read them
                self.s_in.wait_event(ev_comp[k - 2])
            with torch.cuda.stream(self.s_in):
                for dst, src in ((st.q, q_h), (st.k, k_h), (st.v, v_h), (st.do, do_h)):
                    dst.copy_(src, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(self.s_in)
            self.s_comp.wait_event(ev_in)
            if k >= 2:  # ... and step k-2's outputs until they have been copied out
                self.s_comp.wait_event(ev_out[k - 2])
            gpt_attn_fwd(st.q, st.k, st.v, st.o, st.lse, scale, st.doc, self.s_comp)
            gpt_attn_bwd(st.q, st.k, st.v, st.o, st.do, st.lse, st.dq, st.dk, st.dv, st.delta,
                         scale, st.doc, self.s_comp)
            ec = torch.cuda.Event()
            ec.record(self.s_comp)
            ev_comp.append(ec)
            self.s_out.wait_event(ec)
            with torch.cuda.stream(self.s_out):
                for name in ("o", "lse", "dq", "dk", "dv"):
                    out_h[name].copy_(getattr(st, name), non_blocking=True)
                eo = torch.cuda.Event()
                eo.record(self.s_out)
            ev_out.append(eo)
        return ev_out[-1] if ev_out else None

