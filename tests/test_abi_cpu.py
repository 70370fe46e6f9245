"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and rejects bad arguments before making any CUDA call."""
import ctypes
import math
import os
import re

import pytest
import torch

from causal_self_attention_mha_b200 import abi, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "causalattn.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return abi.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gpt_attn_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "gpt_attn_fwd" in names and "gpt_attn_bwd" in names
    for n in names:
        assert hasattr(lib, n), n
        assert n in abi.SIGNATURES, f"binding lacks {n}"


def test_version_and_strerror(lib):
    assert lib.gpt_attn_version() == 1
    for s in range(0, 14):
        msg = lib.gpt_attn_strerror(s)
        assert isinstance(msg, bytes) and len(msg) > 0
    assert lib.gpt_attn_strerror(999) == b"unknown status"


# fake, never-dereferenced, 16-byte aligned addresses: validation must reject before use
P = [0x10000 + 0x100 * i for i in range(12)]


def fwd(lib, q=P[0], k=P[1], v=P[2], o=P[3], lse=P[4], B=1, H=2, T=64, d=64, scale=0.125, doc=None):
    return lib.gpt_attn_fwd(q, k, v, o, lse, B, H, T, d, scale, doc, None)


def test_fwd_argument_errors(lib):
    assert fwd(lib, q=None) == abi.GPT_ATTN_ERR_NULL_PTR
    assert fwd(lib, lse=None) == abi.GPT_ATTN_ERR_NULL_PTR
    assert fwd(lib, B=0) == abi.GPT_ATTN_ERR_BAD_SHAPE
    assert fwd(lib, T=0) == abi.GPT_ATTN_ERR_BAD_SHAPE
    assert fwd(lib, H=-1) == abi.GPT_ATTN_ERR_BAD_SHAPE
    for d in (16, 48, 96, 256):
        assert fwd(lib, d=d) == abi.GPT_ATTN_ERR_UNSUPPORTED_HEAD_DIM
    for s in (0.0, -1.0, math.inf, math.nan):
        assert fwd(lib, scale=s) == abi.GPT_ATTN_ERR_BAD_SCALE
    assert fwd(lib, q=P[0] + 8) == abi.GPT_ATTN_ERR_MISALIGNED
    assert fwd(lib, o=P[3] + 2) == abi.GPT_ATTN_ERR_MISALIGNED
    assert fwd(lib, lse=P[4] + 2) == abi.GPT_ATTN_ERR_MISALIGNED
    assert fwd(lib, doc=P[5] + 1) == abi.GPT_ATTN_ERR_MISALIGNED
    assert fwd(lib, B=1 << 12, H=1 << 12, T=1 << 10, d=128) == abi.GPT_ATTN_ERR_TOO_LARGE


def test_bwd_argument_errors(lib):
    def bwd(**kw):
        a = dict(q=P[0], k=P[1], v=P[2], o=P[3], do=P[4], lse=P[5], dq=P[6], dk=P[7], dv=P[8],
                 delta=P[9], B=1, H=2, T=64, d=64, scale=0.125, doc=None)
        a.update(kw)
        return lib.gpt_attn_bwd(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"],
                                a["dv"], a["delta"], a["B"], a["H"], a["T"], a["d"], a["scale"],
                                a["doc"], None)
    for name in ("q", "k", "v", "o", "do", "lse", "dq", "dk", "dv", "delta"):
        assert bwd(**{name: None}) == abi.GPT_ATTN_ERR_NULL_PTR, name
    assert bwd(T=0) == abi.GPT_ATTN_ERR_BAD_SHAPE
    assert bwd(d=80) == abi.GPT_ATTN_ERR_UNSUPPORTED_HEAD_DIM
    assert bwd(scale=-0.5) == abi.GPT_ATTN_ERR_BAD_SCALE
    assert bwd(dk=P[7] + 4) == abi.GPT_ATTN_ERR_MISALIGNED
    assert lib.gpt_attn_bwd_preprocess(P[0], None, P[2], 1, 1, 8, 32, None) == abi.GPT_ATTN_ERR_NULL_PTR
    assert lib.gpt_attn_bwd_dkdv(P[0], P[1], P[2], P[3], P[4], P[5], P[6], None, 1, 1, 8, 32, 0.1,
                                 None, None) == abi.GPT_ATTN_ERR_NULL_PTR
    assert lib.gpt_attn_bwd_dq(P[0], P[1], P[2], P[3], P[4], P[5], P[6], 1, 1, 8, 40, 0.1,
                               None, None) == abi.GPT_ATTN_ERR_UNSUPPORTED_HEAD_DIM
    assert lib.gpt_attn_check_doc_offsets(None, 1, 8, None) == abi.GPT_ATTN_ERR_NULL_PTR
    assert lib.gpt_attn_check_doc_offsets(P[0], 0, 8, None) == abi.GPT_ATTN_ERR_BAD_SHAPE
    out = ctypes.c_uint(0)
    assert lib.gpt_attn_device_status(None, 0) == abi.GPT_ATTN_ERR_NULL_PTR


def test_window_entry_points_validate_like_the_plain_ones(lib):
    def fw(q=P[0], B=1, d=64, window=16, scale=0.125):
        return lib.gpt_attn_fwd_window(q, P[1], P[2], P[3], P[4], B, 2, 64, d, scale, None,
                                       window, None)

    def bw(dq=P[6], T=64, d=64, window=16):
        return lib.gpt_attn_bwd_window(P[0], P[1], P[2], P[3], P[5], P[4], dq, P[7], P[8], P[9],
                                       1, 2, T, d, 0.125, None, window, None)
    assert fw(q=None) == abi.GPT_ATTN_ERR_NULL_PTR
    assert fw(B=0) == abi.GPT_ATTN_ERR_BAD_SHAPE
    assert fw(d=48) == abi.GPT_ATTN_ERR_UNSUPPORTED_HEAD_DIM
    assert fw(scale=-1.0) == abi.GPT_ATTN_ERR_BAD_SCALE
    assert fw(q=P[0] + 2) == abi.GPT_ATTN_ERR_MISALIGNED
    assert bw(dq=None) == abi.GPT_ATTN_ERR_NULL_PTR
    assert bw(T=0) == abi.GPT_ATTN_ERR_BAD_SHAPE
    assert bw(d=96) == abi.GPT_ATTN_ERR_UNSUPPORTED_HEAD_DIM
    if not torch.cuda.is_available():  # any window value is valid: only the device is missing
        for w in (-5, 0, 1, 63, 64, 10 ** 6):
            assert fw(window=w) == abi.GPT_ATTN_ERR_NO_DEVICE
            assert bw(window=w) == abi.GPT_ATTN_ERR_NO_DEVICE


def test_decode_validation(lib):
    ws = lib.gpt_attn_decode_workspace_size
    assert ws(2, 4, 1, 1000, 128) == 2 * 4 * 1 * 8 * (2 + 128) * 4   # 8 chunks of 128 keys
    assert ws(1, 1, 16, 16, 32) > 0
    for bad in ((0, 4, 1, 100, 64), (1, 0, 1, 100, 64), (1, 1, 0, 100, 64), (1, 1, 17, 100, 64),
                (1, 1, 5, 4, 64), (1, 1, 1, 100, 48)):
        assert ws(*bad) == 0

    def dec(q=P[0], B=1, H=2, Tq=1, L=300, d=64, wsb=1 << 20, scale=0.125):
        return lib.gpt_attn_decode(q, P[1], P[2], P[3], P[4], P[5], wsb, B, H, Tq, L, d, scale,
                                   None)
    assert dec(q=None) == abi.GPT_ATTN_ERR_NULL_PTR
    assert dec(Tq=0) == abi.GPT_ATTN_ERR_BAD_SHAPE
    assert dec(Tq=17, L=300) == abi.GPT_ATTN_ERR_BAD_SHAPE
    assert dec(Tq=5, L=4) == abi.GPT_ATTN_ERR_BAD_SHAPE
    assert dec(d=96) == abi.GPT_ATTN_ERR_UNSUPPORTED_HEAD_DIM
    assert dec(scale=0.0) == abi.GPT_ATTN_ERR_BAD_SCALE
    assert dec(q=P[0] + 8) == abi.GPT_ATTN_ERR_MISALIGNED
    assert dec(wsb=16) == abi.GPT_ATTN_ERR_BAD_SHAPE        # workspace too small
    if not torch.cuda.is_available():
        assert dec() == abi.GPT_ATTN_ERR_NO_DEVICE


def test_prologue_validation(lib):
    def fwd_(q=P[0], k=P[1], qo=P[2], ko=P[3], B=1, H=2, T=64, d=64, base=10000.0, gain=1.2,
             eps=1e-6):
        return lib.gpt_attn_rope_qknorm_fwd(q, k, qo, ko, B, H, T, d, base, gain, eps, None)

    def bwd_(dqo=P[2], dq=P[4], **kw):
        a = dict(q=P[0], k=P[1], dko=P[3], dk=P[5], B=1, H=2, T=64, d=64, base=10000.0,
                 gain=1.2, eps=1e-6)
        a.update(kw)
        return lib.gpt_attn_rope_qknorm_bwd(a["q"], a["k"], dqo, a["dko"], dq, a["dk"], a["B"],
                                            a["H"], a["T"], a["d"], a["base"], a["gain"],
                                            a["eps"], None)
    for call in (fwd_, bwd_):
        assert call(B=0) == abi.GPT_ATTN_ERR_BAD_SHAPE
        assert call(T=0) == abi.GPT_ATTN_ERR_BAD_SHAPE
        assert call(d=48) == abi.GPT_ATTN_ERR_UNSUPPORTED_HEAD_DIM
        assert call(B=4096, H=64, T=4096, d=128) == abi.GPT_ATTN_ERR_TOO_LARGE
        for bad in (dict(base=0.0), dict(base=-2.0), dict(base=math.inf), dict(base=math.nan),
                    dict(gain=math.nan), dict(gain=math.inf), dict(eps=-1e-6), dict(eps=math.nan)):
            assert call(**bad) == abi.GPT_ATTN_ERR_BAD_PARAM, bad
        assert call(q=P[0] + 8) == abi.GPT_ATTN_ERR_MISALIGNED
        assert call(k=None) == abi.GPT_ATTN_ERR_NULL_PTR
        if not torch.cuda.is_available():
            assert call() == abi.GPT_ATTN_ERR_NO_DEVICE
            assert call(gain=-1.2, eps=0.0) == abi.GPT_ATTN_ERR_NO_DEVICE  # both are valid
    assert fwd_(qo=None) == abi.GPT_ATTN_ERR_NULL_PTR
    assert bwd_(dqo=None) == abi.GPT_ATTN_ERR_NULL_PTR
    assert bwd_(dq=P[4] + 2) == abi.GPT_ATTN_ERR_MISALIGNED


def test_prologue_binding_overlap_rule():
    buf = torch.zeros(4 * 1024, dtype=torch.bfloat16)
    a, b = buf[:1024], buf[1024:2048]
    abi._same_or_disjoint("out", a, a, (b,))                 # in place: allowed
    abi._same_or_disjoint("out", b, a, (buf[2048:3072],))    # disjoint: allowed
    with pytest.raises(ValueError):
        abi._same_or_disjoint("out", buf[512:1536], a, ())   # partial overlap with its input
    with pytest.raises(ValueError):
        abi._same_or_disjoint("out", a, a, (buf[1000:1100],))  # overlaps another argument


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_valid_arguments_without_a_gpu_report_no_device(lib):
    assert fwd(lib) == abi.GPT_ATTN_ERR_NO_DEVICE
    assert lib.gpt_attn_selftest_wait_timeout(1000, None) == abi.GPT_ATTN_ERR_NO_DEVICE


def test_binding_rejects_host_tensors(lib):
    q = torch.zeros(1, 1, 8, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        abi.gpt_attn_fwd(q, q, q, q, torch.zeros(1, 1, 8), 0.1)


def test_binding_rejects_tensors_off_the_current_device(monkeypatch):
    """The library launches on the current CUDA device: the binding refuses tensors on another
    device (and a stream of another device) before any pointer reaches the C ABI."""
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    with pytest.raises(ValueError, match="current CUDA device"):
        abi._stream(None, torch.device("cuda", 1))

    class FakeStream:  # what the binding reads of a torch.cuda.Stream
        cuda_stream = 0x1234
        device = torch.device("cuda", 1)

    with pytest.raises(ValueError, match="stream belongs to"):
        abi._stream(FakeStream(), torch.device("cuda", 0))


def test_fp8_forward_argument_errors(lib):
    def f8(q=P[0], k=P[1], v=P[2], dq=0.03, dk=0.03, dv=0.03, o=P[3], lse=P[4], B=1, H=2, T=64,
           d=64, scale=0.125, doc=None):
        return lib.gpt_attn_fwd_fp8(q, k, v, dq, dk, dv, o, lse, B, H, T, d, scale, doc, None)
    for name in ("q", "k", "v", "o", "lse"):
        assert f8(**{name: None}) == abi.GPT_ATTN_ERR_NULL_PTR, name
    for name in ("dq", "dk", "dv"):
        for bad in (0.0, -1.0, math.inf, math.nan):
            assert f8(**{name: bad}) == abi.GPT_ATTN_ERR_BAD_PARAM, (name, bad)
    assert f8(dq=1e-20, dk=1e-20) == abi.GPT_ATTN_ERR_BAD_PARAM  # combined scale underflows
    assert f8(scale=0.0) == abi.GPT_ATTN_ERR_BAD_SCALE
    assert f8(d=96) == abi.GPT_ATTN_ERR_UNSUPPORTED_HEAD_DIM
    assert f8(T=0) == abi.GPT_ATTN_ERR_BAD_SHAPE
    assert f8(q=P[0] + 8) == abi.GPT_ATTN_ERR_MISALIGNED
    assert f8(lse=P[4] + 2) == abi.GPT_ATTN_ERR_MISALIGNED


def test_prepare_records_the_marshalled_call(lib, monkeypatch):
    """prepare() runs the binding's checks and marshalling once, without calling the library,
    and keeps exactly the arguments the binding would pass."""
    calls = []

    class FakeFn:
        def __init__(self, name):
            self.name = name

        def __call__(self, *args):
            calls.append((self.name, args))
            return 0

    class FakeLib:
        def __getattr__(self, name):
            return FakeFn(name)

    def fake_fwd(q, scale, stream=None):  # a binding-shaped function: checks, then one call
        if scale <= 0:
            raise ValueError("scale")
        abi._check("gpt_attn_fwd", abi.load().gpt_attn_fwd(
            0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 1, 2, 64, 64, float(scale), None, 0))

    pc = abi.prepare(fake_fwd, None, 0.125)
    assert pc._name == "gpt_attn_fwd" and len(pc._args) == 12
    assert pc._args[9].value == 0.125 and pc._args[10] is None
    monkeypatch.setattr(pc, "_fn", FakeFn("gpt_attn_fwd"))
    pc()
    pc()
    assert len(calls) == 2 and calls[0][1][9].value == 0.125
    with pytest.raises(ValueError):
        abi.prepare(fake_fwd, None, -1.0)  # the checks run at prepare time

    def two_calls():
        abi.load().gpt_attn_version()
        abi.load().gpt_attn_version()
    with pytest.raises(ValueError, match="one library call"):
        abi.prepare(two_calls)


def test_debug_checks_library_exports_every_symbol(lib):
    """libcausalattn_debug.so (the same sources with device-side bounds checks) is a drop-in
    replacement: it exports every declared entry point, and its validation behaves alike."""
    path = build.build(debug=True)
    dbg = abi.load(path)  # sets argtypes for every declared symbol (raises if one is missing)
    assert dbg.gpt_attn_version() == lib.gpt_attn_version()
    for name in declared_functions():
        assert hasattr(dbg, name), name
    assert dbg.gpt_attn_strerror(-1) == lib.gpt_attn_strerror(-1)


def test_debug_build_command_defines_the_checks():
    cmd = build.nvcc_command("out.so", debug=True)
    assert "-DCA_DEBUG_CHECKS" in cmd and "arch=compute_100a,code=sm_100a" in cmd
    assert "-DCA_DEBUG_CHECKS" not in build.nvcc_command("out.so")
