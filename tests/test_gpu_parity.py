"""GPU parity: the CUDA path through the C ABI against the CPU fp64 oracle, on
the same seeded bf16 inputs.

Tolerances (bf16 inputs, fp32 accumulation, bf16 outputs):
  O    max |gpu - oracle|                       <= 1e-2
  LSE  max |gpu - oracle|                       <= 1e-3
  dQ, dK, dV  ||gpu - oracle||_2 / ||oracle||_2  <= 2e-2   (per tensor; ||oracle|| floored
              at 1e-3 RMS so that exactly-zero gradients are measured in absolute terms)
  RoPE + QK-norm prologue (Q', K', dQ, dK): every element within
              |gpu - oracle| <= 2^-8 |oracle| + 2e-3 (bf16 rounding of the output)
The full-size workloads run in the same launch configuration the benchmark
times and are compared on every head, forward and backward (the persistent
kernels hand different heads to different CTAs in different rounds, so every
head is a schedule path of its own).
"""
import numpy as np
import pytest
import torch

import oracle
from causal_self_attention_mha_b200 import abi, inputs

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL, GRAD_TOL = 1e-2, 1e-3, 2e-2


def run_gpu(q, k, v, do, doc, scale, window=None):
    dev = torch.device("cuda:0")
    q, k, v, do = (t.to(dev).contiguous() for t in (q, k, v, do))
    docd = doc.to(dev).contiguous() if doc is not None else None
    o, lse = abi.attention_forward(q, k, v, scale, docd, window=window)
    dq, dk, dv = abi.attention_backward(q, k, v, o, lse, do, scale, docd, window=window)
    torch.cuda.synchronize()
    return [t.cpu() for t in (o, lse, dq, dk, dv)]


def oracle_heads(q, k, v, do, doc, scale, heads, with_grad=True, window=None):
    """Oracle outputs for the listed (b, h) pairs: dict (b,h) -> (o, lse, dq, dk, dv)."""
    out = {}
    for b, h in heads:
        sl = lambda t: t[b:b + 1, h:h + 1]
        ds = doc[b:b + 1] if doc is not None else None
        o, lse = oracle.attention_forward(sl(q), sl(k), sl(v), scale, ds, window=window)
        g = (oracle.attention_backward(sl(q), sl(k), sl(v), sl(do), scale, ds, window=window)
             if with_grad else None)
        out[(b, h)] = (o, lse, g)
    return out


def rel_l2(a, b):
    """||a - b|| / ||b||, with ||b|| floored at an RMS of 1e-3 per element: where the exact
    gradient is zero (T = 1, uniform V) the GPU's fp32 rounding residue is measured absolutely."""
    floor = 1e-3 * np.sqrt(b.size)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), floor))


def compare(gpu, q, k, v, do, doc, scale, grad_heads=None, label="", window=None):
    """Forward on every head (one oracle call); backward on grad_heads (None = all)."""
    o_g, lse_g, dq_g, dk_g, dv_g = (t.to(torch.float64).numpy() for t in gpu)
    B, H = q.shape[:2]
    o_r, lse_r = oracle.attention_forward(q, k, v, scale, doc, window=window)
    err_o = float(np.max(np.abs(o_g - o_r)))
    err_l = float(np.max(np.abs(lse_g - lse_r)))
    if grad_heads is None:
        dq_r, dk_r, dv_r = oracle.attention_backward(q, k, v, do, scale, doc, window=window)
        sel = (slice(None), slice(None))
        errs = [rel_l2(g[sel], r) for g, r in ((dq_g, dq_r), (dk_g, dk_r), (dv_g, dv_r))]
    else:
        ref = oracle_heads(q, k, v, do, doc, scale, grad_heads, window=window)
        errs = []
        for i, g in enumerate((dq_g, dk_g, dv_g)):
            gs = np.concatenate([g[b, h].ravel() for b, h in grad_heads])
            rs = np.concatenate([ref[(b, h)][2][i].ravel() for b, h in grad_heads])
            errs.append(rel_l2(gs, rs))
    print(f"{label}: O maxabs {err_o:.3e}  LSE maxabs {err_l:.3e}  "
          f"dQ {errs[0]:.3e} dK {errs[1]:.3e} dV {errs[2]:.3e}")
    assert np.all(np.isfinite(o_g)) and np.all(np.isfinite(lse_g))
    assert err_o <= O_TOL, (label, "O", err_o)
    assert err_l <= LSE_TOL, (label, "LSE", err_l)
    for name, e in zip(("dQ", "dK", "dV"), errs):
        assert e <= GRAD_TOL, (label, name, e)
    return err_o, err_l, errs


def no_device_timeouts():
    st = abi.gpt_attn_device_status(clear=True)
    assert st == 0, f"device status word {st:#x}: a kernel gave up on a wait"


# ------------------------------------------------------------ full workloads

@pytest.mark.parametrize("name", list(inputs.WORKLOADS))
def test_workload_parity(name, cuda_device):
    w = inputs.WORKLOADS[name]
    q, k, v, do, doc = inputs.make_workload(w)
    gpu = run_gpu(q, k, v, do, doc, w.scale)
    compare(gpu, q, k, v, do, doc, w.scale, None, label=name)  # every head, every element
    no_device_timeouts()


# ------------------------------------------------- tails, tiny and odd shapes

@pytest.mark.parametrize("T", [1, 2, 17, 63, 64, 65, 127, 128, 129, 200, 255, 257, 300])
@pytest.mark.parametrize("d", [32, 64, 128])
def test_ragged_lengths(T, d, cuda_device):
    B, H = 1, 2
    q, k, v, do = inputs.make_qkvdo(B, H, T, d, 1000 + T + d)
    scale = inputs.fp32_scale(d)
    compare(run_gpu(q, k, v, do, None, scale), q, k, v, do, None, scale, label=f"T{T} d{d}")
    no_device_timeouts()


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("lo,hi", [(1, 4), (5, 40), (60, 300)])
def test_document_masks(d, lo, hi, cuda_device):
    B, H, T = 2, 2, 389
    q, k, v, do = inputs.make_qkvdo(B, H, T, d, 7 * lo + d)
    doc = inputs.random_doc_start(B, T, lo + hi, lo, hi)
    scale = inputs.fp32_scale(d)
    compare(run_gpu(q, k, v, do, doc, scale), q, k, v, do, doc, scale, label=f"doc[{lo},{hi}] d{d}")
    no_device_timeouts()


def test_many_tiles_one_head(cuda_device):
    B, H, T, d = 1, 1, 4096, 64
    q, k, v, do = inputs.make_qkvdo(B, H, T, d, 4242)
    scale = inputs.fp32_scale(d)
    compare(run_gpu(q, k, v, do, None, scale), q, k, v, do, None, scale, label="T4096")


def test_other_scale(cuda_device):
    """The scale is an argument: a non-default value must be honoured end to end."""
    B, H, T, d = 1, 2, 150, 64
    q, k, v, do = inputs.make_qkvdo(B, H, T, d, 31)
    compare(run_gpu(q, k, v, do, None, 0.3), q, k, v, do, None, 0.3, label="scale0.3")


# ------------------------------------------------------------- properties

def test_deterministic(cuda_device):
    w = inputs.WORKLOADS["gpt2_small"]
    q, k, v, do, doc = inputs.make_workload(w)
    a = run_gpu(q, k, v, do, doc, w.scale)
    b = run_gpu(q, k, v, do, doc, w.scale)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


# ---------------------------------------------------------- sliding window

@pytest.mark.parametrize("T,d,w", [
    (300, 64, 1), (300, 64, 64), (300, 128, 127), (333, 32, 128), (333, 64, 129),
    (513, 128, 200), (257, 64, 256), (700, 128, 384),
])
@pytest.mark.parametrize("with_doc", [False, True])
def test_sliding_window(T, d, w, with_doc, cuda_device):
    """Band of w keys (i - w < j <= i), alone and with document masks, every tile edge case."""
    B, H = 2, 2
    q, k, v, do = inputs.make_qkvdo(B, H, T, d, 61 + w)
    doc = inputs.random_doc_start(B, T, 11, 30, 200) if with_doc else None
    scale = inputs.fp32_scale(d)
    compare(run_gpu(q, k, v, do, doc, scale, window=w), q, k, v, do, doc, scale,
            label=f"window{w}_T{T}_d{d}_doc{int(with_doc)}", window=w)
    no_device_timeouts()


def test_window_at_least_t_is_plain_causal(cuda_device):
    """window >= T (and window <= 0) must give bit-for-bit the plain causal results."""
    B, H, T, d = 1, 3, 260, 128
    q, k, v, do = inputs.make_qkvdo(B, H, T, d, 71)
    scale = inputs.fp32_scale(d)
    base = run_gpu(q, k, v, do, None, scale)
    for w in (T, T + 5, 0, -3):
        for a, b in zip(run_gpu(q, k, v, do, None, scale, window=w), base):
            assert torch.equal(a, b), w


def test_window_full_size_workload(cuda_device):
    """wide_d128 with a 512-key window in the benchmark's launch configuration, every head
    (the windowed Jacobian costs O(T w^2) per head, so all 64 are cheap)."""
    w = inputs.WORKLOADS["wide_d128"]
    q, k, v, do, doc = inputs.make_workload(w)
    compare(run_gpu(q, k, v, do, doc, w.scale, window=512), q, k, v, do, doc, w.scale,
            None, label="wide_d128_window512", window=512)
    no_device_timeouts()


# ------------------------------------------------------------ KV-cache decode

def run_decode(q, kc, vc, scale):
    dev = torch.device("cuda:0")
    o, lse = abi.attention_decode(*(t.to(dev).contiguous() for t in (q, kc, vc)), scale)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def decode_inputs(B, H, Tq, L, d, seed):
    g = torch.Generator().manual_seed(seed)
    mk = lambda *shape: torch.randn(*shape, generator=g).to(torch.bfloat16)
    return mk(B, Tq, H, d), mk(B, L, H, d), mk(B, L, H, d)


@pytest.mark.parametrize("B,H,Tq,L,d", [
    (1, 1, 1, 1, 32), (2, 3, 1, 17, 64), (1, 4, 1, 128, 128), (2, 2, 1, 129, 128),
    (3, 2, 4, 300, 64), (1, 8, 16, 1000, 128), (2, 4, 3, 4096, 128), (1, 2, 16, 16, 32),
    (4, 16, 1, 2048, 128), (2, 3, 2, 77, 64), (1, 5, 8, 700, 32), (2, 2, 16, 129, 128),
    (1, 2, 2, 2, 128), (2, 4, 16, 16, 64),
])
def test_decode_parity(B, H, Tq, L, d, cuda_device):
    """gpt_attn_decode against the fp64 decode oracle: O max-abs <= 1e-2, LSE <= 1e-3."""
    q, kc, vc = decode_inputs(B, H, Tq, L, d, 900 + L + Tq)
    scale = inputs.fp32_scale(d)
    o, lse = run_decode(q, kc, vc, scale)
    o_r, lse_r = oracle.decode_forward(q, kc, vc, scale)
    err_o = float(np.max(np.abs(o.double().numpy() - o_r)))
    err_l = float(np.max(np.abs(lse.double().numpy() - lse_r)))
    print(f"decode B{B} H{H} Tq{Tq} L{L} d{d}: O {err_o:.3e} LSE {err_l:.3e}")
    assert err_o <= O_TOL and err_l <= LSE_TOL
    no_device_timeouts()


def test_decode_matches_training_forward_rows(cuda_device):
    """The decode of the last Tq tokens agrees with the training forward's last Tq rows."""
    B, H, T, d, Tq = 2, 4, 400, 128, 5
    q, k, v, _ = inputs.make_qkvdo(B, H, T, d, 17)
    scale = inputs.fp32_scale(d)
    o_full, lse_full = run_gpu(q, k, v, torch.zeros_like(q), None, scale)[:2]
    qd = q[:, :, T - Tq:].transpose(1, 2).contiguous()
    o, lse = run_decode(qd, k.transpose(1, 2).contiguous(), v.transpose(1, 2).contiguous(), scale)
    assert (o.transpose(1, 2).float() - o_full[:, :, T - Tq:].float()).abs().max() <= 1e-2
    assert (lse - lse_full[:, :, T - Tq:]).abs().max() <= 1e-3


def test_decode_deterministic(cuda_device):
    q, kc, vc = decode_inputs(2, 8, 2, 3000, 128, 5)
    a = run_decode(q, kc, vc, 0.088)
    b = run_decode(q, kc, vc, 0.088)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_host_stream_matches_device_path(cuda_device):
    """HostStream (pinned host buffers, neighbouring steps overlapped on three streams,
    two device buffer sets) gives, for every step of a sequence of different inputs,
    bit-for-bit the outputs of the device path, and the first step matches the oracle."""
    B, H, T, d = 2, 3, 333, 64
    scale = inputs.fp32_scale(d)
    doc = inputs.doc_start_from_lengths([[100, 233], [50, 283]], T)
    steps, expect = [], []
    for seed in (41, 42, 43, 44, 45):
        q, k, v, do = inputs.make_qkvdo(B, H, T, d, seed)
        expect.append(run_gpu(q, k, v, do, doc, scale))
        outs = {n: torch.empty(B, H, T, d, dtype=torch.bfloat16).pin_memory()
                for n in ("o", "dq", "dk", "dv")}
        outs["lse"] = torch.empty(B, H, T, dtype=torch.float32).pin_memory()
        steps.append(tuple(t.pin_memory() for t in (q, k, v, do)) + (outs,))
    hs = abi.HostStream(B, H, T, d)
    hs.set_doc_offsets(doc)
    hs.run(steps, scale).synchronize()
    for st, ex in zip(steps, expect):
        out = st[4]
        for name, ref in zip(("o", "lse", "dq", "dk", "dv"), ex):
            assert torch.equal(out[name], ref), name
    q, k, v, do = steps[0][:4]
    compare(expect[0], q, k, v, do, doc, scale, label="hoststream")


def test_uniform_values_on_gpu(cuda_device):
    """All value rows equal: every output row equals that row (up to its bf16 rounding)."""
    B, H, T, d = 1, 2, 300, 64
    q, k, _, do = inputs.make_qkvdo(B, H, T, d, 5)
    u = torch.randn(d, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    v = u.expand(B, H, T, d).contiguous()
    o, lse, dq, dk, dv = run_gpu(q, k, v, do, None, inputs.fp32_scale(d))
    exact = torch.eq(o, v).double().mean().item()
    print(f"uniform V: {exact:.4%} of O elements bit-equal to V")
    assert (o.float() - v.float()).abs().max() <= O_TOL
    assert dq.abs().max() < 2e-2 and dk.abs().max() < 2e-2


def test_autograd_wrapper(cuda_device):
    B, H, T, d = 1, 2, 96, 32
    q, k, v, do = inputs.make_qkvdo(B, H, T, d, 9)
    dev = torch.device("cuda:0")
    tq, tk, tv = (t.to(dev).requires_grad_(True) for t in (q, k, v))
    o = abi.causal_attention(tq, tk, tv)
    o.backward(do.to(dev))
    gpu = [o.detach().cpu(), torch.zeros(B, H, T), tq.grad.cpu(), tk.grad.cpu(), tv.grad.cpu()]
    o_r, _ = oracle.attention_forward(q, k, v, inputs.fp32_scale(d))
    assert np.max(np.abs(gpu[0].double().numpy() - o_r)) <= O_TOL
    g = oracle.attention_backward(q, k, v, do, inputs.fp32_scale(d))
    for a, r in zip(gpu[2:], g):
        assert rel_l2(a.double().numpy(), r) <= GRAD_TOL


# ------------------------------------------------------- errors and faults

def test_doc_offsets_validator(cuda_device):
    dev = torch.device("cuda:0")
    good = inputs.random_doc_start(3, 500, 2, 10, 90).to(dev)
    assert abi.gpt_attn_check_doc_offsets(good)
    bad = good.clone()
    bad[1, 37] = 40  # points past its own position
    assert not abi.gpt_attn_check_doc_offsets(bad)
    bad = good.clone()
    bad[2, 0] = 1
    assert not abi.gpt_attn_check_doc_offsets(bad)


def test_bounded_wait_reports_timeout_and_context_survives(cuda_device):
    """A wait on a barrier nobody signals gives up after its limit, reports through the status
    word, and leaves the CUDA context usable."""
    assert abi.gpt_attn_selftest_wait_timeout(2_000_000) == abi.GPT_ATTN_ERR_DEVICE_TIMEOUT
    assert abi.gpt_attn_device_status() == 0
    B, H, T, d = 1, 1, 130, 64
    q, k, v, do = inputs.make_qkvdo(B, H, T, d, 77)
    compare(run_gpu(q, k, v, do, None, 0.125), q, k, v, do, None, 0.125, label="after-timeout")


def test_gpu_argument_errors(cuda_device):
    q = torch.zeros(1, 1, 64, 48, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 1, 64, device="cuda")
    with pytest.raises(abi.AttnError) as e:
        abi.gpt_attn_fwd(q, q, q, q, lse, 0.1)
    assert e.value.status == abi.GPT_ATTN_ERR_UNSUPPORTED_HEAD_DIM
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(abi.AttnError) as e:
        abi.gpt_attn_fwd(q, q, q, q, lse, float("nan"))
    assert e.value.status == abi.GPT_ATTN_ERR_BAD_SCALE


# ------------------------------------------------------- RoPE + QK-norm prologue
# bf16 in, fp32 arithmetic, bf16 out: each output element is within bf16 rounding of the
# fp64 oracle (rtol 2^-8, half an ulp at the bottom of a binade) plus a small absolute term
# for the fp32 arithmetic and the angle (fp64 reduction, then __sincosf on [-pi, pi]).
PRO_RTOL, PRO_ATOL = 2.0 ** -8, 2e-3


def run_prologue(q, k, dq_out, dk_out, base=10000.0, gain=1.2, eps=1e-6, in_place=False):
    dev = torch.device("cuda:0")
    q, k, dq_out, dk_out = (t.to(dev).contiguous() for t in (q, k, dq_out, dk_out))
    if in_place:
        qo, ko = q.clone(), k.clone()
        abi.gpt_attn_rope_qknorm_fwd(qo, ko, qo, ko, base, gain, eps)
        dq, dk = dq_out.clone(), dk_out.clone()
        abi.gpt_attn_rope_qknorm_bwd(q, k, dq, dk, dq, dk, base, gain, eps)
    else:
        qo, ko = abi.rope_qknorm(q, k, base, gain, eps)
        dq, dk = torch.empty_like(q), torch.empty_like(k)
        abi.gpt_attn_rope_qknorm_bwd(q, k, dq_out, dk_out, dq, dk, base, gain, eps)
    torch.cuda.synchronize()
    return [t.cpu().double().numpy() for t in (qo, ko, dq, dk)]


def check_prologue(got, q, k, dq_out, dk_out, base=10000.0, gain=1.2, eps=1e-6, label=""):
    refs = (oracle.qk_prologue_forward(q, base, gain, eps),
            oracle.qk_prologue_forward(k, base, gain, eps),
            oracle.qk_prologue_backward(q, dq_out, base, gain, eps),
            oracle.qk_prologue_backward(k, dk_out, base, gain, eps))
    for name, g, r in zip(("q'", "k'", "dq", "dk"), got, refs):
        err = np.abs(g - r) - PRO_RTOL * np.abs(r)
        print(f"prologue {label} {name}: max excess {float(err.max()):.2e}")
        assert float(err.max()) <= PRO_ATOL, (name, float(err.max()))


@pytest.mark.parametrize("B,H,T,d", [(1, 1, 1, 32), (2, 3, 37, 32), (1, 5, 130, 64),
                                     (2, 4, 257, 128), (1, 16, 1000, 128), (3, 7, 65, 64),
                                     (1, 1, 40000, 64)])
def test_prologue_parity(B, H, T, d, cuda_device):
    """Every output element of the prologue forward and backward against the fp64 oracle;
    H not a multiple of the 4 heads a thread handles, ragged T, and positions up to 40000
    (the angle reduction)."""
    x = inputs.make_prologue(B, H, T, d, 700 + T + d)
    check_prologue(run_prologue(*x), *x, label=f"B{B} H{H} T{T} d{d}")
    no_device_timeouts()


@pytest.mark.parametrize("base,gain,eps", [(500000.0, 1.0, 1e-5), (10.0, -0.7, 0.0)])
def test_prologue_parameters(base, gain, eps, cuda_device):
    x = inputs.make_prologue(2, 3, 300, 128, 77)
    check_prologue(run_prologue(*x, base=base, gain=gain, eps=eps), *x, base=base, gain=gain,
                   eps=eps, label=f"base {base} gain {gain} eps {eps}")


def test_prologue_in_place_matches_out_of_place(cuda_device):
    x = inputs.make_prologue(2, 6, 201, 64, 78)
    a = run_prologue(*x)
    b = run_prologue(*x, in_place=True)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_prologue_full_size_workload(cuda_device):
    """The benchmark's prologue launch (B=4, H=16, T=2048, d=128), every element."""
    c = inputs.PROLOGUE_WORKLOADS["prologue_wide_d128"]
    x = inputs.make_prologue(c["B"], c["H"], c["T"], c["d"], c["seed"])
    check_prologue(run_prologue(*x), *x, label="prologue_wide_d128")
    no_device_timeouts()


def test_prologue_autograd_then_attention(cuda_device):
    """rope_qk_norm then causal_attention under torch.autograd: the gradients with respect to
    the raw q, k, v match the oracle chain (prologue forward, attention forward and
    backward, prologue backward) on one head."""
    B, H, T, d = 1, 2, 150, 64
    q, k, v, do = inputs.make_qkvdo(B, H, T, d, 79)
    scale = inputs.fp32_scale(d)
    dev = torch.device("cuda:0")
    qd, kd, vd = (t.to(dev).requires_grad_() for t in (q, k, v))
    qn, kn = abi.rope_qk_norm(qd, kd)
    o = abi.causal_attention(qn, kn, vd, scale)
    o.backward(do.to(dev))
    torch.cuda.synchronize()
    qn_r = oracle.qk_prologue_forward(q)
    kn_r = oracle.qk_prologue_forward(k)
    # the oracle attention takes the GPU's bf16 prologue outputs, as the kernels did
    qn_b, kn_b = (t.detach().cpu() for t in (qn, kn))
    for a, r in ((qn_b, qn_r), (kn_b, kn_r)):
        assert float((np.abs(a.double().numpy() - r) - PRO_RTOL * np.abs(r)).max()) <= PRO_ATOL
    o_r, _ = oracle.attention_forward(qn_b, kn_b, v, scale)
    dqn, dkn, dv_r = oracle.attention_backward(qn_b, kn_b, v, do, scale)
    dq_r = oracle.qk_prologue_backward(q, dqn)
    dk_r = oracle.qk_prologue_backward(k, dkn)
    assert float(np.max(np.abs(o.detach().cpu().double().numpy() - o_r))) <= O_TOL
    for g, r in ((qd.grad, dq_r), (kd.grad, dk_r), (vd.grad, dv_r)):
        assert rel_l2(g.cpu().double().numpy(), r) <= GRAD_TOL


# ----------------------------------------------- dQ with delta fused into it

@pytest.mark.parametrize("T,d,with_doc", [(1, 32, False), (200, 64, True), (300, 128, False),
                                          (1024, 128, True)])
def test_dq_step_computes_delta(T, d, with_doc, cuda_device):
    """gpt_attn_bwd_dq_delta writes delta = rowsum(dO * O) (checked in fp64 from the same bf16
    O and dO) and gives the dQ of gpt_attn_bwd_preprocess + gpt_attn_bwd_dq up to the order of
    the fp32 additions in delta."""
    B, H = 2, 3
    q, k, v, do = (t.to(cuda_device) for t in inputs.make_qkvdo(B, H, T, d, 800 + T + d))
    doc = inputs.random_doc_start(B, T, 9 + T, 20, 200).to(cuda_device) if with_doc else None
    scale = inputs.fp32_scale(d)
    o, lse = abi.attention_forward(q, k, v, scale, doc)
    delta_f = torch.full((B, H, T), float("nan"), device=cuda_device)
    dq_f = torch.empty_like(q)
    abi.gpt_attn_bwd_dq_delta(q, k, v, o, do, lse, delta_f, dq_f, scale, doc)
    delta_s = torch.empty_like(delta_f)
    dq_s = torch.empty_like(q)
    abi.gpt_attn_bwd_preprocess(o, do, delta_s)
    abi.gpt_attn_bwd_dq(q, k, v, do, lse, delta_s, dq_s, scale, doc)
    torch.cuda.synchronize()
    ref = (o.double() * do.double()).sum(-1)
    mag = (o.double() * do.double()).abs().sum(-1)
    assert torch.all((delta_f.double() - ref).abs() <= 1e-6 * mag + 1e-6)
    assert rel_l2(dq_f.double().cpu().numpy(), dq_s.double().cpu().numpy()) <= 1e-3
    no_device_timeouts()


def test_prepared_calls_match_direct_calls(cuda_device):
    """abi.prepare: the checked-once call re-issued gives bit-identical results."""
    B, H, T, d = 2, 3, 333, 64
    q, k, v, do = (t.to(cuda_device) for t in inputs.make_qkvdo(B, H, T, d, 901))
    scale = inputs.fp32_scale(d)
    o, lse = abi.attention_forward(q, k, v, scale)
    o2, lse2 = torch.empty_like(o), torch.empty_like(lse)
    fwd = abi.prepare(abi.gpt_attn_fwd, q, k, v, o2, lse2, scale)
    dq, dk, dv = abi.attention_backward(q, k, v, o, lse, do, scale)
    dq2, dk2, dv2 = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    delta = torch.empty_like(lse)
    bwd = abi.prepare(abi.gpt_attn_bwd, q, k, v, o, do, lse, dq2, dk2, dv2, delta, scale)
    for _ in range(2):
        fwd()
        bwd()
        torch.cuda.synchronize()
        assert torch.equal(o2, o) and torch.equal(lse2, lse)
        assert torch.equal(dq2, dq) and torch.equal(dk2, dk) and torch.equal(dv2, dv)
    no_device_timeouts()


def test_calls_from_another_host_thread(cuda_device):
    """Library calls from a second host thread (as torch's autograd engine makes them) give the
    results of the same calls from the main thread, bit for bit."""
    import threading
    B, H, T, d = 1, 2, 200, 64
    q, k, v, do = (t.to(cuda_device) for t in inputs.make_qkvdo(B, H, T, d, 902))
    scale = inputs.fp32_scale(d)
    o, lse = abi.attention_forward(q, k, v, scale)
    ref = abi.attention_backward(q, k, v, o, lse, do, scale)
    torch.cuda.synchronize()
    out, err = {}, []

    def work():
        try:
            torch.cuda.set_device(cuda_device)
            o2, lse2 = abi.attention_forward(q, k, v, scale)
            out["g"] = abi.attention_backward(q, k, v, o2, lse2, do, scale)
            out["f"] = (o2, lse2)
            torch.cuda.synchronize()
        except Exception as e:  # reported on the main thread
            err.append(e)
    th = threading.Thread(target=work)
    th.start()
    th.join()
    assert not err, err
    assert torch.equal(out["f"][0], o) and torch.equal(out["f"][1], lse)
    for a, b in zip(out["g"], ref):
        assert torch.equal(a, b)
