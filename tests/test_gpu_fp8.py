"""GPU parity of the FP8 (e4m3) attention forward against the oracle, through the C ABI.

The oracle (oracle.fp8_attention_forward / fp8_attention_simulated) gives, from the same e4m3
codes: the exact attention o, lse of the dequantised inputs; a rigorous per-element bound on
what rounding the weights to e4m3 can change; and the rounded-weight forward evaluated in fp64
(weights relative to the row's final maximum, as the kernel rounds them).  Tolerances:
  LSE   max |gpu - lse|                          <= 1e-3  (the scores are exact products of
        e4m3 values, accumulated in fp32)
  O     every element: |gpu - o| <= bound * (1 + 2^-8) + 2^-8 |o| + 1e-3
        (bound, then bf16 rounding of the output, then fp32 accumulation)
  O     ||gpu - sim||_2 <= 0.25 ||sim - o||_2 + 2^-8 ||o||_2: the kernel rounds at the same
        points as the simulation, so the two may differ only where the fp32 exponential lands
        on the other side of an e4m3 rounding tie (a full ulp for about one weight in 2^12,
        ~0.05 of the rounding noise) and by the bf16 rounding of the output.
"""
import numpy as np
import pytest
import torch

import oracle
from causal_self_attention_mha_b200 import abi, inputs

pytestmark = pytest.mark.gpu

DS = inputs.FP8_DESCALE


def run_fp8(q8, k8, v8, doc, scale, ds=(DS, DS, DS)):
    dev = torch.device("cuda:0")
    q8, k8, v8 = (t.to(dev).contiguous() for t in (q8, k8, v8))
    docd = doc.to(dev).contiguous() if doc is not None else None
    o, lse = abi.attention_forward_fp8(q8, k8, v8, *ds, scale, docd)
    torch.cuda.synchronize()
    return o.cpu().to(torch.float64).numpy(), lse.cpu().to(torch.float64).numpy()


def oracle_fp8(q8, k8, v8, doc, scale):
    """(o, lse, bound, sim) of the oracle for [B,H,T,d] codes."""
    o, lse, bound = oracle.fp8_attention_forward(q8, k8, v8, DS, DS, DS, scale, doc)
    sim = oracle.fp8_attention_simulated(q8, k8, v8, DS, DS, DS, scale, doc)
    return o, lse, bound, sim


def check(q8, k8, v8, doc, scale, label, heads=None):
    """heads: None for every head, else a list of (b, h) to compare (full-size workloads)."""
    o_g, lse_g = run_fp8(q8, k8, v8, doc, scale)
    if heads is None:
        o, lse, bound, sim = oracle_fp8(q8, k8, v8, doc, scale)
    else:  # one oracle call per picked head, with its own batch row's documents
        parts = [oracle_fp8(q8[b:b + 1, h:h + 1], k8[b:b + 1, h:h + 1], v8[b:b + 1, h:h + 1],
                            doc[b:b + 1] if doc is not None else None, scale) for b, h in heads]
        o, lse, bound, sim = (np.concatenate([pt[j] for pt in parts], axis=1) for j in range(4))
        o_g = np.stack([o_g[b, h] for b, h in heads])[None]
        lse_g = np.stack([lse_g[b, h] for b, h in heads])[None]
    assert np.all(np.isfinite(o_g)) and np.all(np.isfinite(lse_g)), label
    err_l = float(np.max(np.abs(lse_g - lse)))
    lim = bound * (1 + 2.0 ** -8) + 2.0 ** -8 * np.abs(o) + 1e-3
    over = float(np.max(np.abs(o_g - o) - lim))
    agg = float(np.linalg.norm(o_g - sim))
    agg_lim = 0.25 * float(np.linalg.norm(sim - o)) + 2.0 ** -8 * float(np.linalg.norm(o))
    print(f"{label}: LSE maxabs {err_l:.2e}  O max over bound {over:.2e}  "
          f"||gpu-sim|| {agg:.3e} (limit {agg_lim:.3e}, ||sim-o|| {np.linalg.norm(sim - o):.3e})")
    assert err_l <= 1e-3, (label, "LSE", err_l)
    assert over <= 0, (label, "O outside the bound", over)
    assert agg <= agg_lim, (label, "O far from the rounded-weight forward", agg, agg_lim)


def test_single_token_and_tiny(cuda_device):
    for T, d in ((1, 32), (1, 128), (5, 64)):
        q8, k8, v8 = inputs.make_qkv_e4m3(1, 2, T, d, 300 + T + d)
        check(q8, k8, v8, None, inputs.fp32_scale(d), f"T{T} d{d}")


@pytest.mark.parametrize("T", [17, 64, 127, 128, 129, 255, 300])
@pytest.mark.parametrize("d", [32, 64, 128])
def test_ragged_lengths(T, d, cuda_device):
    q8, k8, v8 = inputs.make_qkv_e4m3(1, 3, T, d, 400 + T + d)
    check(q8, k8, v8, None, inputs.fp32_scale(d), f"T{T} d{d}")


@pytest.mark.parametrize("d", [32, 64, 128])
def test_document_mask(d, cuda_device):
    B, H, T = 2, 2, 389
    q8, k8, v8 = inputs.make_qkv_e4m3(B, H, T, d, 500 + d)
    doc = inputs.random_doc_start(B, T, 77 + d, 5, 150)
    check(q8, k8, v8, doc, inputs.fp32_scale(d), f"doc d{d}")


def test_uniform_values_exact(cuda_device):
    """Every key carries one value row u: the normalised weighted sum is u itself."""
    B, H, T, d = 1, 2, 260, 128
    q8, k8, v8 = inputs.make_qkv_e4m3(B, H, T, d, 600)
    v8[:] = v8[:, :, :1, :]
    o_g, _ = run_fp8(q8, k8, v8, None, inputs.fp32_scale(d))
    u = oracle.fp8_dequantize(v8[:, :, :1, :], DS)
    assert np.max(np.abs(o_g - u) - 2.0 ** -8 * np.abs(u)) <= 1e-6


def test_descales_are_applied(cuda_device):
    """Doubling descale_v doubles O; doubling descale_q and halving descale_k changes nothing."""
    B, H, T, d = 1, 2, 200, 64
    q8, k8, v8 = inputs.make_qkv_e4m3(B, H, T, d, 700)
    s = inputs.fp32_scale(d)
    o1, l1 = run_fp8(q8, k8, v8, None, s)
    o2, l2 = run_fp8(q8, k8, v8, None, s, (DS, DS, 2 * DS))
    o3, l3 = run_fp8(q8, k8, v8, None, s, (2 * DS, DS / 2, DS))
    assert np.array_equal(o2, 2 * o1) and np.array_equal(l2, l1)
    assert np.array_equal(o3, o1) and np.array_equal(l3, l1)


@pytest.mark.parametrize("name", list(inputs.WORKLOADS))
def test_workloads(name, cuda_device):
    """The five workloads' shapes (and document layout) in the launch configuration the
    benchmark times; T = 2048 workloads compare 12 heads spread over the batch (the oracle's
    per-head probability matrix is T x T)."""
    w = inputs.WORKLOADS[name]
    q8, k8, v8, doc = inputs.make_fp8_workload(w)
    heads = None
    if w.T >= 2048:
        idx = np.linspace(0, w.B * w.H - 1, 12).round().astype(int)
        heads = [(int(i) // w.H, int(i) % w.H) for i in idx]
    check(q8, k8, v8, doc, w.scale, name, heads)
    assert abi.gpt_attn_device_status(clear=True) == 0
