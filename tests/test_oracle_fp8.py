"""Pins of the FP8 (e4m3) attention-forward oracle (CPU only).

The reading ("How to build an LLM by hand", agmtopy.github.io, section 5, item 4: forward
matmuls with e4m3 operands through torch._scaled_mm, fixed per-tensor scales): Q, K, V are
e4m3 codes with one descale factor each; the attention weights, taken relative to the row
maximum and multiplied by 2^8, are rounded to e4m3 before the weighted sum, which is
normalised by the sum of the rounded weights.  Pinned here:
  * the e4m3 codec against torch's float8_e4m3fn conversion (an independent implementation)
    and the OCP format's fixed points;
  * the quantised-weight forward against closed forms (T = 1, uniform V, weights that are
    exact powers of two so that rounding changes nothing), and against the same forward
    written with torch's e4m3 rounding on tiny inputs;
  * the per-element error bound: it holds for the worst perturbation inside its box and for
    the rounded forward, it is zero where nothing can move, and planted mistakes break it.
"""
import math

import numpy as np
import pytest
import torch

import oracle

S = 1.0 / 32  # descale of the test tensors: stored values are 32 x N(0,1)


def e4m3_inputs(B, H, T, d, seed, mult=32.0):
    g = torch.Generator().manual_seed(seed)
    mk = lambda: (torch.randn(B, H, T, d, generator=g) * mult).to(torch.float8_e4m3fn).view(torch.uint8)
    return mk(), mk(), mk()


# ------------------------------------------------------------------ codec

def test_decode_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = oracle.e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.isnan(got).sum() == 2  # S.1111.111 only


def test_encode_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(0)
    vals = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2  # every tie between neighbours (exact in fp32)
    x = np.concatenate([rng.uniform(-464, 464, 200000), rng.normal(0, 0.01, 50000), vals, -vals,
                        mids, -mids, rng.normal(0, 2.0 ** -8, 20000)])
    x = x.astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(x).float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(x), ref)


def test_format_fixed_points_and_saturation():
    assert oracle.e4m3_encode(448.0) == 0x7E and oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_encode(1.0) == 0x38
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9 and oracle.e4m3_decode(0x08) == 2.0 ** -6
    for big in (449.0, 500.0, 1e6, math.inf):  # saturating rounding, unlike a plain cast
        assert oracle.e4m3_encode(big) == 0x7E and oracle.e4m3_encode(-big) == 0xFE
    assert oracle.e4m3_encode(math.nan) == 0x7F
    assert oracle.e4m3_encode(-0.0) == 0x80 and oracle.e4m3_encode(2.0 ** -11) == 0x00


def test_dequantize_is_exact():
    q8, _, _ = e4m3_inputs(1, 2, 16, 8, 3)
    ref = q8.view(torch.float8_e4m3fn).double().numpy() * S
    assert np.array_equal(oracle.fp8_dequantize(q8, S), ref)


# ------------------------------------------------------- quantised forward

def test_single_token_returns_v():
    q8, k8, v8 = e4m3_inputs(1, 2, 1, 16, 4)
    o_sim = oracle.fp8_attention_simulated(q8, k8, v8, S, S, S, 0.25)
    o, lse, bound = oracle.fp8_attention_forward(q8, k8, v8, S, S, S, 0.25)
    v = oracle.fp8_dequantize(v8, S)
    assert np.array_equal(o_sim, v) and np.array_equal(bound, np.zeros_like(bound))
    qd, kd = oracle.fp8_dequantize(q8, S), oracle.fp8_dequantize(k8, S)
    assert np.allclose(lse[..., 0], 0.25 * np.sum(qd * kd, axis=-1)[..., 0], rtol=0, atol=1e-12)


def test_uniform_v_is_reproduced_exactly():
    q8, k8, v8 = e4m3_inputs(1, 2, 40, 8, 5)
    v8[:] = v8[:, :, :1, :]  # every key carries the same value row
    o_sim = oracle.fp8_attention_simulated(q8, k8, v8, S, S, S, 0.3)
    _, _, bound = oracle.fp8_attention_forward(q8, k8, v8, S, S, S, 0.3)
    v = oracle.fp8_dequantize(v8, S)
    assert np.allclose(o_sim, np.broadcast_to(v[:, :, :1, :], o_sim.shape), rtol=0, atol=1e-12)
    assert np.max(bound) < 1e-12


def test_power_of_two_weights_are_not_changed_by_rounding():
    """Scores ln(2) * integer make every weight relative to the row maximum a power of two
    (>= 2^-14, so 2^8 times it is a normal e4m3 number): rounding is exact and the quantised
    forward equals the exact attention."""
    T, d = 24, 1
    rng = np.random.default_rng(6)
    q8 = oracle.e4m3_encode(np.ones((1, 1, T, d)))
    k8 = oracle.e4m3_encode(rng.integers(0, 14, (1, 1, T, d)).astype(np.float64))
    v8, _, _ = e4m3_inputs(1, 1, T, d, 7)
    o_sim = oracle.fp8_attention_simulated(q8, k8, v8, 1.0, 1.0, S, math.log(2.0))
    o, _, _ = oracle.fp8_attention_forward(q8, k8, v8, 1.0, 1.0, S, math.log(2.0))
    assert np.max(np.abs(o_sim - o)) < 1e-13


def test_quantised_forward_matches_torch_rounding():
    """The same forward with the weights rounded by torch's float8_e4m3fn cast."""
    B, H, T, d = 1, 2, 33, 8
    q8, k8, v8 = e4m3_inputs(B, H, T, d, 8)
    scale = d ** -0.5
    q, k, v = (oracle.fp8_dequantize(x, S) for x in (q8, k8, v8))
    ref = np.empty_like(q)
    for h in range(H):
        s = scale * (q[0, h] @ k[0, h].T)
        s[np.triu_indices(T, 1)] = -np.inf
        r = np.exp(s - s.max(axis=1, keepdims=True))
        qw = torch.from_numpy(256.0 * r).float().to(torch.float8_e4m3fn).double().numpy() / 256.0
        ref[0, h] = (qw @ v[0, h]) / qw.sum(axis=1, keepdims=True)
    got = oracle.fp8_attention_simulated(q8, k8, v8, S, S, S, scale)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_documents_and_window_reduce_to_slices():
    """The document mask of the quantised forward equals the forward of each document alone."""
    B, H, T, d = 1, 1, 30, 4
    q8, k8, v8 = e4m3_inputs(B, H, T, d, 9)
    doc = np.zeros((1, T), np.int32)
    doc[0, 12:] = 12
    got = oracle.fp8_attention_simulated(q8, k8, v8, S, S, S, 0.5, doc)
    a = oracle.fp8_attention_simulated(q8[:, :, :12], k8[:, :, :12], v8[:, :, :12], S, S, S, 0.5)
    b = oracle.fp8_attention_simulated(q8[:, :, 12:], k8[:, :, 12:], v8[:, :, 12:], S, S, S, 0.5)
    assert np.array_equal(got[:, :, :12], a) and np.array_equal(got[:, :, 12:], b)


# ---------------------------------------------------------------- the bound

def _rows(q8, k8, v8, scale):
    q, k, v = (oracle.fp8_dequantize(x, S) for x in (q8, k8, v8))
    o, _, p = oracle.attention_forward(q, k, v, scale, return_probs=True)
    return o, p, v


@pytest.mark.parametrize("seed", [10, 11, 12])
def test_bound_holds_for_the_worst_perturbation(seed):
    """For each output column the error is largest when every weight moves by its full bound
    in the direction of sign(v_jc - o_c); the bound must cover that, and random moves."""
    B, H, T, d = 1, 1, 48, 6
    q8, k8, v8 = e4m3_inputs(B, H, T, d, seed)
    scale = 0.4
    o, _, bound = oracle.fp8_attention_forward(q8, k8, v8, S, S, S, scale)
    o2, p, v = _rows(q8, k8, v8, scale)
    assert np.max(np.abs(o - o2)) == 0
    rng = np.random.default_rng(seed)
    for i in range(T):
        r = p[0, 0, i, :i + 1] / p[0, 0, i, :i + 1].max()
        e = oracle.fp8_weight_error_bound(r)
        for c in range(d):
            dev = v[0, 0, :i + 1, c] - o[0, 0, i, c]
            for qw in (r + e * np.sign(dev), r - e * np.sign(dev),
                       r + e * rng.uniform(-1, 1, r.shape)):
                err = abs(qw @ v[0, 0, :i + 1, c] / qw.sum() - o[0, 0, i, c])
                assert err <= bound[0, 0, i, c] * (1 + 1e-12) + 1e-15, (i, c)


def test_rounded_forward_within_bound_and_bound_not_vacuous():
    B, H, T, d = 1, 2, 300, 32
    q8, k8, v8 = e4m3_inputs(B, H, T, d, 13)
    o, _, bound = oracle.fp8_attention_forward(q8, k8, v8, S, S, S, d ** -0.5)
    sim = oracle.fp8_attention_simulated(q8, k8, v8, S, S, S, d ** -0.5)
    err = np.abs(sim - o)
    assert np.all(err <= bound * (1 + 1e-12) + 1e-15)
    assert np.median(err) > 0  # rounding does move the result ...
    assert np.median(err) < 0.2 * np.median(bound)  # ... well inside the worst case


def test_planted_mistakes_break_the_bound():
    """Mistakes a quantised forward could make, each caught against the bound."""
    B, H, T, d = 1, 1, 200, 16
    q8, k8, v8 = e4m3_inputs(B, H, T, d, 14)
    v8 = oracle.e4m3_encode(oracle.e4m3_decode(v8) + 300.0)  # a large common offset in V
    scale = d ** -0.5
    o, _, bound = oracle.fp8_attention_forward(q8, k8, v8, S, S, S, scale)
    q, k, v = (oracle.fp8_dequantize(x, S) for x in (q8, k8, v8))
    _, _, p = oracle.attention_forward(q, k, v, scale, return_probs=True)
    r = p[0, 0] / p[0, 0].max(axis=1, keepdims=True)
    qw = oracle.e4m3_round(256.0 * r) / 256.0
    lim = bound[0, 0] * (1 + 2.0 ** -8) + 2.0 ** -8 * np.abs(o[0, 0]) + 1e-3
    wrong = {
        # normalised by the exact weights' sum instead of the rounded weights'
        "exact-sum normalisation": (qw @ v[0, 0]) / r.sum(axis=1, keepdims=True),
        # V's descale factor applied twice
        "descale twice": (qw @ (v[0, 0] * S)) / qw.sum(axis=1, keepdims=True),
        # the diagonal key dropped
        "diagonal dropped": ((qw - np.diag(np.diag(qw))) @ v[0, 0])
        / np.maximum((qw - np.diag(np.diag(qw))).sum(axis=1, keepdims=True), 1e-300),
    }
    for name, ow in wrong.items():
        assert np.any(np.abs(ow - o[0, 0]) > lim), name
