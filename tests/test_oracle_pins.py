"""Pins for the CPU fp64 oracle: checks against facts that do not come from the
oracle itself -- closed forms derived by hand, invariants of the definition,
central finite differences, and an independent library routine (torch's CPU
scaled_dot_product_attention in float64 with autograd).

The definition being pinned: "Stanford CS336 walkthrough" (lmnt.cn), section
5.1 model.py CausalSelfAttention.forward (scores q k^T / sqrt(d), upper
triangle -inf, row softmax, att @ v) and section 3.3 (masked weights are zero
after the softmax); the mask keeps the diagonal (torch.tril(ones) in
"Train Your Own LLM from Scratch", section 1).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from causal_self_attention_mha_b200 import inputs


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def fwd(q, k, v, scale, doc=None, probs=False):
    return oracle.attention_forward(q, k, v, scale, doc, return_probs=probs)


def bwd(q, k, v, do, scale, doc=None):
    return oracle.attention_backward(q, k, v, do, scale, doc)


# ---------------------------------------------------------------- closed forms

def test_single_token_closed_form():
    """T = 1: softmax over one key is 1, so O = v_0, LSE = scale <q0,k0>, dQ = dK = 0, dV = dO."""
    B, H, T, d = 2, 3, 1, 8
    q, k, v, do = (rnd((B, H, T, d), s) for s in range(4))
    scale = 0.37
    o, lse = fwd(q, k, v, scale)
    np.testing.assert_array_equal(o, v)
    np.testing.assert_allclose(lse, scale * np.einsum("bhtc,bhtc->bht", q, k), rtol=0, atol=1e-14)
    dq, dk, dv = bwd(q, k, v, do, scale)
    assert np.all(dq == 0) and np.all(dk == 0)
    np.testing.assert_array_equal(dv, do)


def test_first_row_sees_only_itself():
    """Row 0 has a single visible key (the diagonal): O_0 = v_0 and LSE_0 = scale <q0,k0>."""
    B, H, T, d = 1, 2, 9, 4
    q, k, v = (rnd((B, H, T, d), s) for s in range(3))
    o, lse = fwd(q, k, v, 0.5)
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], 0.5 * np.sum(q[:, :, 0] * k[:, :, 0], -1), atol=1e-14)


def test_two_token_closed_form():
    """T = 2 by hand.  Row 1 mixes v0, v1 with p11 = sigmoid(scale <q1, k1 - k0>):
         O_1   = v0 + p11 (v1 - v0),  LSE_1 = log(e^{s10} + e^{s11})
         g     = p10 p11 <dO_1, v1 - v0>
         dQ_1  = scale g (k1 - k0),   dQ_0 = 0
         dK_0  = -scale g q1,         dK_1 = +scale g q1
         dV_0  = dO_0 + p10 dO_1,     dV_1 = p11 dO_1
    """
    d, scale = 5, 0.8
    q, k, v, do = (rnd((1, 1, 2, d), 10 + s) for s in range(4))
    q0, q1 = q[0, 0]
    k0, k1 = k[0, 0]
    v0, v1 = v[0, 0]
    do0, do1 = do[0, 0]
    s10, s11 = scale * q1 @ k0, scale * q1 @ k1
    p11 = 1.0 / (1.0 + math.exp(-(s11 - s10)))
    p10 = 1.0 - p11
    o, lse = fwd(q, k, v, scale)
    np.testing.assert_allclose(o[0, 0, 1], v0 + p11 * (v1 - v0), atol=1e-14)
    np.testing.assert_allclose(lse[0, 0, 1], math.log(math.exp(s10) + math.exp(s11)), atol=1e-14)
    g = p10 * p11 * (do1 @ (v1 - v0))
    dq, dk, dv = bwd(q, k, v, do, scale)
    np.testing.assert_allclose(dq[0, 0, 0], 0.0, atol=1e-15)
    np.testing.assert_allclose(dq[0, 0, 1], scale * g * (k1 - k0), atol=1e-14)
    np.testing.assert_allclose(dk[0, 0, 0], -scale * g * q1, atol=1e-14)
    np.testing.assert_allclose(dk[0, 0, 1], scale * g * q1, atol=1e-14)
    np.testing.assert_allclose(dv[0, 0, 0], do0 + p10 * do1, atol=1e-14)
    np.testing.assert_allclose(dv[0, 0, 1], p11 * do1, atol=1e-14)


def test_uniform_values_give_that_value():
    """All v_j equal to u: every row is a convex combination of copies of u, so O_i = u;
    dP_ij = <dO_i, u> is constant along the row, so dS = 0 and dQ = dK = 0."""
    B, H, T, d = 2, 2, 33, 6
    q, k, do = (rnd((B, H, T, d), s) for s in range(3))
    u = rnd((d,), 7)
    v = np.broadcast_to(u, (B, H, T, d)).copy()
    o, _ = fwd(q, k, v, 0.4)
    np.testing.assert_allclose(o, v, atol=1e-13)
    dq, dk, dv = bwd(q, k, v, do, 0.4)
    np.testing.assert_allclose(dq, 0.0, atol=1e-13)
    np.testing.assert_allclose(dk, 0.0, atol=1e-13)


# ------------------------------------------------------------------ invariants

def test_probability_rows():
    """Rows of P sum to 1, the strict upper triangle is exactly 0, the diagonal is positive."""
    B, H, T, d = 2, 2, 40, 8
    q, k, v = (rnd((B, H, T, d), s) for s in range(3))
    _, _, p = fwd(q, k, v, 1 / math.sqrt(d), probs=True)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-12)
    iu = np.triu_indices(T, 1)
    assert np.all(p[:, :, iu[0], iu[1]] == 0.0)
    assert np.all(np.diagonal(p, axis1=2, axis2=3) > 0)


def test_probability_rows_with_documents():
    """With a document mask, P_ij = 0 outside [doc_start(i), i] and rows still sum to 1."""
    B, H, T, d = 2, 1, 50, 4
    q, k, v = (rnd((B, H, T, d), s) for s in range(3))
    doc = inputs.random_doc_start(B, T, 3, 3, 17).numpy()
    _, _, p = fwd(q, k, v, 0.6, doc, probs=True)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-12)
    for b in range(B):
        for i in range(T):
            outside = np.ones(T, bool)
            outside[doc[b, i]:i + 1] = False
            assert np.all(p[b, :, i, outside] == 0.0)


@pytest.mark.parametrize("t", [0, 5, 17])
def test_future_perturbation_leaves_past_unchanged(t):
    """Changing q, k, v at positions > t leaves O, LSE at positions <= t bit-identical;
    with dO = 0 after t, the gradients at positions <= t are bit-identical too."""
    B, H, T, d = 1, 2, 24, 4
    q, k, v, do = (rnd((B, H, T, d), 20 + s) for s in range(4))
    do[:, :, t + 1:] = 0.0
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    for a, s in ((q2, 1), (k2, 2), (v2, 3)):
        a[:, :, t + 1:] += rnd(a[:, :, t + 1:].shape, 100 + s)
    o1, l1 = fwd(q, k, v, 0.5)
    o2, l2 = fwd(q2, k2, v2, 0.5)
    np.testing.assert_array_equal(o1[:, :, :t + 1], o2[:, :, :t + 1])
    np.testing.assert_array_equal(l1[:, :, :t + 1], l2[:, :, :t + 1])
    assert not np.allclose(o1[:, :, t + 1:], o2[:, :, t + 1:])
    g1 = bwd(q, k, v, do, 0.5)
    g2 = bwd(q2, k2, v2, do, 0.5)
    for a, b in zip(g1, g2):
        np.testing.assert_array_equal(a[:, :, :t + 1], b[:, :, :t + 1])


def test_gradient_sums():
    """A common shift of every key adds a per-row constant to the scores, which the softmax
    ignores: sum_j dK_j = 0 per head (per document with a mask).  Rows of P sum to 1:
    sum_j dV_j = sum_i dO_i."""
    B, H, T, d = 2, 2, 37, 5
    q, k, v, do = (rnd((B, H, T, d), 30 + s) for s in range(4))
    dq, dk, dv = bwd(q, k, v, do, 0.45)
    np.testing.assert_allclose(dk.sum(2), 0.0, atol=1e-12)
    np.testing.assert_allclose(dv.sum(2), do.sum(2), atol=1e-12)
    doc = inputs.random_doc_start(B, T, 5, 4, 15).numpy()
    dq, dk, dv = bwd(q, k, v, do, 0.45, doc)
    for b in range(B):
        for s in np.unique(doc[b]):
            e = s + int(np.sum(doc[b] == s))
            np.testing.assert_allclose(dk[b, :, s:e].sum(1), 0.0, atol=1e-12)
            np.testing.assert_allclose(dv[b, :, s:e].sum(1), do[b, :, s:e].sum(1), atol=1e-12)


def test_linear_in_values():
    """V -> a V scales O, dQ, dK by a and leaves LSE and dV unchanged."""
    B, H, T, d = 1, 2, 19, 3
    q, k, v, do = (rnd((B, H, T, d), 40 + s) for s in range(4))
    a = -2.5
    o1, l1 = fwd(q, k, v, 0.7)
    o2, l2 = fwd(q, k, a * v, 0.7)
    np.testing.assert_allclose(o2, a * o1, atol=1e-13)
    np.testing.assert_array_equal(l1, l2)
    g1 = bwd(q, k, v, do, 0.7)
    g2 = bwd(q, k, a * v, do, 0.7)
    np.testing.assert_allclose(g2[0], a * g1[0], atol=1e-12)
    np.testing.assert_allclose(g2[1], a * g1[1], atol=1e-12)
    np.testing.assert_allclose(g2[2], g1[2], atol=1e-13)


def test_documents_equal_independent_slices():
    """Document-causal attention on a packed row equals plain causal attention run on each
    document slice on its own (forward and backward)."""
    B, H, T, d = 2, 2, 45, 4
    q, k, v, do = (rnd((B, H, T, d), 50 + s) for s in range(4))
    doc = inputs.random_doc_start(B, T, 9, 5, 14).numpy()
    o, lse = fwd(q, k, v, 0.55, doc)
    dq, dk, dv = bwd(q, k, v, do, 0.55, doc)
    for b in range(B):
        for s in np.unique(doc[b]):
            e = s + int(np.sum(doc[b] == s))
            sl = (slice(b, b + 1), slice(None), slice(s, e))
            oo, ll = fwd(q[sl], k[sl], v[sl], 0.55)
            np.testing.assert_allclose(o[sl], oo, atol=1e-14)
            np.testing.assert_allclose(lse[b:b + 1, :, s:e], ll, atol=1e-14)
            gq, gk, gv = bwd(q[sl], k[sl], v[sl], do[sl], 0.55)
            np.testing.assert_allclose(dq[sl], gq, atol=1e-13)
            np.testing.assert_allclose(dk[sl], gk, atol=1e-13)
            np.testing.assert_allclose(dv[sl], gv, atol=1e-13)


# --------------------------------------------------------- numerical derivative

@pytest.mark.parametrize("T,d", [(1, 2), (2, 2), (3, 4), (5, 2), (8, 4)])
@pytest.mark.parametrize("with_doc", [False, True])
def test_central_finite_differences(T, d, with_doc):
    """dQ, dK, dV against central differences of L = sum(dO * O), h = 1e-6, in fp64."""
    B, H = 1, 2
    q, k, v, do = (rnd((B, H, T, d), 60 + 7 * T + d + s) for s in range(4))
    scale = 1 / math.sqrt(d)
    doc = inputs.random_doc_start(B, T, T, 1, 3).numpy() if with_doc else None
    grads = bwd(q, k, v, do, scale, doc)
    h = 1e-6
    for which, g in enumerate(grads):
        num = np.zeros_like(g)
        for idx in np.ndindex(*g.shape):
            args = [q, k, v]
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            lp = np.sum(do * fwd(*plus, scale, doc)[0])
            lm = np.sum(do * fwd(*minus, scale, doc)[0])
            num[idx] = (lp - lm) / (2 * h)
        err = np.linalg.norm(num - g) / max(np.linalg.norm(num), 1e-30)
        if np.linalg.norm(num) < 1e-12:
            assert np.max(np.abs(g)) < 1e-9
        else:
            assert err <= 1e-6, (which, err)


# ------------------------------------------------ independent library routine

def torch_reference(q, k, v, do, scale, doc=None):
    """torch CPU float64 SDPA + autograd: an implementation that shares nothing with the oracle."""
    tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    T = q.shape[2]
    if doc is None:
        o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=scale)
    else:
        i = torch.arange(T).view(T, 1)
        j = torch.arange(T).view(1, T)
        ds = torch.tensor(doc, dtype=torch.int64)  # [B,T]
        mask = (j <= i) & (j >= ds.view(-1, T, 1))  # [B,T,T]
        o = torch.nn.functional.scaled_dot_product_attention(
            tq, tk, tv, attn_mask=mask.unsqueeze(1), scale=scale)
    # LSE by the textbook formula on the same masked scores
    s = torch.einsum("bhic,bhjc->bhij", tq.detach(), tk.detach()) * scale
    i = torch.arange(T).view(T, 1)
    j = torch.arange(T).view(1, T)
    vis = (j <= i) if doc is None else ((j <= i) & (j >= torch.tensor(doc, dtype=torch.int64).view(-1, 1, T, 1)))
    lse = torch.logsumexp(s.masked_fill(~vis, float("-inf")), dim=-1)
    o.backward(torch.tensor(do, dtype=torch.float64))
    return (o.detach().numpy(), lse.numpy(), tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy())


@pytest.mark.parametrize("B,H,T,d,with_doc", [
    (1, 4, 64, 32, False),     # the tiny GPT head shape
    (1, 2, 130, 64, False),    # ragged length
    (2, 1, 200, 128, True),    # documents, d = 128
])
def test_against_torch_sdpa_fp64(B, H, T, d, with_doc):
    q, k, v, do = (t.to(torch.float64).numpy() for t in inputs.make_qkvdo(B, H, T, d, 77))
    scale = inputs.fp32_scale(d)
    doc = inputs.random_doc_start(B, T, 8, 20, 90).numpy() if with_doc else None
    o, lse = fwd(q, k, v, scale, doc)
    dq, dk, dv = bwd(q, k, v, do, scale, doc)
    ro, rl, rq, rk, rv = torch_reference(q, k, v, do, scale, doc)
    for a, b in ((o, ro), (lse, rl), (dq, rq), (dk, rk), (dv, rv)):
        assert np.max(np.abs(a - b)) <= 1e-10


# ------------------------------------------------------------- sliding window
# Reading of "How to build an LLM by hand" (agmtopy.github.io), section 9:
# a window of w keys, the query included: i sees j iff i - w < j <= i.

def test_window_covering_everything_is_plain_causal():
    """w >= T changes nothing: bit-identical to the unwindowed oracle (with and without documents)."""
    B, H, T, d = 2, 2, 37, 8
    q, k, v, do = (rnd((B, H, T, d), 500 + s) for s in range(4))
    doc = inputs.random_doc_start(B, T, 4, 5, 15).numpy()
    for dc in (None, doc):
        base_f = oracle.attention_forward(q, k, v, 0.4, dc)
        base_b = oracle.attention_backward(q, k, v, do, 0.4, dc)
        for w in (T, T + 1, 10 ** 6):
            for a, b in zip(oracle.attention_forward(q, k, v, 0.4, dc, window=w), base_f):
                assert np.array_equal(a, b)
            for a, b in zip(oracle.attention_backward(q, k, v, do, 0.4, dc, window=w), base_b):
                assert np.array_equal(a, b)


def test_window_of_one_key_closed_form():
    """w = 1: each query sees only itself: O = V, LSE_i = scale <q_i, k_i>, dQ = dK = 0, dV = dO."""
    B, H, T, d = 1, 3, 20, 6
    q, k, v, do = (rnd((B, H, T, d), 510 + s) for s in range(4))
    o, lse = oracle.attention_forward(q, k, v, 0.7, window=1)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.7, window=1)
    np.testing.assert_array_equal(o, v)
    np.testing.assert_allclose(lse, 0.7 * np.einsum("bhtc,bhtc->bht", q, k), atol=1e-13)
    assert np.max(np.abs(dq)) == 0.0 and np.max(np.abs(dk)) == 0.0
    np.testing.assert_array_equal(dv, do)


def test_window_two_keys_closed_form():
    """w = 2, row i >= 1 sees keys i-1 and i: a two-term softmax written out by hand."""
    B, H, T, d = 1, 1, 9, 4
    q, k, v, _ = (rnd((B, H, T, d), 520 + s) for s in range(4))
    sc = 0.5
    o, lse = oracle.attention_forward(q, k, v, sc, window=2)
    for i in range(1, T):
        a = sc * float(q[0, 0, i] @ k[0, 0, i - 1])
        b = sc * float(q[0, 0, i] @ k[0, 0, i])
        pa = 1.0 / (1.0 + math.exp(b - a))
        np.testing.assert_allclose(o[0, 0, i], pa * v[0, 0, i - 1] + (1 - pa) * v[0, 0, i], atol=1e-13)
        np.testing.assert_allclose(lse[0, 0, i], max(a, b) + math.log(math.exp(a - max(a, b)) + math.exp(b - max(a, b))), atol=1e-13)
    np.testing.assert_allclose(o[0, 0, 0], v[0, 0, 0], atol=0)


@pytest.mark.parametrize("w", [1, 3, 8])
def test_window_probability_rows(w):
    """Rows of P sum to 1; weights outside [i-w+1, i] (and outside the document) are exactly 0."""
    B, H, T, d = 2, 2, 30, 4
    q, k, v = (rnd((B, H, T, d), 530 + s) for s in range(3))
    doc = inputs.random_doc_start(B, T, 6, 4, 12).numpy()
    _, _, p = oracle.attention_forward(q, k, v, 0.5, doc, return_probs=True, window=w)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-12)
    for b in range(B):
        for i in range(T):
            lo = max(int(doc[b, i]), i - w + 1)
            outside = np.ones(T, dtype=bool)
            outside[lo:i + 1] = False
            assert np.all(p[b, :, i, outside] == 0.0)


def test_window_ignores_keys_that_left_it():
    """Row i's outputs do not change when keys and values older than i - w + 1 change."""
    B, H, T, d, w = 1, 2, 40, 8, 6
    q, k, v, do = (rnd((B, H, T, d), 540 + s) for s in range(4))
    o, lse = oracle.attention_forward(q, k, v, 0.3, window=w)
    i = 25
    k2, v2 = k.copy(), v.copy()
    k2[:, :, : i - w + 1] += 3.0
    v2[:, :, : i - w + 1] -= 5.0
    o2, lse2 = oracle.attention_forward(q, k2, v2, 0.3, window=w)
    assert np.array_equal(o[:, :, i], o2[:, :, i]) and np.array_equal(lse[:, :, i], lse2[:, :, i])


@pytest.mark.parametrize("T,d,w", [(5, 2, 2), (8, 4, 3)])
@pytest.mark.parametrize("with_doc", [False, True])
def test_window_finite_differences(T, d, w, with_doc):
    """Windowed backward against central differences of L = sum(dO * O), h = 1e-6, fp64."""
    B, H = 1, 2
    q, k, v, do = (rnd((B, H, T, d), 560 + 7 * T + d + s) for s in range(4))
    scale = 1 / math.sqrt(d)
    doc = inputs.random_doc_start(B, T, T, 1, 5).numpy() if with_doc else None
    grads = oracle.attention_backward(q, k, v, do, scale, doc, window=w)
    h = 1e-6
    for which, g in enumerate(grads):
        num = np.zeros_like(g)
        for idx in np.ndindex(*g.shape):
            plus = [a.copy() for a in (q, k, v)]
            minus = [a.copy() for a in (q, k, v)]
            plus[which][idx] += h
            minus[which][idx] -= h
            lp = np.sum(do * oracle.attention_forward(*plus, scale, doc, window=w)[0])
            lm = np.sum(do * oracle.attention_forward(*minus, scale, doc, window=w)[0])
            num[idx] = (lp - lm) / (2 * h)
        if np.linalg.norm(num) < 1e-12:
            assert np.max(np.abs(g)) < 1e-9
        else:
            assert np.linalg.norm(num - g) / np.linalg.norm(num) <= 1e-6, which


def torch_band_reference(q, k, v, do, scale, w, doc=None):
    """torch CPU float64 SDPA + autograd with an explicit boolean band (and document) mask."""
    tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    B, T = q.shape[0], q.shape[2]
    i = torch.arange(T).view(1, T, 1)
    j = torch.arange(T).view(1, 1, T)
    start = torch.clamp(i - w + 1, min=0).expand(B, T, 1)
    if doc is not None:
        start = torch.maximum(start, torch.tensor(doc, dtype=torch.int64).view(B, T, 1))
    mask = (j <= i) & (j >= start)  # [B,T,T]
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask.unsqueeze(1),
                                                         scale=scale)
    s = torch.einsum("bhic,bhjc->bhij", tq.detach(), tk.detach()) * scale
    lse = torch.logsumexp(s.masked_fill(~mask.unsqueeze(1), float("-inf")), dim=-1)
    o.backward(torch.tensor(do, dtype=torch.float64))
    return (o.detach().numpy(), lse.numpy(), tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy())


@pytest.mark.parametrize("T,d,w,with_doc", [
    (64, 32, 16, False),
    (130, 64, 50, False),
    (200, 128, 129, True),
    (150, 64, 1, True),
])
def test_window_against_torch_sdpa_fp64(T, d, w, with_doc):
    B, H = 2, 2
    q, k, v, do = (t.to(torch.float64).numpy() for t in inputs.make_qkvdo(B, H, T, d, 88))
    scale = inputs.fp32_scale(d)
    doc = inputs.random_doc_start(B, T, 8, 40, 91).numpy() if with_doc else None
    o, lse = oracle.attention_forward(q, k, v, scale, doc, window=w)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, scale, doc, window=w)
    ro, rl, rq, rk, rv = torch_band_reference(q, k, v, do, scale, w, doc)
    for a, b in ((o, ro), (lse, rl), (dq, rq), (dk, rk), (dv, rv)):
        assert np.max(np.abs(a - b)) <= 1e-10


# ---------------------------------------------------------------- KV-cache decode
# The pages' inference engine attends from the new tokens to a KV cache ("How to
# build an LLM by hand", section 2); new token t of Tq sits at position L - Tq + t.

def _decode_case(B, H, Tq, L, d, seed):
    q = rnd((B, Tq, H, d), seed)
    kc, vc = rnd((B, L, H, d), seed + 1), rnd((B, L, H, d), seed + 2)
    return q, kc, vc


@pytest.mark.parametrize("B,H,Tq,L,d", [(1, 2, 1, 1, 4), (2, 3, 1, 37, 8), (1, 2, 5, 20, 4),
                                        (2, 1, 7, 7, 6)])
def test_decode_is_the_last_rows_of_causal_attention(B, H, Tq, L, d):
    """The numpy decode oracle equals the C causal oracle's last Tq rows, with the new tokens'
    queries placed at the end of an otherwise arbitrary query sequence."""
    q, kc, vc = _decode_case(B, H, Tq, L, d, 600 + L)
    o, lse = oracle.decode_forward(q, kc, vc, 0.45)
    qfull = rnd((B, H, L, d), 700 + L)
    qfull[:, :, L - Tq:, :] = q.transpose(0, 2, 1, 3)
    of, lf = oracle.attention_forward(qfull, kc.transpose(0, 2, 1, 3), vc.transpose(0, 2, 1, 3), 0.45)
    np.testing.assert_allclose(o.transpose(0, 2, 1, 3), of[:, :, L - Tq:], atol=1e-13)
    np.testing.assert_allclose(lse, lf[:, :, L - Tq:], atol=1e-13)


def test_decode_single_cached_token():
    """L = 1: the one new token sees only itself: O = v_0, LSE = scale <q, k_0>."""
    q, kc, vc = _decode_case(2, 2, 1, 1, 5, 650)
    o, lse = oracle.decode_forward(q, kc, vc, 0.8)
    np.testing.assert_array_equal(o, vc)
    np.testing.assert_allclose(lse, 0.8 * np.einsum("bthc,bthc->bht", q, kc), atol=1e-13)


def test_decode_against_torch_sdpa_fp64():
    B, H, Tq, L, d = 2, 3, 4, 90, 16
    q, kc, vc = _decode_case(B, H, Tq, L, d, 660)
    o, lse = oracle.decode_forward(q, kc, vc, 0.25)
    tq, tk, tv = (torch.tensor(a, dtype=torch.float64).transpose(1, 2) for a in (q, kc, vc))
    pos = torch.arange(L - Tq, L).view(Tq, 1)
    mask = torch.arange(L).view(1, L) <= pos
    ro = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=0.25)
    s = torch.einsum("bhtc,bhjc->bhtj", tq, tk) * 0.25
    rl = torch.logsumexp(s.masked_fill(~mask, float("-inf")), dim=-1)
    assert np.max(np.abs(o - ro.transpose(1, 2).numpy())) <= 1e-12
    assert np.max(np.abs(lse - rl.numpy())) <= 1e-12


# ------------------------------------------------------- RoPE + QK-norm prologue

def torch_prologue(x, base=10000.0, gain=1.2, eps=1e-6):
    """An independent torch float64 statement: complex-number RoPE (pairs (i, i + d/2) as
    real and imaginary parts, multiplied by e^{-i pos theta}) and torch's rms_norm."""
    B, H, T, d = x.shape
    h = d // 2
    theta = base ** (-torch.arange(0, d, 2, dtype=torch.float64) / d)
    ang = torch.arange(T, dtype=torch.float64)[:, None] * theta[None, :]
    c = torch.complex(x[..., :h], x[..., h:]) * torch.exp(-1j * ang)
    u = torch.cat([c.real, c.imag], dim=-1)
    return gain * torch.nn.functional.rms_norm(u, (d,), eps=eps)


def test_prologue_against_torch_fp64():
    x = torch.tensor(rnd((2, 3, 50, 64), 800), dtype=torch.float64, requires_grad=True)
    dz = rnd((2, 3, 50, 64), 801)
    z = torch_prologue(x)
    z.backward(torch.tensor(dz))
    np.testing.assert_allclose(oracle.qk_prologue_forward(x.detach().numpy()), z.detach().numpy(),
                               atol=1e-12)
    np.testing.assert_allclose(oracle.qk_prologue_backward(x.detach().numpy(), dz),
                               x.grad.numpy(), atol=1e-12)


def test_prologue_position_zero_is_plain_rms_norm():
    """Position 0 has angle 0: the output is gain * x / rms(x)."""
    x = rnd((1, 2, 1, 32), 810)
    z = oracle.qk_prologue_forward(x, gain=1.2)
    np.testing.assert_allclose(z, 1.2 * x / np.sqrt(np.mean(x * x, -1, keepdims=True) + 1e-6),
                               atol=1e-13)


def test_prologue_rotation_keeps_rms_and_commutes_with_the_norm():
    """Each output row has RMS gain * rms/sqrt(rms^2 + eps) (the rotation keeps the norm)."""
    x = rnd((2, 2, 40, 128), 820)
    z = oracle.qk_prologue_forward(x, gain=1.0, eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(z * z, -1)), 1.0, atol=1e-12)


def test_prologue_scores_depend_on_relative_position_only():
    """<RoPE(q)_m, RoPE(k)_n> is unchanged when both positions move by the same amount."""
    d, T = 16, 30
    q, k = rnd((1, 1, 1, d), 830), rnd((1, 1, 1, d), 831)
    Q = np.repeat(q, T, axis=2)
    K = np.repeat(k, T, axis=2)
    zq = oracle.qk_prologue_forward(Q, gain=1.0, eps=0.0)[0, 0]
    zk = oracle.qk_prologue_forward(K, gain=1.0, eps=0.0)[0, 0]
    for m, n, s in ((5, 2, 7), (20, 11, 3), (9, 9, 15)):
        np.testing.assert_allclose(zq[m] @ zk[n], zq[m + s] @ zk[n + s], atol=1e-12)


def test_prologue_finite_differences():
    x = rnd((1, 1, 6, 8), 840)
    dz = rnd((1, 1, 6, 8), 841)
    g = oracle.qk_prologue_backward(x, dz)
    h = 1e-6
    num = np.zeros_like(x)
    for idx in np.ndindex(*x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        num[idx] = (np.sum(dz * oracle.qk_prologue_forward(xp)) -
                    np.sum(dz * oracle.qk_prologue_forward(xm))) / (2 * h)
    assert np.linalg.norm(num - g) / np.linalg.norm(num) <= 1e-6
