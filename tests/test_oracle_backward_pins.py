"""Pins of the oracle's attention-core gradients (oracle_attend_bwd) against
things other than the function itself: central finite differences of the
oracle's forward attention (itself pinned against the library's attention in
test_oracle_pins.py), autograd of an fp64 torch composition of the same
attention, and closed forms (dv = P^T dout from the forward's probabilities;
uniform attention).  A dropped term of the softmax Jacobian, a missing
1/sqrt(d), a transposed index or a masked key that leaks gradient fails one of
them.
"""
import math

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore")


def _inputs(rng, Nq, Nk, H, d, scale=1.0):
    q = rng.normal(size=(Nq, H, d)) * scale
    k = rng.normal(size=(Nk, H, d)) * scale
    v = rng.normal(size=(Nk, H, d))
    bias = rng.normal(size=(H, Nq, Nk))
    dout = rng.normal(size=(Nq, H, d))
    return q, k, v, bias, dout


def _loss(q, k, v, bias, dout, mask):
    return float(np.sum(oracle.attend(q, k, v, bias, mask) * dout))


@pytest.mark.parametrize("mask", [None, np.array([1, 0, 1, 1, 0], np.uint8)])
def test_gradients_match_central_differences(mask):
    rng = np.random.default_rng(11)
    q, k, v, bias, dout = _inputs(rng, 4, 5, 2, 3)
    grads = oracle.attend_bwd(q, k, v, bias, dout, mask)
    eps = 1e-6
    for x, g in zip((q, k, v, bias), grads):
        num = np.empty_like(x)
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + eps
            lp = _loss(q, k, v, bias, dout, mask)
            x[idx] = keep - eps
            lm = _loss(q, k, v, bias, dout, mask)
            x[idx] = keep
            num[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(g, num, atol=1e-8, rtol=1e-6)


@pytest.mark.parametrize("Nq,Nk,H,d", [(7, 9, 3, 4), (16, 33, 4, 32)])
def test_gradients_match_torch_autograd(Nq, Nk, H, d):
    rng = np.random.default_rng(Nq * 100 + Nk)
    q, k, v, bias, dout = _inputs(rng, Nq, Nk, H, d, scale=0.7)
    mask = (rng.random(Nk) > 0.3).astype(np.uint8)
    mask[0] = 1
    T = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v, bias)]
    tq, tk, tv, tb = T
    s = torch.einsum("jhc,khc->hjk", tq, tk) / math.sqrt(d) + tb
    s = s.masked_fill(torch.tensor(mask == 0)[None, None, :], float("-inf"))
    o = torch.einsum("hjk,khc->jhc", torch.softmax(s, dim=-1), tv)
    (o * torch.tensor(dout)).sum().backward()
    got = oracle.attend_bwd(q, k, v, bias, dout, mask)
    for g, t in zip(got, T):
        np.testing.assert_allclose(g, t.grad.numpy(), atol=1e-12, rtol=1e-10)


def test_dv_is_probabilities_transposed_times_dout():
    rng = np.random.default_rng(5)
    q, k, v, bias, dout = _inputs(rng, 6, 8, 2, 5)
    mask = np.array([1, 1, 0, 1, 1, 1, 0, 1], np.uint8)
    _, probs = oracle.attend(q, k, v, bias, mask, want_probs=True)  # (H, Nq, Nk)
    _, _, dv, _ = oracle.attend_bwd(q, k, v, bias, dout, mask)
    np.testing.assert_allclose(dv, np.einsum("hjk,jhc->khc", probs, dout), atol=1e-13)


def test_uniform_attention_closed_form():
    """q = 0 and bias = 0: p = 1/Nk, so dbias_jk = (dout_j.v_k - dout_j.mean_k v_k)/Nk
    and dk = 0 (every score gradient multiplies q = 0)."""
    rng = np.random.default_rng(9)
    Nq, Nk, H, d = 3, 4, 2, 3
    q = np.zeros((Nq, H, d))
    k = rng.normal(size=(Nk, H, d))
    v = rng.normal(size=(Nk, H, d))
    bias = np.zeros((H, Nq, Nk))
    dout = rng.normal(size=(Nq, H, d))
    dq, dk, dv, db = oracle.attend_bwd(q, k, v, bias, dout)
    vbar = v.mean(axis=0)
    exp_db = (np.einsum("jhc,khc->hjk", dout, v) - np.einsum("jhc,hc->hj", dout, vbar)[:, :, None]) / Nk
    np.testing.assert_allclose(db, exp_db, atol=1e-14)
    np.testing.assert_allclose(dk, 0.0, atol=0)
    np.testing.assert_allclose(dq, np.einsum("hjk,khc->jhc", exp_db, k) / math.sqrt(d), atol=1e-14)


def test_fully_masked_query_rows_get_zero_gradients():
    rng = np.random.default_rng(3)
    q, k, v, bias, dout = _inputs(rng, 3, 4, 2, 3)
    for g in oracle.attend_bwd(q, k, v, bias, dout, np.zeros(4, np.uint8)):
        assert not np.any(g)


def test_core_backward_sums_the_bias_gradient_over_rows():
    rng = np.random.default_rng(21)
    R, N, H, d = 3, 6, 2, 4
    q = rng.normal(size=(R, N, H, d))
    k = rng.normal(size=(R, N, H, d))
    v = rng.normal(size=(R, N, H, d))
    bias = rng.normal(size=(H, N, N))
    dout = rng.normal(size=(R, N, H, d))
    dq, dk, dv, db = oracle.tri_attn_core_bwd(q, k, v, bias, dout)
    acc = np.zeros_like(bias)
    for r in range(R):
        g = oracle.attend_bwd(q[r], k[r], v[r], bias, dout[r])
        np.testing.assert_array_equal(dq[r], g[0])
        np.testing.assert_array_equal(dk[r], g[1])
        np.testing.assert_array_equal(dv[r], g[2])
        acc += g[3]
    np.testing.assert_allclose(db, acc, atol=1e-14)
