"""Pins for the backward oracle: central finite differences of the forward definition, torch
autograd in fp64 on an independently written forward, and the identities that follow from the
softmax (shifting all keys of a head changes nothing, so their gradients sum to zero; the weights
of a row sum to one, so the value gradients of a group sum to the group's upstream gradients)."""

import numpy as np
import pytest
import torch

import oracle
from oracle.backward import attention_backward_ref, softmax_backward_rowterm


def _inputs(rng, B, h_q, h_kv, S_q, T, d):
    return (rng.standard_normal((B, h_q, S_q, d)), rng.standard_normal((B, h_kv, T, d)),
            rng.standard_normal((B, h_kv, T, d)), rng.standard_normal((B, h_q, S_q, d)))


@pytest.mark.parametrize("causal,window", [(True, None), (True, 3), (False, None)])
def test_finite_differences(causal, window):
    """dL/dx for L = sum(dO * O) by central differences, every element of q, k and v."""
    rng = np.random.default_rng(3)
    B, h_q, h_kv, S_q, T, d = 2, 4, 2, 5, 7, 3
    q, k, v, dO = _inputs(rng, B, h_q, h_kv, S_q, T, d)
    q_start, kv_len = np.array([2, 0]), np.array([7, 6])
    kw = dict(q_start=q_start, kv_len=kv_len, causal=causal, window=window)

    def loss(qq, kk, vv):
        O, _ = oracle.attention_ref(qq, kk, vv, **kw)
        return float((O * dO).sum())

    dQ, dK, dV = attention_backward_ref(q, k, v, dO, **kw)
    eps = 1e-6
    for x, g in ((q, dQ), (k, dK), (v, dV)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + eps
            lp = loss(q, k, v)
            x[idx] = old - eps
            lm = loss(q, k, v)
            x[idx] = old
            num[idx] = (lp - lm) / (2 * eps)
        assert np.allclose(g, num, rtol=0, atol=1e-7), np.abs(g - num).max()


@pytest.mark.parametrize("h_q,h_kv,window", [(8, 2, None), (4, 4, None), (6, 1, 5)])
def test_matches_torch_autograd(h_q, h_kv, window):
    rng = np.random.default_rng(h_q + h_kv)
    B, S, d = 2, 16, 8
    q, k, v, dO = _inputs(rng, B, h_q, h_kv, S, S, d)
    dQ, dK, dV = attention_backward_ref(q, k, v, dO, window=window)
    r = h_q // h_kv
    tq = torch.tensor(q, requires_grad=True)
    tk = torch.tensor(k, requires_grad=True)
    tv = torch.tensor(v, requires_grad=True)
    ones = torch.ones(S, S, dtype=torch.bool)
    mask = torch.tril(ones) if window is None else torch.tril(ones) & torch.triu(ones, diagonal=-(window - 1))
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(r, dim=1), tv.repeat_interleave(r, dim=1), attn_mask=mask)
    out.backward(torch.tensor(dO))
    assert np.allclose(dQ, tq.grad.numpy(), rtol=0, atol=1e-12)
    assert np.allclose(dK, tk.grad.numpy(), rtol=0, atol=1e-12)
    assert np.allclose(dV, tv.grad.numpy(), rtol=0, atol=1e-12)


def test_group_sum_identities():
    rng = np.random.default_rng(9)
    B, h_q, h_kv, S_q, T, d = 2, 6, 2, 9, 12, 5
    q, k, v, dO = _inputs(rng, B, h_q, h_kv, S_q, T, d)
    q_start, kv_len = np.array([3, 0]), np.array([12, 9])
    dQ, dK, dV = attention_backward_ref(q, k, v, dO, q_start=q_start, kv_len=kv_len)
    r = h_q // h_kv
    for b in range(B):
        n = kv_len[b]
        for g in range(h_kv):
            # keys shifted together leave every softmax unchanged
            assert np.allclose(dK[b, g, :n].sum(axis=0), 0.0, atol=1e-12)
            # every row's weights sum to 1
            assert np.allclose(dV[b, g, :n].sum(axis=0), dO[b, g * r:(g + 1) * r].sum(axis=(0, 1)), atol=1e-12)
        assert np.all(dK[b, :, n:] == 0) and np.all(dV[b, :, n:] == 0)


def test_row_term_equals_p_dp():
    rng = np.random.default_rng(4)
    B, h_q, h_kv, S, d = 1, 2, 1, 6, 4
    q, k, v, dO = _inputs(rng, B, h_q, h_kv, S, S, d)
    O, _ = oracle.attention_ref(q, k, v)
    D = softmax_backward_rowterm(O, dO)
    scale = 1 / np.sqrt(d)
    for a in range(h_q):
        S_ = np.where(np.tril(np.ones((S, S), bool)), q[0, a] @ k[0, 0].T * scale, -np.inf)
        P = np.exp(S_ - S_.max(1, keepdims=True))
        P /= P.sum(1, keepdims=True)
        dP = dO[0, a] @ v[0, 0].T
        assert np.allclose(D[0, a], (P * dP).sum(1), atol=1e-13)
