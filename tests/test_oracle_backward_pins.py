"""Pins for the oracle's backward pass and row log-sum-exp.

Checked against: central finite differences of the oracle's own forward
(brute force, independent of the gradient formulas), PyTorch float64 autograd
through scaled_dot_product_attention with repeat-interleaved K/V, closed forms
at Q = 0, and GQA = MHA on repeated K/V with the repeated gradients summed.
Planted mistakes check that these pins catch a dropped softmax-Jacobian term
and a missing group sum.
"""
import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _loss(q, k, v, dout, causal, scale):
    return float(np.sum(oracle.attention(q, k, v, causal, scale) * dout))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H_q,H_kv", [(2, 2), (4, 2), (3, 1)])
def test_backward_matches_finite_differences(H_q, H_kv, causal):
    B, N, d, scale, h = 1, 5, 3, 0.6, 1e-6
    q, k, v = _rand((B, N, H_q, d), 1), _rand((B, N, H_kv, d), 2), _rand((B, N, H_kv, d), 3)
    dout = _rand((B, N, H_q, d), 4)
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, causal, scale)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], dout, causal, scale)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], dout, causal, scale)
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=0, atol=1e-7, err_msg=name)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H_q,H_kv", [(4, 4), (4, 2), (8, 1)])
def test_backward_matches_torch_autograd(H_q, H_kv, causal):
    B, N, d, scale = 2, 11, 8, 8 ** -0.5
    q, k, v = _rand((B, N, H_q, d), 5), _rand((B, N, H_kv, d), 6), _rand((B, N, H_kv, d), 7)
    dout = _rand((B, N, H_q, d), 8)
    R = H_q // H_kv
    tq = torch.from_numpy(q).permute(0, 2, 1, 3).requires_grad_()
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).requires_grad_()
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).requires_grad_()
    o = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(R, dim=1), tv.repeat_interleave(R, dim=1), is_causal=causal, scale=scale)
    o.backward(torch.from_numpy(dout).permute(0, 2, 1, 3))
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, causal, scale)
    np.testing.assert_allclose(dq, tq.grad.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


def test_zero_query_closed_forms():
    # Q = 0: uniform weights 1/N (non-causal), so dV_g = sum over the group's heads of
    # mean_t dO; dK = scale * dS^T Q = 0; dQ_i = scale * sum_u (1/N)(dP_u - mean dP) k_u.
    B, N, H_q, H_kv, d, scale = 1, 6, 4, 2, 3, 0.5
    q = np.zeros((B, N, H_q, d))
    k, v, dout = _rand((B, N, H_kv, d), 9), _rand((B, N, H_kv, d), 10), _rand((B, N, H_q, d), 11)
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, False, scale)
    assert np.array_equal(dk, np.zeros_like(dk))
    for g in range(H_kv):
        heads = [i for i in range(H_q) if (i * H_kv) // H_q == g]
        want = sum(dout[0, :, i, :].sum(axis=0) / N for i in heads)
        np.testing.assert_allclose(dv[0, :, g, :], np.broadcast_to(want, (N, d)), atol=1e-14)
        for i in heads:
            dp = dout[0, :, i, :] @ v[0, :, g, :].T                    # [t, u]
            ds = (dp - dp.mean(axis=1, keepdims=True)) / N
            np.testing.assert_allclose(dq[0, :, i, :], scale * ds @ k[0, :, g, :], atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_backward_equals_mha_on_repeated_kv(causal):
    B, N, H_q, H_kv, d, scale = 2, 7, 6, 2, 4, 0.3
    q, k, v = _rand((B, N, H_q, d), 12), _rand((B, N, H_kv, d), 13), _rand((B, N, H_kv, d), 14)
    dout = _rand((B, N, H_q, d), 15)
    R = H_q // H_kv
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, causal, scale)
    dq2, dk2, dv2 = oracle.attention_backward(q, np.repeat(k, R, axis=2), np.repeat(v, R, axis=2), dout,
                                              causal, scale)
    assert np.array_equal(dq, dq2)
    np.testing.assert_allclose(dk, dk2.reshape(B, N, H_kv, R, d).sum(axis=3), atol=1e-13)
    np.testing.assert_allclose(dv, dv2.reshape(B, N, H_kv, R, d).sum(axis=3), atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_lse_matches_torch(causal):
    B, N, H_q, H_kv, d, scale = 2, 9, 4, 2, 5, 0.4
    q, k = _rand((B, N, H_q, d), 16), _rand((B, N, H_kv, d), 17)
    lse = oracle.attention_lse(q, k, causal, scale)
    s = scale * torch.einsum("bthd,buhd->bhtu", torch.from_numpy(q),
                             torch.from_numpy(np.repeat(k, 2, axis=2)))
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).permute(0, 2, 1).numpy(), atol=1e-12)


def test_planted_dropped_jacobian_term_is_caught(monkeypatch):
    def wrong(qh, kh, vh, doh, causal, scale):
        dq, dk, dv = orig(qh, kh, vh, doh, causal, scale)
        s = scale * (qh @ kh.T)
        p = np.exp(s - s.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        ds_wrong = p * (doh @ vh.T)            # rowsum term dropped
        return scale * ds_wrong @ kh, dk, dv
    orig = oracle._head_backward
    monkeypatch.setattr(oracle, "_head_backward", wrong)
    with pytest.raises(AssertionError):
        test_backward_matches_torch_autograd(4, 2, False)


def test_planted_missing_group_sum_is_caught(monkeypatch):
    orig = oracle.attention_backward

    def wrong(q, k, v, dout, causal, scale):
        dq, dk, dv = orig(q, k, v, dout, causal, scale)
        return dq, dk / 2, dv                  # as if only one of two heads counted
    monkeypatch.setattr(oracle, "attention_backward", wrong)
    with pytest.raises(AssertionError):
        test_backward_matches_torch_autograd(4, 2, True)
