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


@pytest.mark.parametrize("causal", [False, True])
def test_q_rows_match_torch_autograd(causal):
    # the row-sampled dq against PyTorch float64 autograd at a scattered subset of positions
    B, N, H_q, H_kv, d, scale = 2, 40, 6, 2, 8, 0.35
    q, k, v = _rand((B, N, H_q, d), 20), _rand((B, N, H_kv, d), 21), _rand((B, N, H_kv, d), 22)
    dout = _rand((B, N, H_q, d), 23)
    R = H_q // H_kv
    tq = torch.from_numpy(q).permute(0, 2, 1, 3).requires_grad_()
    o = torch.nn.functional.scaled_dot_product_attention(
        tq, torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(R, dim=1),
        torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(R, dim=1), is_causal=causal, scale=scale)
    o.backward(torch.from_numpy(dout).permute(0, 2, 1, 3))
    want = tq.grad.permute(0, 2, 1, 3).numpy().reshape(B * N, H_q, d)
    rows = np.array([0, 1, 7, 39, 40, 41, 55, 79])
    got = oracle.attention_backward_q_rows(q.reshape(B * N, H_q, d)[rows], k, v,
                                           dout.reshape(B * N, H_q, d)[rows], rows, N, causal, scale, chunk=3)
    np.testing.assert_allclose(got, want[rows], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_column_sums(causal):
    # Rows of P sum to 1 and rows of dS sum to 0, so for every group g
    #   sum_u dV_g[u] = sum over the group's heads i of sum_t dO_i[t],   sum_u dK_g[u] = 0.
    B, N, H_q, H_kv, d, scale = 1, 23, 6, 3, 5, 0.5
    q, k, v = _rand((B, N, H_q, d), 24), _rand((B, N, H_kv, d), 25), _rand((B, N, H_kv, d), 26)
    dout = _rand((B, N, H_q, d), 27)
    _, dk, dv = oracle.attention_backward(q, k, v, dout, causal, scale)
    for g in range(H_kv):
        heads = [i for i in range(H_q) if (i * H_kv) // H_q == g]
        np.testing.assert_allclose(dv[0, :, g, :].sum(axis=0), dout[0][:, heads, :].sum(axis=(0, 1)), atol=1e-12)
        np.testing.assert_allclose(dk[0, :, g, :].sum(axis=0), np.zeros(d), atol=1e-12)


# ---------------------------------------------------------------- the backward's rounding bound
def _rounded_model(q, k, v, dout, causal, scale, drop_d=False):
    """The backward with the roundings a bf16-operand kernel makes: P and dS rounded to bf16,
    D taken from a bf16 forward output, outputs rounded to bf16 (float64 elsewhere)."""
    r = oracle.bf16_round
    B, N, H_q, d = q.shape
    H_kv = k.shape[2]
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    keys = np.arange(N)
    for b in range(B):
        for i in range(H_q):
            g = (i * H_kv) // H_q
            qh, kh, vh, doh = q[b, :, i], k[b, :, g], v[b, :, g], dout[b, :, i]
            s = scale * qh @ kh.T
            if causal:
                s[keys[None, :] > keys[:, None]] = -np.inf
            p = np.exp(s - s.max(1, keepdims=True))
            p /= p.sum(1, keepdims=True)
            o = r(r(p) @ vh)
            dsum = 0.0 if drop_d else np.sum(doh * o, axis=1, keepdims=True)
            ds = r(p * (doh @ vh.T - dsum))
            dq[b, :, i] = r(scale * ds @ kh)
            dk[b, :, g] += scale * ds.T @ qh
            dv[b, :, g] += r(p).T @ doh
    return dq, r(dk), r(dv)


def _bf16_inputs(shape, seed):
    return oracle.bf16_round(_rand(shape, seed))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H_q,H_kv,N", [(4, 4, 64), (8, 2, 96), (6, 4, 50)])
def test_rounded_model_within_bound(H_q, H_kv, N, causal):
    from helpers import assert_close_bound
    d, scale = 64, 0.125
    q, k, v = _bf16_inputs((1, N, H_q, d), 30), _bf16_inputs((1, N, H_kv, d), 31), _bf16_inputs((1, N, H_kv, d), 32)
    dout = _bf16_inputs((1, N, H_q, d), 33)
    exact = oracle.attention_backward(q, k, v, dout, causal, scale)
    bound = oracle.attention_backward_bound(q, k, v, dout, causal, scale)
    model = _rounded_model(q, k, v, dout, causal, scale)
    for name, m, e, bd in zip("qkv", model, exact, bound):
        assert_close_bound(m, e, bd, "d" + name)


def test_bound_catches_planted_mistakes():
    from helpers import assert_close_bound
    N, H_q, H_kv, d, scale = 96, 8, 2, 64, 0.125
    q, k, v = _bf16_inputs((1, N, H_q, d), 34), _bf16_inputs((1, N, H_kv, d), 35), _bf16_inputs((1, N, H_kv, d), 36)
    dout = _bf16_inputs((1, N, H_q, d), 37)
    exact = oracle.attention_backward(q, k, v, dout, True, scale)
    bound = oracle.attention_backward_bound(q, k, v, dout, True, scale)
    dropped = _rounded_model(q, k, v, dout, True, scale, drop_d=True)
    with pytest.raises(AssertionError):
        assert_close_bound(dropped[0], exact[0], bound[0], "dq without D")
    with pytest.raises(AssertionError):
        assert_close_bound(exact[1] * 1.01, exact[1], bound[1], "dk scaled by 1.01")
    with pytest.raises(AssertionError):   # one key tile's worth of dv missing
        dv = exact[2].copy()
        dv[0, 10] = 0.0
        assert_close_bound(dv, exact[2], bound[2], "dv row dropped")


def test_q_rows_bound_matches_full_bound():
    N, H_q, H_kv, d, scale = 40, 4, 2, 16, 0.3
    q, k, v, dout = _rand((1, N, H_q, d), 38), _rand((1, N, H_kv, d), 39), _rand((1, N, H_kv, d), 40), \
        _rand((1, N, H_q, d), 41)
    eq, _, _ = oracle.attention_backward_bound(q, k, v, dout, True, scale)
    rows = np.array([0, 5, 17, 39])
    _, b = oracle.attention_backward_q_rows(q[0][rows], k, v, dout[0][rows], rows, N, True, scale,
                                            with_bound=True)
    np.testing.assert_allclose(b, eq[0][rows], rtol=1e-12, atol=0)


# ---------------------------------------------------------------- dk / dv at selected key positions
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H_q,H_kv", [(4, 4), (6, 2), (5, 3), (8, 1)])
def test_kv_rows_match_full_backward(H_q, H_kv, causal):
    # the row-selected dk/dv (score rows formed in chunks smaller than N) against the full backward
    B, N, d, scale = 2, 29, 6, 0.45
    q, k, v = _rand((B, N, H_q, d), 50), _rand((B, N, H_kv, d), 51), _rand((B, N, H_kv, d), 52)
    dout = _rand((B, N, H_q, d), 53)
    _, dk, dv = oracle.attention_backward(q, k, v, dout, causal, scale)
    _, ek, ev = oracle.attention_backward_bound(q, k, v, dout, causal, scale)
    rows = np.array([0, 3, 4, 17, 28, 29, 30, 44, 57])          # both batches, first and last keys
    gk, gv, bk, bv = oracle.attention_backward_kv_rows(q, k, v, dout, rows, causal, scale, chunk=5,
                                                       with_bound=True)
    np.testing.assert_allclose(gk, dk.reshape(B * N, H_kv, d)[rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(gv, dv.reshape(B * N, H_kv, d)[rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(bk, ek.reshape(B * N, H_kv, d)[rows], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(bv, ev.reshape(B * N, H_kv, d)[rows], rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_kv_rows_match_torch_autograd(causal):
    B, N, H_q, H_kv, d, scale = 2, 37, 6, 2, 8, 0.35
    q, k, v = _rand((B, N, H_q, d), 54), _rand((B, N, H_kv, d), 55), _rand((B, N, H_kv, d), 56)
    dout = _rand((B, N, H_q, d), 57)
    R = H_q // H_kv
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).requires_grad_()
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).requires_grad_()
    o = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).permute(0, 2, 1, 3), tk.repeat_interleave(R, dim=1), tv.repeat_interleave(R, dim=1),
        is_causal=causal, scale=scale)
    o.backward(torch.from_numpy(dout).permute(0, 2, 1, 3))
    want_k = tk.grad.permute(0, 2, 1, 3).numpy().reshape(B * N, H_kv, d)
    want_v = tv.grad.permute(0, 2, 1, 3).numpy().reshape(B * N, H_kv, d)
    rows = np.array([1, 2, 20, 36, 37, 50, 73])
    gk, gv = oracle.attention_backward_kv_rows(q, k, v, dout, rows, causal, scale, chunk=8)
    np.testing.assert_allclose(gk, want_k[rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(gv, want_v[rows], rtol=0, atol=1e-12)


def test_kv_rows_planted_missing_head_is_caught(monkeypatch):
    # a group that collects only one of its heads' shares must fail the autograd pin
    orig = oracle.attention_backward_kv_rows

    def wrong(q, k, v, dout, rows, causal, scale, chunk=128, with_bound=False):
        R = q.shape[2] // k.shape[2]
        keep = np.arange(q.shape[2]) % R == 0
        return orig(q * keep[None, None, :, None], k, v, dout, rows, causal, scale, chunk, with_bound)
    monkeypatch.setattr(oracle, "attention_backward_kv_rows", wrong)
    with pytest.raises(AssertionError):
        test_kv_rows_match_torch_autograd(False)
