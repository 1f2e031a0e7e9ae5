"""Pins for the float64 oracle: facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: a worked
example with closed-form weights, the head-to-group diagram, closed forms
(Q = 0, one key, one dominant key), invariants (MHA special case, GQA equals MHA
on physically repeated K/V, permutation invariance), an independent pure-Python
loop and PyTorch's float64 scaled_dot_product_attention on tiny inputs. The
last group plants mistakes in the oracle and checks that a pin catches each.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _naive_attention(q, k, v, causal, scale):
    """Definition restated with Python loops and math.exp; groups by contiguous blocks."""
    B, N, H_q, d = q.shape
    H_kv = k.shape[2]
    R = H_q // H_kv
    out = np.zeros_like(q)
    for b in range(B):
        for i in range(H_q):
            g = i // R
            for t in range(N):
                keys = range(t + 1) if causal else range(N)
                sc = [scale * sum(q[b, t, i, c] * k[b, u, g, c] for c in range(d)) for u in keys]
                mx = max(sc)
                w = [math.exp(s - mx) for s in sc]
                tot = sum(w)
                for c in range(d):
                    out[b, t, i, c] = sum(wu * v[b, u, g, c] for wu, u in zip(w, keys)) / tot
    return out


# ---------------------------------------------------------------- pages' facts

def test_group_map_matches_gqa_diagram():
    with open(os.path.join(GOLDEN, "gqa_head_groups.json")) as f:
        spec = json.load(f)
    for case in spec["cases"]:
        got = [oracle.group_of_head(i, case["H_q"], case["H_kv"]) for i in range(case["H_q"])]
        assert got == case["groups"]


def test_repeat_kv_matches_numpy_repeat():
    kv = _rand((2, 3, 4, 5), 45)
    assert np.array_equal(oracle.repeat_kv(kv, 8), np.repeat(kv, 2, axis=2))
    assert np.array_equal(oracle.repeat_kv(kv, 4), kv)
    assert np.array_equal(oracle.repeat_kv(kv[:, :, :1], 3), np.repeat(kv[:, :, :1], 3, axis=2))


def test_group_map_floor_rule_uneven():
    # floor(i*H_kv/H_q) for H_q=6, H_kv=4: group sizes 2,1,2,1 and every group is used.
    got = [oracle.group_of_head(i, 6, 4) for i in range(6)]
    assert got == [0, 0, 1, 2, 2, 3]


@pytest.mark.parametrize("causal", [False, True])
def test_worked_example_closed_form(causal):
    with open(os.path.join(GOLDEN, "worked_example_softmax.json")) as f:
        ex = json.load(f)
    q = np.array(ex["q"], dtype=np.float64)[None]
    first = {"0": 0.0, "ln2": math.log(2.0), "ln3": math.log(3.0)}
    k = np.array([[[first[s], ex["k_second_coord"]]] for s in ex["k_first_coord"]])[None]
    v = np.array(ex["v"], dtype=np.float64)[None]
    out = oracle.attention(q, k, v, causal, ex["scale"])
    want = np.array(ex["expected_causal" if causal else "expected_noncausal"])[None]
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-14)


# ---------------------------------------------------------------- special cases

@pytest.mark.parametrize("causal", [False, True])
def test_mha_matches_independent_loop(causal):
    q, k, v = _rand((2, 5, 3, 4), 1), _rand((2, 5, 3, 4), 2), _rand((2, 5, 3, 4), 3)
    np.testing.assert_allclose(oracle.attention(q, k, v, causal, 0.37),
                               _naive_attention(q, k, v, causal, 0.37), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H_q,H_kv", [(4, 2), (4, 1), (6, 3), (8, 8)])
def test_gqa_matches_independent_loop(H_q, H_kv, causal):
    q, k, v = _rand((1, 6, H_q, 3), 4), _rand((1, 6, H_kv, 3), 5), _rand((1, 6, H_kv, 3), 6)
    np.testing.assert_allclose(oracle.attention(q, k, v, causal, 0.5),
                               _naive_attention(q, k, v, causal, 0.5), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H_q,H_kv", [(8, 4), (16, 1), (6, 2), (4, 4)])
def test_gqa_equals_mha_on_physically_repeated_kv(H_q, H_kv, causal):
    q = _rand((2, 9, H_q, 8), 7)
    k, v = _rand((2, 9, H_kv, 8), 8), _rand((2, 9, H_kv, 8), 9)
    R = H_q // H_kv
    k_rep, v_rep = np.repeat(k, R, axis=2), np.repeat(v, R, axis=2)   # contiguous blocks
    a = oracle.attention(q, k, v, causal, 0.25)
    b = oracle.attention(q, k_rep, v_rep, causal, 0.25)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("H_q,H_kv", [(8, 2), (3, 3), (6, 4)])
def test_zero_query_gives_mean_of_values(H_q, H_kv):
    B, N, d = 2, 7, 5
    q = np.zeros((B, N, H_q, d))
    k, v = _rand((B, N, H_kv, d), 10), _rand((B, N, H_kv, d), 11)
    out_nc = oracle.attention(q, k, v, False, 0.125)
    out_c = oracle.attention(q, k, v, True, 0.125)
    prefix = np.cumsum(v, axis=1) / np.arange(1, N + 1)[None, :, None, None]
    for i in range(H_q):
        g = (i * H_kv) // H_q
        np.testing.assert_allclose(out_nc[:, :, i, :], np.broadcast_to(v[:, :, g, :].mean(axis=1, keepdims=True),
                                   (B, N, d)), rtol=0, atol=1e-14)
        np.testing.assert_allclose(out_c[:, :, i, :], prefix[:, :, g, :], rtol=0, atol=1e-14)


def test_vanishing_scale_gives_mean_of_values():
    q, k, v = _rand((1, 6, 2, 4), 12), _rand((1, 6, 1, 4), 13), _rand((1, 6, 1, 4), 14)
    out = oracle.attention(q, k, v, False, 1e-300)
    np.testing.assert_allclose(out[0, :, 0], np.broadcast_to(v[0, :, 0].mean(0), (6, 4)), atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_single_key_returns_its_value(causal):
    q, k, v = _rand((3, 1, 4, 6), 15), _rand((3, 1, 2, 6), 16), _rand((3, 1, 2, 6), 17)
    out = oracle.attention(q, k, v, causal, 0.3)
    for i in range(4):
        assert np.array_equal(out[:, 0, i, :], v[:, 0, i // 2, :])


def test_causal_first_row_returns_first_value():
    q, k, v = _rand((2, 5, 2, 3), 18), _rand((2, 5, 1, 3), 19), _rand((2, 5, 1, 3), 20)
    out = oracle.attention(q, k, v, True, 0.7)
    for i in range(2):
        assert np.array_equal(out[:, 0, i, :], v[:, 0, 0, :])


def test_noncausal_key_value_permutation_invariance():
    q, k, v = _rand((2, 11, 4, 6), 21), _rand((2, 11, 2, 6), 22), _rand((2, 11, 2, 6), 23)
    perm = np.random.default_rng(24).permutation(11)
    a = oracle.attention(q, k, v, False, 0.4)
    b = oracle.attention(q, k[:, perm], v[:, perm], False, 0.4)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_one_dominant_key_selects_its_value():
    N, d = 9, 4
    q = np.zeros((1, N, 1, d)); q[..., 0] = 1.0
    k = _rand((1, N, 1, d), 25, 0.1); k[0, 6, 0, 0] = 60.0
    v = _rand((1, N, 1, d), 26)
    out = oracle.attention(q, k, v, False, 1.0)
    np.testing.assert_allclose(out[0, :, 0], np.broadcast_to(v[0, 6, 0], (N, d)), atol=1e-20)


def test_large_scores_do_not_overflow():
    # exp without the max subtraction would overflow here; the definition does not.
    q = np.full((1, 4, 1, 2), 30.0); k = np.full((1, 4, 1, 2), 30.0)
    k[0, 2, 0, :] = 31.0
    v = _rand((1, 4, 1, 2), 27)
    out = oracle.attention(q, k, v, False, 1.0)
    assert np.all(np.isfinite(out))
    np.testing.assert_allclose(out[0, 0, 0], v[0, 2, 0], atol=1e-20)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H_q,H_kv", [(4, 4), (4, 2), (8, 1), (6, 3)])
def test_matches_torch_float64_sdpa(H_q, H_kv, causal):
    B, N, d = 2, 13, 8
    q, k, v = _rand((B, N, H_q, d), 28), _rand((B, N, H_kv, d), 29), _rand((B, N, H_kv, d), 30)
    R = H_q // H_kv
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(R, dim=1)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(R, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=d ** -0.5)
    out = oracle.attention(q, k, v, causal, d ** -0.5)
    np.testing.assert_allclose(out, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_rows_mode_equals_full_mode(causal):
    B, N, H_q, H_kv, d = 2, 40, 4, 2, 8
    q, k, v = _rand((B, N, H_q, d), 31), _rand((B, N, H_kv, d), 32), _rand((B, N, H_kv, d), 33)
    full = oracle.attention(q, k, v, causal, 0.3)
    rows = np.array([0, 1, 17, 39, 40, 41, 63, 79])
    q_rows = q.reshape(B * N, H_q, d)[rows]
    got = oracle.attention_rows(q_rows, k, v, rows, N, causal, 0.3, chunk=3)
    np.testing.assert_allclose(got, full.reshape(B * N, H_q, d)[rows], rtol=0, atol=1e-14)


# ---------------------------------------------------------------- layer

@pytest.mark.parametrize("H_q,H_kv", [(4, 4), (4, 2)])
def test_layer_matches_torch_module_semantics(H_q, H_kv):
    """Layer mode restated with torch float64 ops: no-bias projections, [B,T,H,d] views,
    K/V expanded per group, causal SDPA, merged heads, output projection."""
    B, N, dm, d = 2, 6, 16, 4
    x = _rand((B, N, dm), 34)
    wq, wk, wv = _rand((H_q * d, dm), 35, 0.2), _rand((H_kv * d, dm), 36, 0.2), _rand((H_kv * d, dm), 37, 0.2)
    wo = _rand((dm, H_q * d), 38, 0.2)
    T = torch.from_numpy
    tq = torch.nn.functional.linear(T(x), T(wq)).view(B, N, H_q, d).transpose(1, 2)
    tk = torch.nn.functional.linear(T(x), T(wk)).view(B, N, H_kv, d).transpose(1, 2)
    tv = torch.nn.functional.linear(T(x), T(wv)).view(B, N, H_kv, d).transpose(1, 2)
    R = H_q // H_kv
    tk = tk.unsqueeze(2).expand(-1, -1, R, -1, -1).reshape(B, H_q, N, d)
    tv = tv.unsqueeze(2).expand(-1, -1, R, -1, -1).reshape(B, H_q, N, d)
    a = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    ref = torch.nn.functional.linear(a.transpose(1, 2).reshape(B, N, H_q * d), T(wo)).numpy()
    out = oracle.layer(x, wq, wk, wv, wo, H_q, H_kv, d, True, d ** -0.5, storage_rounding=False)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_layer_rows_equals_full_layer():
    B, N, dm, d, H_q, H_kv = 2, 9, 16, 4, 4, 2
    x = _rand((B, N, dm), 39)
    wq, wk, wv = _rand((H_q * d, dm), 40, 0.2), _rand((H_kv * d, dm), 41, 0.2), _rand((H_kv * d, dm), 42, 0.2)
    wo = _rand((dm, H_q * d), 43, 0.2)
    for sr in (False, True):
        full = oracle.layer(x, wq, wk, wv, wo, H_q, H_kv, d, True, 0.5, storage_rounding=sr)
        rows = np.array([0, 4, 8, 9, 17])
        got = oracle.layer_rows(x, wq, wk, wv, wo, rows, H_q, H_kv, d, True, 0.5, storage_rounding=sr)
        np.testing.assert_allclose(got, full.reshape(B * N, dm)[rows], rtol=0, atol=1e-13)


# ---------------------------------------------------------------- bf16 helpers

def test_bf16_round_ties_and_torch_agreement():
    one = 1.0
    assert oracle.bf16_round(np.array([one + 2 ** -8]))[0] == 1.0                 # tie -> even
    assert oracle.bf16_round(np.array([one + 3 * 2 ** -8]))[0] == one + 2 ** -6   # tie -> even (up)
    assert oracle.bf16_round(np.array([one + 2 ** -8 + 2 ** -30]))[0] == one + 2 ** -7
    vals = np.random.default_rng(44).standard_normal(20000).astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.bf16_round(vals), ref)


def test_widen_bf16_exact():
    bits = synth.bf16_bits((1000,), 0, "q")
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.widen_bf16(bits), ref)


# ---------------------------------------------------------------- planted mistakes

def test_planted_wrong_group_map_is_caught(monkeypatch):
    monkeypatch.setattr(oracle, "group_of_head", lambda i, H_q, H_kv: i % H_kv)
    with pytest.raises(AssertionError):
        test_gqa_equals_mha_on_physically_repeated_kv(8, 4, False)


def test_planted_off_by_one_causal_mask_is_caught(monkeypatch):
    orig = oracle._head_rows

    def wrong(qh, kh, vh, t_idx, causal, scale, chunk):
        return orig(qh, kh, vh, t_idx - 1 if causal else t_idx, causal, scale, chunk)
    monkeypatch.setattr(oracle, "_head_rows", wrong)
    with pytest.raises((AssertionError, FloatingPointError, ValueError)):
        with np.errstate(all="ignore"):
            test_worked_example_closed_form(True)


def test_planted_dropped_scale_is_caught(monkeypatch):
    orig = oracle._head_rows
    monkeypatch.setattr(oracle, "_head_rows",
                        lambda qh, kh, vh, t, c, s, ch: orig(qh, kh, vh, t, c, 1.0, ch))
    with pytest.raises(AssertionError):
        test_matches_torch_float64_sdpa(4, 2, False)


def test_planted_transposed_value_is_caught(monkeypatch):
    orig = oracle._softmax_rows_times_v
    monkeypatch.setattr(oracle, "_softmax_rows_times_v", lambda s, vh: orig(s, vh[::-1]))
    with pytest.raises(AssertionError):
        test_worked_example_closed_form(False)


def test_planted_missing_normalisation_is_caught(monkeypatch):
    monkeypatch.setattr(oracle, "_softmax_rows_times_v",
                        lambda s, vh: np.exp(s - s.max(1, keepdims=True)) @ vh)
    with pytest.raises(AssertionError):
        test_zero_query_gives_mean_of_values(8, 2)


# ---------------------------------------------------------------- decode
@pytest.mark.parametrize("H_q,H_kv", [(4, 4), (8, 2), (6, 4), (16, 1)])
def test_decode_is_last_causal_row(H_q, H_kv):
    # the new token at position N-1 sees every cached key: the last row of causal attention
    rng = np.random.default_rng(50)
    B, N, d, scale = 2, 37, 8, 0.3
    q = rng.standard_normal((B, N, H_q, d))
    k, v = rng.standard_normal((B, N, H_kv, d)), rng.standard_normal((B, N, H_kv, d))
    want = oracle.attention(q, k, v, True, scale)[:, N - 1]
    got = oracle.decode(q[:, N - 1], k, v, scale)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-13)


def test_decode_closed_forms():
    rng = np.random.default_rng(51)
    B, N, H_q, H_kv, d = 1, 9, 4, 2, 5
    k, v = rng.standard_normal((B, N, H_kv, d)), rng.standard_normal((B, N, H_kv, d))
    # q = 0: uniform weights, the mean of the group's cached values
    out = oracle.decode(np.zeros((B, H_q, d)), k, v, 0.7)
    for i in range(H_q):
        np.testing.assert_allclose(out[0, i], v[0, :, (i * H_kv) // H_q].mean(axis=0), atol=1e-14)
    # one cached key: its value, whatever the query
    out1 = oracle.decode(rng.standard_normal((B, H_q, d)), k[:, :1], v[:, :1], 0.7)
    for i in range(H_q):
        np.testing.assert_allclose(out1[0, i], v[0, 0, (i * H_kv) // H_q], atol=0)


def test_decode_against_torch_sdpa():
    rng = np.random.default_rng(52)
    B, N, H_q, H_kv, d, scale = 2, 23, 8, 2, 16, 0.25
    q = rng.standard_normal((B, H_q, d))
    k, v = rng.standard_normal((B, N, H_kv, d)), rng.standard_normal((B, N, H_kv, d))
    R = H_q // H_kv
    tq = torch.from_numpy(q)[:, :, None, :]
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(R, dim=1)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(R, dim=1)
    want = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale)[:, :, 0].numpy()
    np.testing.assert_allclose(oracle.decode(q, k, v, scale), want, atol=1e-12)
