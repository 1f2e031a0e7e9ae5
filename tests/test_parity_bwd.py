"""GPU parity: sqa_attn_fwd_lse and sqa_attn_bwd (CUDA, through the C ABI) against the float64 oracle.

Same seeded bf16 q, k, v and upstream gradient dO on both sides; the CUDA
backward takes the CUDA forward's own out and lse, as a training step would.
Shapes the oracle finishes in seconds compare every element of dq, dk and dv.
Bar: relative L2 <= 5e-3 as in the forward, and per element
|got - want| <= 2 * E + 2^-8 |want| + 1e-6 with E the oracle's first-order
rounding-error scale of a bf16-operand backward (gradients scale with dO V^T,
about 8 for unit-variance inputs at d = 64, so the forward's absolute 1e-2
does not carry over). At N = 32768 dq is
compared on >= 1024 sampled query rows and dk, dv element by element on >= 1024
sampled key rows (the oracle forms every score row in full for those keys'
softmax columns); the identities below, which hold at any size, are checked
on all of dk and dv as well:
  sum_u dV_g[u] = sum over the group's heads i of sum_t dO_i[t]   (rows of P sum to 1)
  K_g^T dK_g    = sum_i dQ_i^T Q_i                                (both are scale * Q^T dS K)
  V_g^T dV_g    = sum_i O_i^T dO_i                                (V^T P^T dO = O^T dO)
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import (REL_L2_TOL, assert_close_bound, attn_inputs, bf16_tensor_to_f64, default_scale,
                     sampled_rows, to_device_bf16)

pytestmark = pytest.mark.gpu


def _inputs(B, N, H_q, H_kv, d, seed, factor=1.0):
    qb, kb, vb = attn_inputs(B, N, H_q, H_kv, d, seed, factor)
    dob = synth.bf16_bits((B, N, H_q, d), seed, "do")
    return qb, kb, vb, dob


def run_fwd_bwd(qb, kb, vb, dob, causal, scale):
    """Forward with lse, then backward, through the C ABI; returns device tensors."""
    import torch
    import reduced_query_head_b200 as sqa
    B, N, H_q, d = qb.shape
    H_kv = kb.shape[2]
    q, k, v, do = (to_device_bf16(x) for x in (qb, kb, vb, dob))
    nan = float("nan")
    out = torch.full((B, N, H_q, d), nan, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H_q, N), nan, dtype=torch.float32, device="cuda")
    sqa.sqa_attn_fwd_lse(q, k, v, out, lse, B, N, H_q, H_kv, d, int(causal), scale)
    ws_bytes = sqa.sqa_attn_bwd_workspace_bytes(B, N, H_q)
    ws = torch.full((ws_bytes,), 0xFF, dtype=torch.uint8, device="cuda")   # NaN bit patterns as floats
    dq = torch.full((B, N, H_q, d), nan, dtype=torch.bfloat16, device="cuda")
    dk = torch.full((B, N, H_kv, d), nan, dtype=torch.bfloat16, device="cuda")
    dv = torch.full((B, N, H_kv, d), nan, dtype=torch.bfloat16, device="cuda")
    sqa.sqa_attn_bwd(q, k, v, out, do, lse, dq, dk, dv, ws, ws_bytes, B, N, H_q, H_kv, d, int(causal), scale)
    st = sqa.sqa_device_status()
    assert st == sqa.SQA_OK, sqa.sqa_status_string(st)
    return out, lse, dq, dk, dv


def _full_check(B, N, H_q, H_kv, d, causal, seed, scale=None, factor=1.0):
    scale = default_scale(d) if scale is None else scale
    qb, kb, vb, dob = _inputs(B, N, H_q, H_kv, d, seed, factor)
    _, lse, dq, dk, dv = run_fwd_bwd(qb, kb, vb, dob, causal, scale)
    q, k, v, do = (oracle.widen_bf16(x) for x in (qb, kb, vb, dob))
    want_lse = oracle.attention_lse(q, k, causal, scale).transpose(0, 2, 1)
    got_lse = lse.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got_lse))
    assert float(np.max(np.abs(got_lse - want_lse))) <= LSE_TOL
    want = oracle.attention_backward(q, k, v, do, causal, scale)
    bound = oracle.attention_backward_bound(q, k, v, do, causal, scale)
    tag = str((B, N, H_q, H_kv, d, causal))
    for name, got, w, bd in zip(("dq", "dk", "dv"), (dq, dk, dv), want, bound):
        assert_close_bound(bf16_tensor_to_f64(got), w, bd, name + " " + tag)


# The forward's row sum uses an exp2 whose relative error is far below 1e-4
# per term, so ln of the sum moves by less than that; fp32 adds ~1e-6 at
# |lse| ~ 10. 1e-3 leaves a wide margin while catching a missing max or scale.
LSE_TOL = 1e-3

SHAPES = [
    # B, N, H_q, H_kv, d
    (1, 1, 1, 1, 64),        # one token
    (1, 127, 4, 4, 64),      # ragged tile, MHA
    (1, 128, 8, 2, 64),      # exactly one tile
    (1, 129, 16, 1, 64),     # one past a tile, MQA, 16 heads stacked in the dq kernel
    (2, 255, 4, 2, 128),     # batch 2, d = 128
    (3, 300, 6, 4, 64),      # uneven groups (floor map)
    (1, 513, 12, 3, 128),    # R = 4 with 12 heads
    (1, 640, 128, 1, 64),    # R = 128: one token per dq tile
    (1, 1024, 8, 4, 64),     # the small SQA shape of the forward tests
    (1, 1000, 32, 8, 128),   # d = 128 head configuration of the cost sweep
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B%dN%dHq%dHkv%dd%d" % s)
def test_backward_full_output(shape, causal):
    _full_check(*shape, causal, seed=31)


@pytest.mark.parametrize("scale", [0.05, 0.5])
def test_backward_nondefault_scale(scale):
    _full_check(1, 300, 4, 2, 64, True, seed=32, scale=scale)
    _full_check(1, 300, 4, 2, 128, False, seed=33, scale=scale)


def test_backward_many_tiles():
    """32 key tiles and query tiles each: every pipeline stage wraps several times."""
    _full_check(1, 4096, 8, 2, 64, True, seed=34)
    _full_check(1, 4096, 4, 4, 64, False, seed=35)


def test_backward_is_deterministic():
    qb, kb, vb, dob = _inputs(1, 777, 8, 2, 64, seed=36)
    import torch
    a = run_fwd_bwd(qb, kb, vb, dob, True, 0.125)
    b = run_fwd_bwd(qb, kb, vb, dob, True, 0.125)
    for x, y in zip(a, b):   # no atomics anywhere: the same bits every run
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def test_backward_rejects_bad_workspace():
    import torch
    import reduced_query_head_b200 as sqa
    B, N, H_q, H_kv, d = 1, 256, 4, 2, 64
    t = lambda *s: torch.zeros(*s, dtype=torch.bfloat16, device="cuda")
    q, k, v, o, do = t(B, N, H_q, d), t(B, N, H_kv, d), t(B, N, H_kv, d), t(B, N, H_q, d), t(B, N, H_q, d)
    lse = torch.zeros(B, H_q, N, dtype=torch.float32, device="cuda")
    dq, dk, dv = t(B, N, H_q, d), t(B, N, H_kv, d), t(B, N, H_kv, d)
    need = sqa.sqa_attn_bwd_workspace_bytes(B, N, H_q)
    assert need >= 2 * B * H_q * N * 4
    ws = torch.zeros(need + 256, dtype=torch.uint8, device="cuda")
    st = sqa.sqa_attn_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, need - 1, B, N, H_q, H_kv, d, 0, 0.125,
                          raise_on_error=False)
    assert st == sqa.SQA_ERR_WORKSPACE
    st = sqa.sqa_attn_bwd(q, k, v, o, do, lse, dq, dk, dv, ws.data_ptr() + 16, need, B, N, H_q, H_kv, d, 0, 0.125,
                          raise_on_error=False)
    assert st == sqa.SQA_ERR_WORKSPACE
    st = sqa.sqa_attn_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, need, B, N, H_q, H_kv, 96, 0, 0.125,
                          raise_on_error=False)
    assert st == sqa.SQA_ERR_UNSUPPORTED
    assert sqa.sqa_device_status() == sqa.SQA_OK


# ------------------------------------------------------------ N = 32768 (sampled + identities)
LONG = [("MHA", 16, 16, 64, False), ("GQA", 16, 4, 64, False), ("SQA", 8, 4, 64, False),
        ("xSMQA", 4, 1, 64, False), ("SQA-causal-d128", 16, 4, 128, True)]


def _rel_fro(got, want):
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


@pytest.mark.parametrize("name,H_q,H_kv,d,causal", LONG, ids=[c[0] for c in LONG])
def test_backward_long_sampled(name, H_q, H_kv, d, causal):
    import torch
    B, N, seed = 1, 32768, 40 + H_q + H_kv
    scale = default_scale(d)
    qb, kb, vb, dob = _inputs(B, N, H_q, H_kv, d, seed)
    out, _, dq, dk, dv = run_fwd_bwd(qb, kb, vb, dob, causal, scale)
    rows = sampled_rows(B, N, seed)
    idx = torch.from_numpy(rows).cuda()
    got = bf16_tensor_to_f64(dq.view(B * N, H_q, d)[idx])
    q, k, v, do = (oracle.widen_bf16(x) for x in (qb, kb, vb, dob))
    want, bound = oracle.attention_backward_q_rows(q.reshape(B * N, H_q, d)[rows], k, v,
                                                   do.reshape(B * N, H_q, d)[rows], rows, N, causal, scale,
                                                   with_bound=True)
    assert_close_bound(got, want, bound, "dq rows " + name)

    kv_rows = sampled_rows(B, N, seed + 1)
    idx_kv = torch.from_numpy(kv_rows).cuda()
    got_k = bf16_tensor_to_f64(dk.view(B * N, H_kv, d)[idx_kv])
    got_v = bf16_tensor_to_f64(dv.view(B * N, H_kv, d)[idx_kv])
    want_k, want_v, bound_k, bound_v = oracle.attention_backward_kv_rows(q, k, v, do, kv_rows, causal, scale,
                                                                         with_bound=True)
    assert_close_bound(got_k, want_k, bound_k, "dk rows " + name)
    assert_close_bound(got_v, want_v, bound_v, "dv rows " + name)

    dq64, dk64, dv64, o64 = (bf16_tensor_to_f64(x)[0] for x in (dq, dk, dv, out))
    for g in range(H_kv):
        heads = [i for i in range(H_q) if (i * H_kv) // H_q == g]
        # Column sum of dV against the inputs alone. Its error is a sum of bf16
        # roundings of P (|P| <= 1 per term, rows summing to 1) and of dV; as
        # independent errors of at most half a bf16 step, their standard
        # deviation is at most 2^-9 / sqrt(3) * sqrt(sum_t dO^2 + sum_u dV^2): allow 6 of them.
        want_sum = do[0][:, heads, :].sum(axis=(0, 1))
        got_sum = dv64[:, g, :].sum(axis=0)
        sigma = 2.0 ** -9 / np.sqrt(3.0) * np.sqrt((do[0][:, heads, :] ** 2).sum(axis=(0, 1)) +
                                                    (dv64[:, g, :] ** 2).sum(axis=0))
        assert np.all(np.abs(got_sum - want_sum) <= 6 * sigma + 1e-3), (name, g)
        # K^T dK = sum_i dQ_i^T Q_i and V^T dV = sum_i O_i^T dO_i
        lhs_k = k[0, :, g, :].T @ dk64[:, g, :]
        rhs_k = sum(dq64[:, i, :].T @ q[0, :, i, :] for i in heads)
        assert _rel_fro(lhs_k, rhs_k) <= REL_L2_TOL, (name, g, _rel_fro(lhs_k, rhs_k))
        lhs_v = v[0, :, g, :].T @ dv64[:, g, :]
        rhs_v = sum(o64[:, i, :].T @ do[0, :, i, :] for i in heads)
        assert _rel_fro(lhs_v, rhs_v) <= REL_L2_TOL, (name, g, _rel_fro(lhs_v, rhs_v))
    assert np.all(np.isfinite(dk64)) and np.all(np.isfinite(dv64))
