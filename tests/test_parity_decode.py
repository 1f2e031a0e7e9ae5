"""GPU parity: sqa_decode_fwd (CUDA, through the C ABI) against the float64 oracle.

One new token per sequence (q [B, H_q, d]) attends to its whole K/V cache
[B, N, H_kv, d]. Same seeded bf16 inputs on both sides; every output element
is compared. Bar: the forward's, relative L2 <= 5e-3 and per element
|got - want| <= 1e-2 + 2^-8 |want| (bf16 P for the P.V product and a bf16
output, as in the attention core).
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import assert_close, bf16_tensor_to_f64, default_scale, to_device_bf16

pytestmark = pytest.mark.gpu


def run_decode(qb, kb, vb, scale):
    import torch
    import reduced_query_head_b200 as sqa
    B, H_q, d = qb.shape
    N, H_kv = kb.shape[1], kb.shape[2]
    q, k, v = to_device_bf16(qb), to_device_bf16(kb), to_device_bf16(vb)
    out = torch.full((B, H_q, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws_bytes = sqa.sqa_decode_workspace_bytes(B, N, H_q, H_kv, d)
    ws = torch.full((ws_bytes,), 0xFF, dtype=torch.uint8, device="cuda")
    sqa.sqa_decode_fwd(q, k, v, out, ws, ws_bytes, B, N, H_q, H_kv, d, scale)
    st = sqa.sqa_device_status()
    assert st == sqa.SQA_OK, sqa.sqa_status_string(st)
    return out


def _check(B, N, H_q, H_kv, d, seed, scale=None):
    scale = default_scale(d) if scale is None else scale
    qb = synth.bf16_bits((B, H_q, d), seed, "q")
    kb = synth.bf16_bits((B, N, H_kv, d), seed, "k")
    vb = synth.bf16_bits((B, N, H_kv, d), seed, "v")
    got = bf16_tensor_to_f64(run_decode(qb, kb, vb, scale))
    want = oracle.decode(oracle.widen_bf16(qb), oracle.widen_bf16(kb), oracle.widen_bf16(vb), scale)
    return assert_close(got, want, str((B, N, H_q, H_kv, d)), out_rounding=True)


SHAPES = [
    # B, N, H_q, H_kv, d
    (1, 1, 1, 1, 64),          # one cached token
    (1, 17, 4, 4, 64),         # part of one 16-key warp slice
    (2, 100, 8, 2, 64),        # ragged tile
    (1, 1000, 16, 1, 64),      # MQA: 16 heads of one group in one 16-row block
    (3, 777, 6, 4, 64),        # uneven groups (floor map)
    (2, 300, 40, 2, 64),       # 20 heads per group: two 16-row blocks
    (1, 500, 96, 2, 64),       # 48 heads per group: two CTA head blocks
    (1, 4096, 32, 8, 128),     # d = 128
    (1, 2048, 64, 2, 128),     # d = 128, 32 heads per group: two head blocks
    (2, 333, 5, 5, 128),       # MHA, odd head count, ragged
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B%dN%dHq%dHkv%dd%d" % s)
def test_decode_full_output(shape):
    _check(*shape, seed=60)


@pytest.mark.parametrize("scale", [0.02, 0.5])
def test_decode_nondefault_scale(scale):
    _check(2, 1500, 8, 4, 64, seed=61, scale=scale)


@pytest.mark.parametrize("H_q,H_kv", [(16, 16), (16, 4), (16, 1), (8, 4)], ids=["MHA", "GQA", "MQA", "SQA"])
def test_decode_long_cache(H_q, H_kv):
    """N = 32768: many splits per (sequence, group); all of them merge in the combine step."""
    _check(4, 32768, H_q, H_kv, 64, seed=62)


def test_decode_matches_last_row_of_the_forward():
    """The decode of the last token equals row N-1 of the causal forward on the same cache."""
    import torch
    from helpers import run_attn
    B, N, H_q, H_kv, d = 1, 1000, 8, 2, 64
    qb = synth.bf16_bits((B, N, H_q, d), 63, "q")
    kb = synth.bf16_bits((B, N, H_kv, d), 63, "k")
    vb = synth.bf16_bits((B, N, H_kv, d), 63, "v")
    full = run_attn(qb, kb, vb, True, 0.125)[:, N - 1].float()
    dec = run_decode(np.ascontiguousarray(qb[:, N - 1]), kb, vb, 0.125).float()
    assert float((full - dec).abs().max()) <= 2e-2
    assert float(torch.linalg.norm(full - dec) / torch.linalg.norm(full)) <= 5e-3


def test_decode_rejects_bad_workspace():
    import torch
    import reduced_query_head_b200 as sqa
    B, N, H_q, H_kv, d = 1, 256, 8, 2, 64
    q = torch.zeros(B, H_q, d, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(B, N, H_kv, d, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(B, H_q, d, dtype=torch.bfloat16, device="cuda")
    need = sqa.sqa_decode_workspace_bytes(B, N, H_q, H_kv, d)
    assert need > 0
    ws = torch.zeros(need + 256, dtype=torch.uint8, device="cuda")
    assert sqa.sqa_decode_fwd(q, k, k, out, ws, need - 1, B, N, H_q, H_kv, d, 0.125,
                              raise_on_error=False) == sqa.SQA_ERR_WORKSPACE
    assert sqa.sqa_decode_fwd(q, k, k, out, ws.data_ptr() + 16, need, B, N, H_q, H_kv, d, 0.125,
                              raise_on_error=False) == sqa.SQA_ERR_WORKSPACE
    assert sqa.sqa_decode_fwd(q, k, k, out, ws, need, B, N, H_q, H_kv, 96, 0.125,
                              raise_on_error=False) == sqa.SQA_ERR_UNSUPPORTED
    assert sqa.sqa_decode_fwd(q, k, k, out, ws, need, B, N, 2, 4, d, 0.125,
                              raise_on_error=False) == sqa.SQA_ERR_INVALID_ARG
    assert sqa.sqa_device_status() == sqa.SQA_OK
