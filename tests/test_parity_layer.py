"""GPU parity for the projection GEMM and the full attention layer.

sqa_linear_fwd and sqa_layer_fwd run through the C ABI; the float64 oracle
gets the same seeded bf16 inputs. The layer's oracle rounds Q, K, V and the
merged attention output to bf16 where the GPU path stores them.
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import assert_close, bf16_tensor_to_f64, errors, sampled_rows, to_device_bf16

pytestmark = pytest.mark.gpu


def _linear(M, K, N_out, seed):
    import torch
    import reduced_query_head_b200 as sqa
    xb = synth.bf16_bits((M, K), seed, "x")
    wb = synth.bf16_bits((N_out, K), seed, "wq", 0.02)
    y = torch.full((M, N_out), float("nan"), dtype=torch.bfloat16, device="cuda")
    sqa.sqa_linear_fwd(to_device_bf16(xb), to_device_bf16(wb), y, M, K, N_out)
    assert sqa.sqa_device_status() == sqa.SQA_OK
    return bf16_tensor_to_f64(y), oracle.linear(oracle.widen_bf16(xb), oracle.widen_bf16(wb))


@pytest.mark.parametrize("M,K,N_out", [(1, 64, 8), (100, 72, 64), (128, 64, 256), (300, 200, 264),
                                       (1000, 512, 520), (129, 1024, 768), (4096, 2048, 2048)])
def test_linear_matches_float64(M, K, N_out):
    got, want = _linear(M, K, N_out, 7)
    assert_close(got, want, "linear %dx%dx%d" % (M, K, N_out), out_rounding=True)


def _layer_inputs(B, N, dm, H_q, H_kv, d, seed):
    x = synth.bf16_bits((B, N, dm), seed, "x")
    wq = synth.bf16_bits((H_q * d, dm), seed, "wq", 0.02)
    wk = synth.bf16_bits((H_kv * d, dm), seed, "wk", 0.02)
    wv = synth.bf16_bits((H_kv * d, dm), seed, "wv", 0.02)
    wo = synth.bf16_bits((dm, H_q * d), seed, "wo", 0.02)
    return x, wq, wk, wv, wo


def _run_layer(bits, B, N, dm, H_q, H_kv, d, causal, scale):
    import torch
    import reduced_query_head_b200 as sqa
    x, wq, wk, wv, wo = (to_device_bf16(b) for b in bits)
    ws_bytes = sqa.sqa_layer_workspace_bytes(B, N, dm, H_q, H_kv, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    out = torch.full((B, N, dm), float("nan"), dtype=torch.bfloat16, device="cuda")
    sqa.sqa_layer_fwd(x, wq, wk, wv, wo, out, ws, ws_bytes, B, N, dm, H_q, H_kv, d, int(causal), scale)
    assert sqa.sqa_device_status() == sqa.SQA_OK
    return out


@pytest.mark.parametrize("B,N,dm,H_q,H_kv,d,causal", [
    (2, 300, 256, 4, 2, 64, True),
    (1, 257, 512, 8, 8, 64, False),
    (1, 200, 384, 4, 1, 128, True),
    (2, 129, 320, 6, 4, 64, True),       # uneven groups
    (3, 512, 256, 8, 2, 64, True),       # causal, N a multiple of 128: Wo takes row blocks latest first
    (2, 384, 256, 4, 4, 128, True),
    (3, 200, 256, 4, 2, 64, False),      # 128-row blocks of A that straddle two sequences
    (2, 1000, 512, 16, 2, 64, True),
])
def test_layer_small_full(B, N, dm, H_q, H_kv, d, causal):
    bits = _layer_inputs(B, N, dm, H_q, H_kv, d, 13)
    scale = d ** -0.5
    got = bf16_tensor_to_f64(_run_layer(bits, B, N, dm, H_q, H_kv, d, causal, scale))
    f = [oracle.widen_bf16(b) for b in bits]
    want = oracle.layer(f[0], f[1], f[2], f[3], f[4], H_q, H_kv, d, causal, scale, storage_rounding=True)
    assert_close(got, want, "layer", out_rounding=True)
    # the pure float64 chain differs only by the bf16 storage rounding
    want64 = oracle.layer(f[0], f[1], f[2], f[3], f[4], H_q, H_kv, d, causal, scale, storage_rounding=False)
    assert errors(got, want64)[1] < 2e-2


def test_config4_causal_layer_sampled():
    """x [4,16384,2048]; Wq 2048->16*64, Wk/Wv 2048->8*64, Wo 1024->2048, W ~ N(0, 0.02^2); causal, scale 1/8."""
    import torch
    B, N, dm, H_q, H_kv, d = 4, 16384, 2048, 16, 8, 64
    bits = _layer_inputs(B, N, dm, H_q, H_kv, d, 0)
    out = _run_layer(bits, B, N, dm, H_q, H_kv, d, True, 0.125)
    rows = sampled_rows(B, N, 0)
    got = bf16_tensor_to_f64(out.view(B * N, dm)[torch.from_numpy(rows).cuda()])
    f = [oracle.widen_bf16(b) for b in bits]
    want = oracle.layer_rows(f[0], f[1], f[2], f[3], f[4], rows, H_q, H_kv, d, True, 0.125, storage_rounding=True)
    assert_close(got, want, "config4 layer")


def test_encoder_layer_noncausal_sampled():
    """Encoder-style (non-causal) SQA layer on one long sequence: x [1,32768,2048], H_q=8, H_kv=4."""
    import torch
    B, N, dm, H_q, H_kv, d = 1, 32768, 2048, 8, 4, 64
    bits = _layer_inputs(B, N, dm, H_q, H_kv, d, 5)
    out = _run_layer(bits, B, N, dm, H_q, H_kv, d, False, 0.125)
    rows = sampled_rows(B, N, 5)
    got = bf16_tensor_to_f64(out.view(B * N, dm)[torch.from_numpy(rows).cuda()])
    f = [oracle.widen_bf16(b) for b in bits]
    want = oracle.layer_rows(f[0], f[1], f[2], f[3], f[4], rows, H_q, H_kv, d, False, 0.125, storage_rounding=True)
    assert_close(got, want, "encoder layer")


def test_layer_repeated_calls_reuse_the_workspace():
    """Back-to-back calls on one workspace (the row-block counters start from zero every call)
    give the same bits; the output projection reads each block only once it is complete."""
    import torch
    B, N, dm, H_q, H_kv, d = 2, 640, 256, 8, 4, 64
    bits = _layer_inputs(B, N, dm, H_q, H_kv, d, 17)
    import reduced_query_head_b200 as sqa
    x, wq, wk, wv, wo = (to_device_bf16(b) for b in bits)
    ws_bytes = sqa.sqa_layer_workspace_bytes(B, N, dm, H_q, H_kv, d)
    ws = torch.full((ws_bytes,), 0x7F, dtype=torch.uint8, device="cuda")   # garbage counters
    outs = []
    for _ in range(3):
        out = torch.full((B, N, dm), float("nan"), dtype=torch.bfloat16, device="cuda")
        sqa.sqa_layer_fwd(x, wq, wk, wv, wo, out, ws, ws_bytes, B, N, dm, H_q, H_kv, d, 1, d ** -0.5)
        outs.append(out)
    assert sqa.sqa_device_status() == sqa.SQA_OK
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    f = [oracle.widen_bf16(b) for b in bits]
    want = oracle.layer(f[0], f[1], f[2], f[3], f[4], H_q, H_kv, d, True, d ** -0.5, storage_rounding=True)
    assert_close(bf16_tensor_to_f64(outs[0]), want, "layer, reused workspace", out_rounding=True)
