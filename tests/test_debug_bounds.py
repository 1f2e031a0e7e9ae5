"""The debug build: every kernel with device bounds checks (SQA_DEBUG_BOUNDS).

The sanitizer is closed on this machine, so a second build of the library checks
every tile coordinate and global index before it is used and records
SQA_ERR_BOUNDS in the device status word instead of making the access. These
tests run small and odd shapes (N in {1, 2, 127, 128, 129, 255, 1000}, heads per
group 1, 2, 4 and 16, causal and not, d = 64 and 128, both forms of the split
last wave) through every entry point of that build: no check may fail, and the
results must still match the float64 oracle. A diagnostic call shows that a
failing check does reach the host as SQA_ERR_BOUNDS, without any access behind
it.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from helpers import (assert_close, assert_close_bound, attn_inputs, bf16_tensor_to_f64, default_scale,
                     to_device_bf16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbg():
    import reduced_query_head_b200 as sqa
    return sqa.load_debug_library()


def _status_ok(dbg):
    import reduced_query_head_b200 as sqa
    st = dbg.sqa_device_status(None)
    assert st == sqa.SQA_OK, sqa.sqa_status_string(st)


def test_failing_check_reaches_the_host(dbg):
    import reduced_query_head_b200 as sqa
    assert dbg.sqa_check_bounds_report(None) == sqa.SQA_ERR_BOUNDS
    assert dbg.sqa_device_status(None) == sqa.SQA_OK        # the report cleared it
    assert sqa.sqa_check_bounds_report() == sqa.SQA_OK      # release build: checks compiled away


SHAPES = [(N, H_q, H_kv) for N in (1, 2, 127, 128, 129, 255, 1000)
          for H_q, H_kv in ((4, 4), (8, 4), (16, 4), (16, 1))]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,H_q,H_kv", SHAPES)
def test_forward_odd_shapes(dbg, N, H_q, H_kv, causal):
    import torch
    d, B = 64, 1
    qb, kb, vb = attn_inputs(B, N, H_q, H_kv, d, 41)
    q, k, v = (to_device_bf16(x) for x in (qb, kb, vb))
    out = torch.full((B, N, H_q, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    assert dbg.sqa_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, N, H_q, H_kv, d,
                            int(causal), ctypes.c_float(0.125), None) == 0
    _status_ok(dbg)
    want = oracle.attention(oracle.widen_bf16(qb), oracle.widen_bf16(kb), oracle.widen_bf16(vb), causal, 0.125)
    assert_close(bf16_tensor_to_f64(out), want, "debug fwd %s" % ((N, H_q, H_kv, causal),), out_rounding=True)


@pytest.mark.parametrize("B,N,H_q,H_kv,d,causal", [
    (2, 255, 4, 2, 128, False), (1, 1000, 8, 4, 128, True), (1, 640, 128, 1, 64, False),   # split: single tiles
    (1, 4096, 4, 4, 64, False), (3, 300, 6, 4, 64, False),                                 # split: pairs; uneven
    (1, 80, 8, 2, 128, True), (1, 161, 16, 1, 128, False), (1, 1600, 4, 4, 128, False)])  # d=128 80-key steps
def test_forward_more_shapes(dbg, B, N, H_q, H_kv, d, causal):
    import torch
    qb, kb, vb = attn_inputs(B, N, H_q, H_kv, d, 42)
    q, k, v = (to_device_bf16(x) for x in (qb, kb, vb))
    out = torch.full((B, N, H_q, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    scale = default_scale(d)
    assert dbg.sqa_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, N, H_q, H_kv, d,
                            int(causal), ctypes.c_float(scale), None) == 0
    _status_ok(dbg)
    want = oracle.attention(oracle.widen_bf16(qb), oracle.widen_bf16(kb), oracle.widen_bf16(vb), causal, scale)
    assert_close(bf16_tensor_to_f64(out), want, "debug fwd", out_rounding=True)


@pytest.mark.parametrize("B,N,H_q,H_kv,d,causal", [(1, 129, 16, 1, 64, True), (2, 255, 4, 2, 128, False),
                                                   (1, 300, 8, 2, 64, False)])
def test_backward_odd_shapes(dbg, B, N, H_q, H_kv, d, causal):
    import torch
    scale = default_scale(d)
    qb, kb, vb = attn_inputs(B, N, H_q, H_kv, d, 43)
    dob = synth.bf16_bits((B, N, H_q, d), 43, "do")
    q, k, v, do = (to_device_bf16(x) for x in (qb, kb, vb, dob))
    out = torch.empty((B, N, H_q, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H_q, N), dtype=torch.float32, device="cuda")
    assert dbg.sqa_attn_fwd_lse(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, N, H_q,
                                H_kv, d, int(causal), ctypes.c_float(scale), None) == 0
    ws_bytes = dbg.sqa_attn_bwd_workspace_bytes(B, N, H_q)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    grads = [torch.full_like(q, float("nan")), torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))]
    assert dbg.sqa_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), do.data_ptr(), lse.data_ptr(),
                            *[g.data_ptr() for g in grads], ws.data_ptr(), ws_bytes, B, N, H_q, H_kv, d,
                            int(causal), ctypes.c_float(scale), None) == 0
    _status_ok(dbg)
    f = [oracle.widen_bf16(x) for x in (qb, kb, vb, dob)]
    want = oracle.attention_backward(*f, causal, scale)
    bound = oracle.attention_backward_bound(*f, causal, scale)
    for name, g, w, e in zip(("dq", "dk", "dv"), grads, want, bound):
        assert_close_bound(bf16_tensor_to_f64(g), w, e, "debug " + name)


@pytest.mark.parametrize("B,N,H_q,H_kv,d", [(1, 1, 4, 4, 64), (3, 1000, 8, 2, 64), (2, 129, 16, 1, 128)])
def test_decode_odd_shapes(dbg, B, N, H_q, H_kv, d):
    import torch
    scale = default_scale(d)
    qb = synth.bf16_bits((B, H_q, d), 44, "q")
    kb = synth.bf16_bits((B, N, H_kv, d), 44, "k")
    vb = synth.bf16_bits((B, N, H_kv, d), 44, "v")
    q, k, v = (to_device_bf16(x) for x in (qb, kb, vb))
    out = torch.full((B, H_q, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws_bytes = dbg.sqa_decode_workspace_bytes(B, N, H_q, H_kv, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    assert dbg.sqa_decode_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), ws.data_ptr(), ws_bytes, B, N,
                              H_q, H_kv, d, ctypes.c_float(scale), None) == 0
    _status_ok(dbg)
    want = oracle.decode(oracle.widen_bf16(qb), oracle.widen_bf16(kb), oracle.widen_bf16(vb), scale)
    assert_close(bf16_tensor_to_f64(out), want, "debug decode", out_rounding=True)


@pytest.mark.parametrize("B,N,dm,H_q,H_kv,d,causal", [(2, 384, 256, 8, 2, 64, True), (3, 200, 256, 4, 2, 64, False)])
def test_layer_odd_shapes(dbg, B, N, dm, H_q, H_kv, d, causal):
    import torch
    bits = [synth.bf16_bits((B, N, dm), 45, "x")] + [
        synth.bf16_bits(s, 45, n, 0.02) for s, n in (((H_q * d, dm), "wq"), ((H_kv * d, dm), "wk"),
                                                      ((H_kv * d, dm), "wv"), ((dm, H_q * d), "wo"))]
    dev = [to_device_bf16(b) for b in bits]
    ws_bytes = dbg.sqa_layer_workspace_bytes(B, N, dm, H_q, H_kv, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    out = torch.full((B, N, dm), float("nan"), dtype=torch.bfloat16, device="cuda")
    assert dbg.sqa_layer_fwd(*[t.data_ptr() for t in dev], out.data_ptr(), ws.data_ptr(), ws_bytes, B, N, dm, H_q,
                             H_kv, d, int(causal), ctypes.c_float(d ** -0.5), None) == 0
    _status_ok(dbg)
    f = [oracle.widen_bf16(b) for b in bits]
    want = oracle.layer(*f, H_q, H_kv, d, causal, d ** -0.5, storage_rounding=True)
    assert_close(bf16_tensor_to_f64(out), want, "debug layer", out_rounding=True)


def test_rows_odd_offset(dbg):
    import torch
    B, N, off, n, H_q, H_kv, d = 1, 777, 333, 300, 8, 2, 64
    qb, kb, vb = attn_inputs(B, N, H_q, H_kv, d, 46)
    q = to_device_bf16(np.ascontiguousarray(qb[:, off:off + n]))
    k, v = to_device_bf16(kb), to_device_bf16(vb)
    out = torch.full((B, n, H_q, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    for causal in (0, 1):
        assert dbg.sqa_attn_fwd_rows(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, n, N, off, H_q, H_kv,
                                     d, causal, ctypes.c_float(0.125), None) == 0
        _status_ok(dbg)
        rows = np.arange(off, off + n)
        want = oracle.attention_rows(oracle.widen_bf16(qb[0, off:off + n]), oracle.widen_bf16(kb),
                                     oracle.widen_bf16(vb), rows, N, bool(causal), 0.125)
        assert_close(bf16_tensor_to_f64(out)[0], want, "debug rows", out_rounding=True)
