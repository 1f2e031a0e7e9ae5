"""The layer entry point that allocates nothing (sqa_layer_fwd_static_ws).

It serves callers that cannot allocate device memory themselves -- a framework
that owns all device memory through its own allocator, or a plugin interface
that passes the library only inputs and outputs -- by using one library-owned
scratch array per device. This file checks, through the C ABI, that it gives
the same result as sqa_layer_fwd with a caller-provided workspace on two calls
in a row (the array keeps the previous call's contents), and that a problem
too large for the array is refused before anything runs. It is named so that
pytest collects it last, and it needs nothing from earlier tests.
"""
import ctypes

import pytest

from helpers import assert_close, bf16_tensor_to_f64, to_device_bf16

pytestmark = pytest.mark.gpu


def _inputs(B, N, dm, H_q, H_kv, d, seed):
    import synth
    return [synth.bf16_bits((B, N, dm), seed, "x"),
            synth.bf16_bits((H_q * d, dm), seed, "wq", 0.02),
            synth.bf16_bits((H_kv * d, dm), seed, "wk", 0.02),
            synth.bf16_bits((H_kv * d, dm), seed, "wv", 0.02),
            synth.bf16_bits((dm, H_q * d), seed, "wo", 0.02)]


def _with_workspace(dev, B, N, dm, H_q, H_kv, d, causal, scale):
    import torch
    import reduced_query_head_b200 as sqa
    ws_bytes = sqa.sqa_layer_workspace_bytes(B, N, dm, H_q, H_kv, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    out = torch.full((B, N, dm), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = sqa.lib.sqa_layer_fwd(*[t.data_ptr() for t in dev], out.data_ptr(), ws.data_ptr(), ws_bytes, B, N, dm, H_q,
                               H_kv, d, int(causal), ctypes.c_float(scale), None)
    assert st == sqa.SQA_OK, sqa.sqa_status_string(st)
    assert sqa.sqa_device_status() == sqa.SQA_OK
    return out


def _static(dev, B, N, dm, H_q, H_kv, d, causal, scale):
    import torch
    import reduced_query_head_b200 as sqa
    out = torch.full((B, N, dm), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = sqa.lib.sqa_layer_fwd_static_ws(*[t.data_ptr() for t in dev], out.data_ptr(), B, N, dm, H_q, H_kv, d,
                                         int(causal), ctypes.c_float(scale), None)
    assert st == sqa.SQA_OK, sqa.sqa_status_string(st)
    assert sqa.sqa_device_status() == sqa.SQA_OK
    return out


@pytest.mark.parametrize("B,N,dm,H_q,H_kv,d,causal", [
    (2, 1000, 512, 8, 2, 64, True),
    (1, 3000, 1024, 16, 8, 64, True),     # 12 MiB of scratch
    (1, 777, 384, 4, 1, 128, False),
])
def test_static_workspace_matches_caller_workspace_twice(B, N, dm, H_q, H_kv, d, causal):
    scale = d ** -0.5
    # two calls in a row on different inputs: the second must not see the first one's leftovers
    for seed in (21, 22):
        dev = [to_device_bf16(b) for b in _inputs(B, N, dm, H_q, H_kv, d, seed)]
        want = bf16_tensor_to_f64(_with_workspace(dev, B, N, dm, H_q, H_kv, d, causal, scale))
        got = bf16_tensor_to_f64(_static(dev, B, N, dm, H_q, H_kv, d, causal, scale))
        assert_close(got, want, "static vs caller workspace, seed %d" % seed, out_rounding=True)


def test_too_large_for_the_array_is_refused():
    import reduced_query_head_b200 as sqa
    B, N, dm, H_q, H_kv, d = 4, 16384, 2048, 16, 8, 64        # needs 384 MiB of scratch
    assert sqa.sqa_layer_workspace_bytes(B, N, dm, H_q, H_kv, d) > sqa.SQA_STATIC_WORKSPACE_BYTES
    p = 1 << 20   # never dereferenced: the size check comes first
    st = sqa.lib.sqa_layer_fwd_static_ws(p, p, p, p, p, p, B, N, dm, H_q, H_kv, d, 1, ctypes.c_float(0.125), None)
    assert st == sqa.SQA_ERR_WORKSPACE
    st = sqa.lib.sqa_layer_fwd_static_ws(p, p, p, p, p, p, 0, N, dm, H_q, H_kv, d, 1, ctypes.c_float(0.125), None)
    assert st == sqa.SQA_ERR_INVALID_ARG
    # argument errors are reported as such even when the problem is also too large for the array
    st = sqa.lib.sqa_layer_fwd_static_ws(p, p, p, p, p, p, B, N, dm, H_q, H_kv, d, 2, ctypes.c_float(0.125), None)
    assert st == sqa.SQA_ERR_INVALID_ARG
