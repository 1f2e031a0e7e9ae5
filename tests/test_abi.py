"""The C-ABI library loads and exports every declared symbol; host-side checks.

Runs without a GPU: only entry points that return before touching the device
are called (argument validation, status strings, sizes).
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    with open(os.path.join(ROOT, "include", "sqa.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sqa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def sqa():
    from reduced_query_head_b200 import build
    build.build()
    import reduced_query_head_b200
    return reduced_query_head_b200


def test_header_declares_the_boundary():
    fns = _declared_functions()
    for name in ("sqa_attn_fwd", "sqa_layer_fwd", "sqa_layer_workspace_bytes", "sqa_device_status",
                 "sqa_status_string"):
        assert name in fns


def test_library_exports_every_declared_symbol(sqa):
    lib = ctypes.CDLL(sqa.build.LIB)
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert set(_declared_functions()) == set(sqa.EXPORTED_SYMBOLS)


def test_debug_library_exports_the_same_symbols(sqa):
    """The bounds-checked build is the same C ABI."""
    lib = sqa.load_debug_library()
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert lib.sqa_status_string(sqa.SQA_ERR_BOUNDS) == b"SQA_ERR_BOUNDS"


def test_status_strings_and_version(sqa):
    assert sqa.sqa_status_string(sqa.SQA_OK) == "SQA_OK"
    assert sqa.sqa_status_string(sqa.SQA_ERR_TIMEOUT) == "SQA_ERR_TIMEOUT"
    assert sqa.sqa_status_string(99) == "SQA_ERR_UNKNOWN"
    assert sqa.sqa_version() >= 100


P = 1 << 20  # a 16-byte aligned fake address; never dereferenced (validation fails first)


@pytest.mark.parametrize("args,code", [
    ((0, P, P, P, 1, 128, 8, 4, 64, 0, 0.125), 1),        # null q
    ((P + 2, P, P, P, 1, 128, 8, 4, 64, 0, 0.125), 1),    # misaligned q
    ((P, P, P, P, 0, 128, 8, 4, 64, 0, 0.125), 1),        # B = 0
    ((P, P, P, P, 1, 0, 8, 4, 64, 0, 0.125), 1),          # N = 0
    ((P, P, P, P, 1, 128, 4, 8, 64, 0, 0.125), 1),        # H_kv > H_q
    ((P, P, P, P, 1, 128, 8, 0, 64, 0, 0.125), 1),        # H_kv = 0
    ((P, P, P, P, 1, 128, 8, 4, 64, 2, 0.125), 1),        # causal not 0/1
    ((P, P, P, P, 1, 128, 8, 4, 64, 0, 0.0), 1),          # scale 0
    ((P, P, P, P, 1, 128, 8, 4, 64, 0, -1.0), 1),         # negative scale
    ((P, P, P, P, 1, 128, 8, 4, 64, 0, float("nan")), 1),
    ((P, P, P, P, 1, 128, 8, 4, 64, 0, float("inf")), 1),
    ((P, P, P, P, 1, 128, 8, 4, 96, 0, 0.125), 2),        # d_head unsupported
    ((P, P, P, P, 1, 128, 8, 4, 32, 0, 0.125), 2),
    ((P, P, P, P, 1 << 16, 1 << 16, 64, 8, 128, 0, 0.1), 1),  # too large for 40-bit strides
])
def test_attn_argument_validation(sqa, args, code):
    st = sqa.lib.sqa_attn_fwd(*args[:10], ctypes.c_float(args[10]), None)
    assert st == code, sqa.sqa_status_string(st)


def test_layer_workspace_size(sqa):
    B, N, dm, H_q, H_kv, d = 4, 16384, 2048, 16, 8, 64
    M = B * N
    # Q, K, V and the attention output in bf16, then one int counter per 128-row block of the
    # attention output (rows stored so far), rounded up to 256 bytes
    counters = -(-(M // 128) * 4 // 256) * 256
    want = 2 * M * H_q * d * 2 + 2 * M * H_kv * d * 2 + counters
    assert sqa.sqa_layer_workspace_bytes(B, N, dm, H_q, H_kv, d) == want
    assert sqa.sqa_layer_workspace_bytes(1, 3, 16, 2, 1, 64) % 256 == 0
    assert sqa.sqa_layer_workspace_bytes(0, 3, 16, 2, 1, 64) == 0
    assert sqa.sqa_layer_workspace_bytes(1, 3, 16, 1, 2, 64) == 0


def test_layer_argument_validation(sqa):
    L = sqa.lib
    ws = sqa.sqa_layer_workspace_bytes(1, 128, 64, 2, 1, 64)
    ok = (P, P, P, P, P, P, P, ws, 1, 128, 64, 2, 1, 64, 1)
    assert L.sqa_layer_fwd(*ok[:7], ws - 256, *ok[8:], ctypes.c_float(0.125), None) == 5   # small workspace
    assert L.sqa_layer_fwd(*ok[:6], P + 16, *ok[7:], ctypes.c_float(0.125), None) == 5     # misaligned ws
    assert L.sqa_layer_fwd(*ok[:6], 0, *ok[7:], ctypes.c_float(0.125), None) == 5          # null ws
    bad_dm = ok[:10] + (60,) + ok[11:]
    assert L.sqa_layer_fwd(*bad_dm, ctypes.c_float(0.125), None) == 1                      # d_model % 8
    bad_d = ok[:13] + (80,) + ok[14:]
    assert L.sqa_layer_fwd(*bad_d, ctypes.c_float(0.125), None) == 2
    assert L.sqa_layer_fwd(0, *ok[1:], ctypes.c_float(0.125), None) == 1                   # null x


def test_linear_argument_validation(sqa):
    L = sqa.lib
    assert L.sqa_linear_fwd(P, P, P, 0, 64, 64, None) == 1
    assert L.sqa_linear_fwd(P, P, P, 16, 60, 64, None) == 1
    assert L.sqa_linear_fwd(P, P, P, 16, 64, 36, None) == 1
    assert L.sqa_linear_fwd(P, 0, P, 16, 64, 64, None) == 1


def test_wait_limit_roundtrip(sqa):
    prev = sqa.sqa_set_wait_limit_ns(12345)
    assert sqa.sqa_set_wait_limit_ns(0) == 12345
    assert sqa.sqa_set_wait_limit_ns(prev) == 2_000_000_000
    assert sqa.lib.sqa_check_wait_timeout(10, None) == 1      # limit below range -> invalid


def test_decode_workspace_size_and_validation(sqa):
    assert sqa.sqa_decode_workspace_bytes(0, 128, 8, 2, 64) == 0
    assert sqa.sqa_decode_workspace_bytes(1, 128, 2, 4, 64) == 0      # H_kv > H_q
    assert sqa.sqa_decode_workspace_bytes(1, 128, 8, 2, 96) == 0      # unsupported head size
    small = sqa.sqa_decode_workspace_bytes(1, 128, 8, 2, 64)
    big = sqa.sqa_decode_workspace_bytes(4, 32768, 16, 4, 128)
    assert small > 0 and big > small and small % 256 == 0 and big % 256 == 0
    fake = 1 << 20                                                      # aligned, never dereferenced
    ws = sqa.sqa_decode_workspace_bytes(1, 128, 8, 2, 64)
    for args, code in [((None, fake, fake, fake, fake, ws, 1, 128, 8, 2, 64, 0.1), sqa.SQA_ERR_INVALID_ARG),
                       ((fake, fake, fake, fake, fake, ws, 1, 128, 2, 4, 64, 0.1), sqa.SQA_ERR_INVALID_ARG),
                       ((fake, fake, fake, fake, fake, ws, 1, 128, 8, 2, 64, -1.0), sqa.SQA_ERR_INVALID_ARG),
                       ((fake, fake, fake, fake, fake, ws, 1, 128, 8, 2, 80, 0.1), sqa.SQA_ERR_UNSUPPORTED),
                       ((fake, fake, fake, fake, fake + 8, ws, 1, 128, 8, 2, 64, 0.1), sqa.SQA_ERR_WORKSPACE),
                       ((fake, fake, fake, fake, fake, ws - 1, 1, 128, 8, 2, 64, 0.1), sqa.SQA_ERR_WORKSPACE)]:
        assert sqa.sqa_decode_fwd(*args, stream=0, raise_on_error=False) == code, args


def test_rows_argument_validation(sqa):
    fake = 1 << 20
    for n_q, n_k, off, code in [(0, 128, 0, sqa.SQA_ERR_INVALID_ARG), (64, 128, 65, sqa.SQA_ERR_INVALID_ARG),
                                (64, 128, -1, sqa.SQA_ERR_INVALID_ARG), (1, 0, 0, sqa.SQA_ERR_INVALID_ARG)]:
        assert sqa.sqa_attn_fwd_rows(fake, fake, fake, fake, 1, n_q, n_k, off, 8, 2, 64, 1, 0.125, stream=0,
                                     raise_on_error=False) == code
    assert sqa.sqa_attn_fwd_rows(fake, fake, fake, fake, 1, 64, 128, 0, 8, 2, 96, 1, 0.125, stream=0,
                                 raise_on_error=False) == sqa.SQA_ERR_UNSUPPORTED


def test_layer_argument_errors_come_before_the_workspace_check(sqa):
    # a problem too large for the library's own array, with an argument sqa_layer_fwd rejects:
    # the argument error is what comes back (nothing touches the device on either path)
    B, N, dm, H_q, H_kv, d = 4, 16384, 2048, 16, 8, 64
    f = sqa.lib.sqa_layer_fwd_static_ws
    ok = (P, P, P, P, P, P)
    assert f(*ok, B, N, dm, H_q, H_kv, d, 1, ctypes.c_float(0.125), None) == sqa.SQA_ERR_WORKSPACE
    assert f(*ok, B, N, dm, H_q, H_kv, d, 2, ctypes.c_float(0.125), None) == sqa.SQA_ERR_INVALID_ARG
    assert f(*ok, B, N, dm, H_q, H_kv, d, 1, ctypes.c_float(0.0), None) == sqa.SQA_ERR_INVALID_ARG
    assert f(*ok, B, N, dm + 4, H_q, H_kv, d, 1, ctypes.c_float(0.125), None) == sqa.SQA_ERR_INVALID_ARG
    assert f(P + 8, P, P, P, P, P, B, N, dm, H_q, H_kv, d, 1, ctypes.c_float(0.125), None) == sqa.SQA_ERR_INVALID_ARG
    assert f(*ok, B, N, dm, H_q, H_kv, 96, 1, ctypes.c_float(0.125), None) == sqa.SQA_ERR_UNSUPPORTED


def test_layer_sizes_that_overflow_are_refused(sqa):
    # head counts whose projection widths or workspace regions do not fit are refused, and the
    # workspace size query returns 0 for them instead of a wrapped-around small number
    big = 1 << 26
    assert sqa.sqa_layer_workspace_bytes(1, 16, 64, big, big, 64) == 0
    assert sqa.sqa_layer_workspace_bytes(1 << 20, 1 << 10, 64, 1024, 1, 64) == 0
    st = sqa.lib.sqa_layer_fwd(P, P, P, P, P, P, P, 1 << 40, 1, 16, 64, big, big, 64, 0, ctypes.c_float(0.125), None)
    assert st == sqa.SQA_ERR_INVALID_ARG
    st = sqa.lib.sqa_layer_fwd_static_ws(P, P, P, P, P, P, 1, 16, 64, big, big, 64, 0, ctypes.c_float(0.125), None)
    assert st == sqa.SQA_ERR_INVALID_ARG
