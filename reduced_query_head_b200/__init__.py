"""Python binding for libsqa (decoupled-head attention on B200 / sm_100a).

Argument marshalling only: every step runs in the CUDA kernels of
``libsqa.so``. The functions take torch CUDA tensors (bf16, contiguous) or raw
device pointers, and the current torch CUDA stream unless one is given. There
is no fallback: if the library is missing, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os

from .build import LIB as _LIB_PATH

__all__ = [
    "SQA_OK", "SQA_ERR_INVALID_ARG", "SQA_ERR_UNSUPPORTED", "SQA_ERR_CUDA", "SQA_ERR_TIMEOUT",
    "SQA_ERR_WORKSPACE", "SQA_ERR_BOUNDS", "SqaError", "lib", "load_debug_library", "EXPORTED_SYMBOLS", "sqa_attn_fwd", "sqa_attn_fwd_lse", "sqa_attn_fwd_rows",
    "sqa_attn_fwd_grids", "sqa_attn_bwd_workspace_bytes", "sqa_attn_bwd", "sqa_decode_workspace_bytes", "sqa_decode_fwd", "sqa_layer_fwd",
    "sqa_layer_workspace_bytes", "sqa_layer_fwd_static_ws", "SQA_STATIC_WORKSPACE_BYTES", "sqa_linear_fwd",
    "sqa_device_status", "sqa_set_wait_limit_ns",
    "sqa_check_wait_timeout", "sqa_check_exp2_poly", "sqa_check_bounds_report", "sqa_status_string", "sqa_version",
]

SQA_OK, SQA_ERR_INVALID_ARG, SQA_ERR_UNSUPPORTED, SQA_ERR_CUDA, SQA_ERR_TIMEOUT, SQA_ERR_WORKSPACE, SQA_ERR_BOUNDS = range(7)
SQA_STATIC_WORKSPACE_BYTES = 64 << 20   # include/sqa.h

EXPORTED_SYMBOLS = (
    "sqa_attn_fwd", "sqa_attn_fwd_lse", "sqa_attn_fwd_rows", "sqa_attn_fwd_grids", "sqa_attn_bwd_workspace_bytes",
    "sqa_attn_bwd",
    "sqa_decode_workspace_bytes", "sqa_decode_fwd", "sqa_layer_workspace_bytes", "sqa_layer_fwd", "sqa_layer_fwd_static_ws", "sqa_linear_fwd",
    "sqa_device_status",
    "sqa_set_wait_limit_ns", "sqa_check_wait_timeout", "sqa_check_exp2_poly", "sqa_check_bounds_report",
    "sqa_status_string", "sqa_version",
)

if not os.path.exists(_LIB_PATH):
    raise ImportError(
        "libsqa.so is not built (expected at %s); run `python reduced_query_head_b200/build.py` "
        "or `python __graft_entry__.py`" % _LIB_PATH)

_vp, _i, _f, _sz, _ll, _ull = (ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t,
                               ctypes.c_longlong, ctypes.c_ulonglong)


def _declare(L):
    """Argument and result types of every entry point of a loaded libsqa."""
    L.sqa_attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp]
    L.sqa_attn_fwd.restype = _i
    L.sqa_attn_fwd_lse.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp]
    L.sqa_attn_fwd_lse.restype = _i
    L.sqa_attn_fwd_rows.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _vp]
    L.sqa_attn_fwd_rows.restype = _i
    L.sqa_attn_fwd_grids.argtypes = [_i, _i, _i, _i, _i, _i]
    L.sqa_attn_fwd_grids.restype = _i
    L.sqa_attn_bwd_workspace_bytes.argtypes = [_i, _i, _i]
    L.sqa_attn_bwd_workspace_bytes.restype = _sz
    L.sqa_attn_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _i, _i, _i, _i, _i, _i, _f, _vp]
    L.sqa_attn_bwd.restype = _i
    L.sqa_decode_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
    L.sqa_decode_workspace_bytes.restype = _sz
    L.sqa_decode_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _sz, _i, _i, _i, _i, _i, _f, _vp]
    L.sqa_decode_fwd.restype = _i
    L.sqa_layer_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i]
    L.sqa_layer_workspace_bytes.restype = _sz
    L.sqa_layer_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _i, _i, _i, _i, _i, _i, _i, _f, _vp]
    L.sqa_layer_fwd.restype = _i
    L.sqa_layer_fwd_static_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _vp]
    L.sqa_layer_fwd_static_ws.restype = _i
    L.sqa_linear_fwd.argtypes = [_vp, _vp, _vp, _ll, _i, _i, _vp]
    L.sqa_linear_fwd.restype = _i
    L.sqa_device_status.argtypes = [_vp]
    L.sqa_device_status.restype = _i
    L.sqa_set_wait_limit_ns.argtypes = [_ull]
    L.sqa_set_wait_limit_ns.restype = _ull
    L.sqa_check_wait_timeout.argtypes = [_ull, _vp]
    L.sqa_check_wait_timeout.restype = _i
    L.sqa_check_exp2_poly.argtypes = [_vp, _vp, _vp, _ll, _vp]
    L.sqa_check_exp2_poly.restype = _i
    L.sqa_check_bounds_report.argtypes = [_vp]
    L.sqa_check_bounds_report.restype = _i
    L.sqa_status_string.argtypes = [_i]
    L.sqa_status_string.restype = ctypes.c_char_p
    L.sqa_version.argtypes = []
    L.sqa_version.restype = _i
    return L


lib = _declare(ctypes.CDLL(_LIB_PATH))


def load_debug_library():
    """The debug build of the library (device bounds checks that record SQA_ERR_BOUNDS in the
    device status word instead of faulting), built on demand, with the same entry points."""
    from .build import build
    return _declare(ctypes.CDLL(build(debug=True)))


class SqaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__("%s failed: %s" % (what, sqa_status_string(status)))
        self.status = status


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, what: str, raise_on_error: bool):
    if raise_on_error and status != SQA_OK:
        raise SqaError(status, what)
    return status


def sqa_attn_fwd(q, k, v, out, B, N, H_q, H_kv, d_head, causal, scale, stream=None, raise_on_error=True):
    st = lib.sqa_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, N, H_q, H_kv, d_head, int(causal),
                          float(scale), _stream(stream))
    return _check(st, "sqa_attn_fwd", raise_on_error)


def sqa_attn_fwd_lse(q, k, v, out, lse, B, N, H_q, H_kv, d_head, causal, scale, stream=None, raise_on_error=True):
    """sqa_attn_fwd that also writes lse [B, H_q, N] fp32 (natural-log row log-sum-exp)."""
    st = lib.sqa_attn_fwd_lse(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, N, H_q, H_kv, d_head,
                              int(causal), float(scale), _stream(stream))
    return _check(st, "sqa_attn_fwd_lse", raise_on_error)


def sqa_attn_fwd_rows(q, k, v, out, B, N_q, N_k, q_offset, H_q, H_kv, d_head, causal, scale, stream=None,
                      raise_on_error=True):
    """Rows q_offset .. q_offset+N_q-1 of attention over N_k tokens (q/out [B,N_q,H_q,d], k/v [B,N_k,H_kv,d])."""
    st = lib.sqa_attn_fwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, N_q, N_k, q_offset, H_q, H_kv, d_head,
                               int(causal), float(scale), _stream(stream))
    return _check(st, "sqa_attn_fwd_rows", raise_on_error)


def sqa_attn_fwd_grids(B, N, H_q, H_kv, d_head, causal):
    """Kernel launches one sqa_attn_fwd call enqueues for these sizes on the current device (1 or 2; 0 if invalid)."""
    return int(lib.sqa_attn_fwd_grids(B, N, H_q, H_kv, d_head, int(causal)))


def sqa_attn_bwd_workspace_bytes(B, N, H_q):
    return int(lib.sqa_attn_bwd_workspace_bytes(B, N, H_q))


def sqa_attn_bwd(q, k, v, out, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, N, H_q, H_kv, d_head, causal,
                 scale, stream=None, raise_on_error=True):
    """Gradients dq [B,N,H_q,d], dk/dv [B,N,H_kv,d] (group-summed) of sum(out * dout)."""
    st = lib.sqa_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                          _ptr(dv), _ptr(workspace), int(workspace_bytes), B, N, H_q, H_kv, d_head, int(causal),
                          float(scale), _stream(stream))
    return _check(st, "sqa_attn_bwd", raise_on_error)


def sqa_decode_workspace_bytes(B, N, H_q, H_kv, d_head):
    return int(lib.sqa_decode_workspace_bytes(B, N, H_q, H_kv, d_head))


def sqa_decode_fwd(q, k_cache, v_cache, out, workspace, workspace_bytes, B, N, H_q, H_kv, d_head, scale,
                   stream=None, raise_on_error=True):
    """One new token per sequence (q [B,H_q,d]) against its K/V cache [B,N,H_kv,d] -> out [B,H_q,d]."""
    st = lib.sqa_decode_fwd(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(workspace),
                            int(workspace_bytes), B, N, H_q, H_kv, d_head, float(scale), _stream(stream))
    return _check(st, "sqa_decode_fwd", raise_on_error)


def sqa_layer_workspace_bytes(B, N, d_model, H_q, H_kv, d_head):
    return int(lib.sqa_layer_workspace_bytes(B, N, d_model, H_q, H_kv, d_head))


def sqa_layer_fwd(x, Wq, Wk, Wv, Wo, out, workspace, workspace_bytes, B, N, d_model, H_q, H_kv, d_head, causal,
                  scale, stream=None, raise_on_error=True):
    st = lib.sqa_layer_fwd(_ptr(x), _ptr(Wq), _ptr(Wk), _ptr(Wv), _ptr(Wo), _ptr(out), _ptr(workspace),
                           int(workspace_bytes), B, N, d_model, H_q, H_kv, d_head, int(causal), float(scale),
                           _stream(stream))
    return _check(st, "sqa_layer_fwd", raise_on_error)


def sqa_layer_fwd_static_ws(x, Wq, Wk, Wv, Wo, out, B, N, d_model, H_q, H_kv, d_head, causal, scale, stream=None,
                            raise_on_error=True):
    """The layer with the library's own scratch array instead of a caller workspace (for callers that
    cannot allocate device memory); problems needing more than SQA_STATIC_WORKSPACE_BYTES are refused."""
    st = lib.sqa_layer_fwd_static_ws(_ptr(x), _ptr(Wq), _ptr(Wk), _ptr(Wv), _ptr(Wo), _ptr(out), B, N, d_model,
                                     H_q, H_kv, d_head, int(causal), float(scale), _stream(stream))
    return _check(st, "sqa_layer_fwd_static_ws", raise_on_error)


def sqa_linear_fwd(x, W, y, M, K, N_out, stream=None, raise_on_error=True):
    st = lib.sqa_linear_fwd(_ptr(x), _ptr(W), _ptr(y), M, K, N_out, _stream(stream))
    return _check(st, "sqa_linear_fwd", raise_on_error)


def sqa_device_status(stream=None):
    return int(lib.sqa_device_status(_stream(stream)))


def sqa_set_wait_limit_ns(ns: int) -> int:
    return int(lib.sqa_set_wait_limit_ns(int(ns)))


def sqa_check_wait_timeout(limit_ns: int, stream=None) -> int:
    return int(lib.sqa_check_wait_timeout(int(limit_ns), _stream(stream)))


def sqa_check_exp2_poly(x, poly, ref, n, stream=None, raise_on_error=True):
    """poly[i] = the kernels' FMA-pipe polynomial 2^x[i], ref[i] = CUDA exp2f(x[i]) (fp32 device arrays)."""
    st = lib.sqa_check_exp2_poly(_ptr(x), _ptr(poly), _ptr(ref), int(n), _stream(stream))
    return _check(st, "sqa_check_exp2_poly", raise_on_error)


def sqa_check_bounds_report(stream=None) -> int:
    """SQA_ERR_BOUNDS if this library was built with device bounds checks, SQA_OK otherwise."""
    return int(lib.sqa_check_bounds_report(_stream(stream)))


def sqa_status_string(status: int) -> str:
    return lib.sqa_status_string(int(status)).decode()


def sqa_version() -> int:
    return int(lib.sqa_version())
