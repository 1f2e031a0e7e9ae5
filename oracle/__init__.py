"""Float64 CPU oracle for decoupled-head attention. TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package. The CUDA
library never does, and this package imports nothing from it.

What it computes is the plain definition, written out step by step:

* Head -> group map. Query head i reads key/value group g(i) = floor(i*H_kv/H_q).
  For H_q divisible by H_kv this is i // (H_q/H_kv): contiguous blocks of query
  heads share one group, as drawn in the GQA explainer ("GQA -- Grouped-Query
  Attention", head-to-group diagram: Q1..Q4 -> KV1, Q5..Q8 -> KV2), and as its
  PyTorch module builds it with ``unsqueeze(2).expand(...)`` ("PyTorchでのGQA実装").
  G = H gives MHA, G = 1 gives MQA (same page, "MHA・MQA・GQAの関係").
  Sparse Query Attention changes only H_q ("Sparse Query Attention (SQA)", abstract).
* Explicit repetition. For each query head the group's K and V are copied out
  into that head's own matrices before any arithmetic.
* Scores. s_u = scale * <q_t, k_u> over keys u (all keys, or u <= t when causal:
  ``scaled_dot_product_attention(..., is_causal=True)`` in the GQA module);
  masked keys are excluded (exp(-inf) = 0 exactly).
* Two-pass softmax. m = max_u s_u; e_u = exp(s_u - m); l = sum_u e_u;
  out = (sum_u e_u v_u) / l.
* Layer. q/k/v = x W^T with no bias, viewed [B, N, H, d]; attention as above;
  heads merged back to [B, N, H_q*d]; out = A Wo^T (the GQA module's
  ``q_proj/k_proj/v_proj/o_proj`` with ``bias=False``).

Everything is float64 from the exact bf16 values. Library matmuls (numpy/BLAS)
serve as the dot-product step; nothing else is blocked, fused or reordered.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

__all__ = [
    "group_of_head", "repeat_kv", "widen_bf16", "bf16_round", "attention",
    "attention_rows", "linear", "layer", "layer_rows", "attention_lse", "attention_backward",
    "attention_backward_q_rows", "attention_backward_kv_rows", "attention_backward_bound", "decode",
]


def group_of_head(i: int, H_q: int, H_kv: int) -> int:
    """KV group read by query head i: floor(i * H_kv / H_q)."""
    return (i * H_kv) // H_q


def widen_bf16(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), returned as float64.

    bfloat16 keeps 7 fraction bits; from a float64 that drops the low 45 of 52.
    Only the normal bf16 range is needed here (inputs are O(1)); values below
    2^-126 in magnitude are rounded on the float32 grid first, which is exact
    for them.
    """
    a = np.asarray(a, dtype=np.float64)
    bits = a.view(np.uint64).copy()
    sign = bits & np.uint64(0x8000000000000000)
    mag = bits & np.uint64(0x7FFFFFFFFFFFFFFF)
    lsb = (mag >> np.uint64(45)) & np.uint64(1)
    mag = (mag + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    out = (sign | mag).view(np.float64)
    tiny = np.abs(a) < 2.0 ** -126
    if np.any(tiny):
        f = a[tiny].astype(np.float32).view(np.uint32).astype(np.uint64)
        flsb = (f >> np.uint64(16)) & np.uint64(1)
        f = (f + np.uint64(0x7FFF) + flsb) & np.uint64(0xFFFF0000)
        out[tiny] = f.astype(np.uint32).view(np.float32).astype(np.float64)
    return out


def repeat_kv(kv: np.ndarray, H_q: int) -> np.ndarray:
    """[B, N, H_kv, d] -> [B, N, H_q, d], head i holding a copy of group g(i)."""
    B, N, H_kv, d = kv.shape
    out = np.empty((B, N, H_q, d), dtype=np.float64)
    for i in range(H_q):
        out[:, :, i, :] = kv[:, :, group_of_head(i, H_q, H_kv), :]
    return out


def _softmax_rows_times_v(s: np.ndarray, vh: np.ndarray) -> np.ndarray:
    """Two-pass softmax of each score row, then the weighted sum of values."""
    m = np.max(s, axis=1, keepdims=True)          # pass 1: row max
    e = np.exp(s - m)                              # pass 2: exponentials (masked -> 0)
    l = np.sum(e, axis=1, keepdims=True)
    return (e @ vh) / l


def _head_rows(qh, kh, vh, t_idx, causal, scale, chunk):
    """Attention of query rows ``qh`` (tokens ``t_idx``) of one head against kh, vh."""
    N = kh.shape[0]
    out = np.empty((qh.shape[0], vh.shape[1]), dtype=np.float64)
    keys = np.arange(N)
    for a in range(0, qh.shape[0], chunk):
        b = min(a + chunk, qh.shape[0])
        # keys past the chunk's last causal position are masked for every row
        # of the chunk, so they are left out of the row instead of set to -inf
        n = min(N, int(t_idx[a:b].max()) + 1) if causal else N
        s = scale * (qh[a:b] @ kh[:n].T)          # explicit score rows
        if causal:
            s[keys[None, :n] > t_idx[a:b, None]] = -np.inf
        out[a:b] = _softmax_rows_times_v(s, vh[:n])
    return out


def attention(q, k, v, causal: bool, scale: float, chunk: int = 256) -> np.ndarray:
    """Full output [B, N, H_q, d] from float64 q [B,N,H_q,d], k/v [B,N,H_kv,d]."""
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    B, N, H_q, d = q.shape
    H_kv = k.shape[2]
    if H_kv > H_q or k.shape != (B, N, H_kv, d) or v.shape != k.shape:
        raise ValueError("shape mismatch")
    out = np.empty_like(q)
    t_all = np.arange(N)
    for b in range(B):
        for i in range(H_q):
            g = group_of_head(i, H_q, H_kv)
            kh = np.array(k[b, :, g, :])      # explicit repetition: head i's own copy
            vh = np.array(v[b, :, g, :])
            out[b, :, i, :] = _head_rows(q[b, :, i, :], kh, vh, t_all, causal, scale, chunk)
    return out


def attention_rows(q_rows, k, v, rows, N: int, causal: bool, scale: float, chunk: int = 32) -> np.ndarray:
    """Output for selected token positions only.

    ``rows`` are flat positions b*N + t; ``q_rows`` is [len(rows), H_q, d] holding
    the query vectors of exactly those positions; k/v are the full [B,N,H_kv,d].
    Returns [len(rows), H_q, d]. Same arithmetic as :func:`attention`.
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.int64)
    B, Nk, H_kv, d = k.shape
    assert Nk == N
    H_q = q_rows.shape[1]
    out = np.empty((len(rows), H_q, d), dtype=np.float64)
    bs, ts = rows // N, rows % N

    def one_head(b, i):
        sel = np.nonzero(bs == b)[0]
        g = group_of_head(i, H_q, H_kv)
        kh = np.asarray(k[b, :, g, :], dtype=np.float64).copy()   # explicit repetition
        vh = np.asarray(v[b, :, g, :], dtype=np.float64).copy()
        out[sel, i, :] = _head_rows(q_rows[sel, i, :], kh, vh, ts[sel], causal, scale, chunk)

    # (batch, head) pairs are independent: run them on a thread pool
    _map_pairs(one_head, [(int(b), i) for b in np.unique(bs) for i in range(H_q)])
    return out


def _map_pairs(fn, pairs):
    """Apply fn(*pair) to independent work items; threads when there are several."""
    workers = min(len(pairs), os.cpu_count() or 1)
    if workers <= 1:
        for pr in pairs:
            fn(*pr)
        return
    try:
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(limits=1, user_api="blas")
    except Exception:   # pragma: no cover - threadpoolctl is optional
        limit = None
    try:
        with ThreadPoolExecutor(max_workers=workers) as ex:
            for f in [ex.submit(fn, *pr) for pr in pairs]:
                f.result()
    finally:
        if limit is not None:
            limit.restore_original_limits()


def linear(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """y = x W^T in float64 (``nn.Linear(..., bias=False)`` with weight [out, in])."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T


def layer(x, wq, wk, wv, wo, H_q: int, H_kv: int, d: int, causal: bool, scale: float,
          storage_rounding: bool = True) -> np.ndarray:
    """Full layer forward, x [B, N, d_model] -> out [B, N, d_model] (float64).

    With ``storage_rounding`` the projected q, k, v and the merged attention
    output are rounded to bf16 where a bf16 pipeline stores them; otherwise the
    whole chain stays in float64.
    """
    x = np.asarray(x, dtype=np.float64)
    B, N, dm = x.shape
    rnd = bf16_round if storage_rounding else (lambda a: a)
    xf = x.reshape(B * N, dm)
    q = rnd(linear(xf, wq)).reshape(B, N, H_q, d)
    k = rnd(linear(xf, wk)).reshape(B, N, H_kv, d)
    v = rnd(linear(xf, wv)).reshape(B, N, H_kv, d)
    a = rnd(attention(q, k, v, causal, scale)).reshape(B * N, H_q * d)
    return linear(a, wo).reshape(B, N, dm)


def layer_rows(x, wq, wk, wv, wo, rows, H_q: int, H_kv: int, d: int, causal: bool, scale: float,
               storage_rounding: bool = True) -> np.ndarray:
    """Layer output at selected flat positions ``rows`` only: [len(rows), d_model].

    K and V are projected for every position (attention needs all keys); Q,
    attention and the output projection only for the selected rows.
    """
    x = np.asarray(x, dtype=np.float64)
    B, N, dm = x.shape
    rnd = bf16_round if storage_rounding else (lambda a: a)
    xf = x.reshape(B * N, dm)
    rows = np.asarray(rows, dtype=np.int64)
    k = rnd(linear(xf, wk)).reshape(B, N, H_kv, d)
    v = rnd(linear(xf, wv)).reshape(B, N, H_kv, d)
    q_rows = rnd(linear(xf[rows], wq)).reshape(len(rows), H_q, d)
    a = rnd(attention_rows(q_rows, k, v, rows, N, causal, scale)).reshape(len(rows), H_q * d)
    return linear(a, wo)


# ---------------------------------------------------------------------------
# Backward pass (gradients of the attention core).
#
# With S = scale * Q_i K_g^T (masked keys excluded), P = softmax(S) by rows and
# O_i = P V_g, the chain rule for a loss with upstream gradient dO_i gives, for
# each query head i and its group g = g(i):
#   dV_g += P^T dO_i
#   dP    = dO_i V_g^T
#   dS    = P * (dP - rowsum(P * dP))      (softmax Jacobian, row by row)
#   dQ_i  = scale * dS K_g
#   dK_g += scale * dS^T Q_i
# A group's K and V are shared by the query heads that read it (the repetition
# of the GQA module's expand), so their gradients are the sums over those heads.
# ---------------------------------------------------------------------------

def attention_lse(q, k, causal: bool, scale: float) -> np.ndarray:
    """Natural-log log-sum-exp of every score row: [B, N, H_q] (float64)."""
    q, k = (np.asarray(t, dtype=np.float64) for t in (q, k))
    B, N, H_q, d = q.shape
    H_kv = k.shape[2]
    out = np.empty((B, N, H_q), dtype=np.float64)
    keys = np.arange(N)
    for b in range(B):
        for i in range(H_q):
            kh = np.array(k[b, :, group_of_head(i, H_q, H_kv), :])
            s = scale * (q[b, :, i, :] @ kh.T)
            if causal:
                s[keys[None, :] > keys[:, None]] = -np.inf
            m = np.max(s, axis=1)
            out[b, :, i] = m + np.log(np.sum(np.exp(s - m[:, None]), axis=1))
    return out


def _head_backward(qh, kh, vh, doh, causal, scale):
    """Gradients for one query head against its group's K/V (all float64)."""
    N = kh.shape[0]
    s = scale * (qh @ kh.T)
    if causal:
        keys = np.arange(N)
        s[keys[None, :] > keys[:, None]] = -np.inf
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    p = e / np.sum(e, axis=1, keepdims=True)
    dv = p.T @ doh
    dp = doh @ vh.T
    ds = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
    dq = scale * (ds @ kh)
    dk = scale * (ds.T @ qh)
    return dq, dk, dv


def attention_backward(q, k, v, dout, causal: bool, scale: float):
    """(dq [B,N,H_q,d], dk [B,N,H_kv,d], dv [B,N,H_kv,d]) for upstream gradient dout [B,N,H_q,d]."""
    q, k, v, dout = (np.asarray(t, dtype=np.float64) for t in (q, k, v, dout))
    B, N, H_q, d = q.shape
    H_kv = k.shape[2]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for i in range(H_q):
            g = group_of_head(i, H_q, H_kv)
            kh = np.array(k[b, :, g, :])      # explicit repetition: head i's own copy
            vh = np.array(v[b, :, g, :])
            dqi, dki, dvi = _head_backward(q[b, :, i, :], kh, vh, dout[b, :, i, :], causal, scale)
            dq[b, :, i, :] = dqi
            dk[b, :, g, :] += dki               # a shared group collects every head's gradient
            dv[b, :, g, :] += dvi
    return dq, dk, dv


def attention_backward_q_rows(q_rows, k, v, dout_rows, rows, N: int, causal: bool, scale: float,
                              chunk: int = 32, with_bound: bool = False):
    """dq for selected token positions only: [len(rows), H_q, d].

    ``rows`` are flat positions b*N + t; ``q_rows`` and ``dout_rows`` hold the
    query vectors and upstream gradients of exactly those positions. A query
    row's gradient needs only its own score row, so each row follows the same
    steps as :func:`_head_backward` (softmax, dP, the Jacobian's row sum, dS K).
    With ``with_bound`` also returns the rows' error scales as
    :func:`attention_backward_bound` defines them.
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    dout_rows = np.asarray(dout_rows, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.int64)
    B, Nk, H_kv, d = k.shape
    assert Nk == N
    H_q = q_rows.shape[1]
    out = np.empty((len(rows), H_q, d), dtype=np.float64)
    bound = np.empty_like(out) if with_bound else None
    bs, ts = rows // N, rows % N
    keys = np.arange(N)

    def one_head(b, i):
        sel = np.nonzero(bs == b)[0]
        g = group_of_head(i, H_q, H_kv)
        kh = np.asarray(k[b, :, g, :], dtype=np.float64).copy()   # explicit repetition
        vh = np.asarray(v[b, :, g, :], dtype=np.float64).copy()
        for a in range(0, len(sel), chunk):
            idx = sel[a:a + chunk]
            t_idx = ts[idx]
            n = min(N, int(t_idx.max()) + 1) if causal else N
            s = scale * (q_rows[idx, i, :] @ kh[:n].T)
            if causal:
                s[keys[None, :n] > t_idx[:, None]] = -np.inf
            m = np.max(s, axis=1, keepdims=True)
            e = np.exp(s - m)
            p = e / np.sum(e, axis=1, keepdims=True)
            dp = dout_rows[idx, i, :] @ vh[:n].T
            ds = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
            out[idx, i, :] = scale * (ds @ kh[:n])
            if with_bound:
                a = np.sum(np.abs(dout_rows[idx, i, :]) * (p @ np.abs(vh[:n])), axis=1, keepdims=True)
                bound[idx, i, :] = scale * ((_U * np.abs(ds) + 2 * _U * p * a) @ np.abs(kh[:n]))

    _map_pairs(one_head, [(int(b), i) for b in np.unique(bs) for i in range(H_q)])
    return (out, bound) if with_bound else out


def attention_backward_kv_rows(q, k, v, dout, kv_rows, causal: bool, scale: float, chunk: int = 128,
                               with_bound: bool = False):
    """(dk, dv) for selected key positions only: each [len(kv_rows), H_kv, d].

    ``kv_rows`` are flat positions b*N + u; q, k, v and dout are the full
    arrays. A key's gradient collects the column u of every query head's
    softmax, and P[t, u] needs all of score row t (its maximum and sum), as
    does the row's D = sum_u P[t,u] dP[t,u]. So for each query head i of group
    g every score row is formed in full, a chunk of query rows at a time,
    following the steps of :func:`_head_backward` (softmax, dP, the Jacobian's
    row sum); only the selected key columns are carried on into
    dV_g[u] += P[:,u]^T dO_i and dK_g[u] += scale * dS[:,u]^T Q_i, summed over
    the heads of the group. With ``with_bound`` also returns the error scales
    (ek, ev) of :func:`attention_backward_bound` at those positions.
    """
    q, k, v, dout = (np.asarray(t, dtype=np.float64) for t in (q, k, v, dout))
    kv_rows = np.asarray(kv_rows, dtype=np.int64)
    B, N, H_q, d = q.shape
    H_kv = k.shape[2]
    bs, us = kv_rows // N, kv_rows % N
    pairs = [(int(b), i) for b in np.unique(bs) for i in range(H_q)]
    parts = {}

    def one_head(b, i):
        sel = np.nonzero(bs == b)[0]
        u_sel = us[sel]
        g = group_of_head(i, H_q, H_kv)
        kh = np.array(k[b, :, g, :])      # explicit repetition: head i's own copy
        vh = np.array(v[b, :, g, :])
        qh, doh = q[b, :, i, :], dout[b, :, i, :]
        dk_h = np.zeros((len(sel), d))
        dv_h = np.zeros((len(sel), d))
        ek_h = np.zeros((len(sel), d)) if with_bound else None
        ev_h = np.zeros((len(sel), d)) if with_bound else None
        keys = np.arange(N)
        for a in range(0, N, chunk):
            t_idx = keys[a:a + chunk]
            n = min(N, int(t_idx[-1]) + 1) if causal else N
            live = u_sel < n                # keys past the chunk's last row have P = 0 there
            if not np.any(live):
                continue
            s = scale * (qh[t_idx] @ kh[:n].T)     # full score rows of the chunk
            if causal:
                s[keys[None, :n] > t_idx[:, None]] = -np.inf
            m = np.max(s, axis=1, keepdims=True)
            e = np.exp(s - m)
            p = e / np.sum(e, axis=1, keepdims=True)
            dp = doh[t_idx] @ vh[:n].T
            dsum = np.sum(p * dp, axis=1, keepdims=True)
            cols = u_sel[live]
            p_c = p[:, cols]
            ds_c = p_c * (dp[:, cols] - dsum)
            dv_h[live] += p_c.T @ doh[t_idx]
            dk_h[live] += scale * (ds_c.T @ qh[t_idx])
            if with_bound:
                arow = np.sum(np.abs(doh[t_idx]) * (p @ np.abs(vh[:n])), axis=1, keepdims=True)
                eds = _U * np.abs(ds_c) + 2 * _U * p_c * arow
                ek_h[live] += scale * (eds.T @ np.abs(qh[t_idx]))
                ev_h[live] += _U * (p_c.T @ np.abs(doh[t_idx]))
        parts[(b, i)] = (sel, g, dk_h, dv_h, ek_h, ev_h)

    _map_pairs(one_head, pairs)
    dk = np.zeros((len(kv_rows), H_kv, d))
    dv = np.zeros_like(dk)
    ek = np.zeros_like(dk) if with_bound else None
    ev = np.zeros_like(dk) if with_bound else None
    for b, i in pairs:                      # a shared group collects every head's gradient
        sel, g, dk_h, dv_h, ek_h, ev_h = parts[(b, i)]
        dk[sel, g] += dk_h
        dv[sel, g] += dv_h
        if with_bound:
            ek[sel, g] += ek_h
            ev[sel, g] += ev_h
    return (dk, dv, ek, ev) if with_bound else (dk, dv)


# ---------------------------------------------------------------------------
# Rounding-error scale of a bf16-operand backward (tolerance for the tests).
#
# A backward that feeds P and dS to bf16 matrix products with fp32 sums makes,
# to first order, these errors (u = 2^-9, half a bf16 step, relative):
#   P rounded:            |dP_err| <= u |P|
#   D from a bf16 forward output O~ (|O~ - O| <= 2u sum_u P |v|, forward P and
#   output rounding):     |D_err[t]| <= 2u A[t],  A[t] = sum_c |dO[t,c]| sum_u P[t,u] |v[u,c]|
#   dS = P (dP - D) rounded, with that D:
#                         |dS_err| <= u |dS| + 2u P A
# which the products carry to
#   dQ: scale * |dS_err| |K|,  dK: scale * |dS_err|^T |Q|,  dV: u |P|^T |dO|.
# ---------------------------------------------------------------------------

_U = 2.0 ** -9


def _head_backward_bound(qh, kh, vh, doh, causal, scale):
    """Error scales (eq, ek, ev) of one head's gradients, as stated above."""
    N = kh.shape[0]
    s = scale * (qh @ kh.T)
    if causal:
        keys = np.arange(N)
        s[keys[None, :] > keys[:, None]] = -np.inf
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    p = e / np.sum(e, axis=1, keepdims=True)
    dp = doh @ vh.T
    ds = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
    a = np.sum(np.abs(doh) * (p @ np.abs(vh)), axis=1, keepdims=True)
    eds = _U * np.abs(ds) + 2 * _U * p * a
    return scale * (eds @ np.abs(kh)), scale * (eds.T @ np.abs(qh)), _U * (p.T @ np.abs(doh))


def attention_backward_bound(q, k, v, dout, causal: bool, scale: float):
    """Per-element error scales (eq, ek, ev) shaped like attention_backward's results."""
    q, k, v, dout = (np.asarray(t, dtype=np.float64) for t in (q, k, v, dout))
    B, N, H_q, d = q.shape
    H_kv = k.shape[2]
    eq = np.zeros_like(q)
    ek = np.zeros_like(k)
    ev = np.zeros_like(v)
    for b in range(B):
        for i in range(H_q):
            g = group_of_head(i, H_q, H_kv)
            bq, bk, bv = _head_backward_bound(q[b, :, i, :], k[b, :, g, :], v[b, :, g, :], dout[b, :, i, :],
                                              causal, scale)
            eq[b, :, i, :] = bq
            ek[b, :, g, :] += bk
            ev[b, :, g, :] += bv
    return eq, ek, ev


# ---------------------------------------------------------------------------
# Decode: one new token per sequence attends to its whole key/value cache.
#
# The GQA explainer's motivation is the autoregressive step ("背景と動機", the
# KV-cache table): each step reads the cache of H_kv groups, and every query
# head of a group reads the same cached K/V. The new token sits at the end of
# the cache (its own K/V already appended), so it sees every cached key: the
# last row of causal attention over the cache.
# ---------------------------------------------------------------------------

def decode(q, k_cache, v_cache, scale: float) -> np.ndarray:
    """out [B, H_q, d] for q [B, H_q, d] against k_cache/v_cache [B, N, H_kv, d] (float64)."""
    q = np.asarray(q, dtype=np.float64)
    k_cache = np.asarray(k_cache, dtype=np.float64)
    v_cache = np.asarray(v_cache, dtype=np.float64)
    B, H_q, d = q.shape
    H_kv = k_cache.shape[2]
    out = np.empty_like(q)
    for b in range(B):
        for i in range(H_q):
            g = group_of_head(i, H_q, H_kv)
            kh = np.array(k_cache[b, :, g, :])     # explicit repetition: head i's own copy
            vh = np.array(v_cache[b, :, g, :])
            s = scale * (kh @ q[b, i, :])           # explicit score row over all cached keys
            out[b, i, :] = _softmax_rows_times_v(s[None, :], vh)[0]
    return out
