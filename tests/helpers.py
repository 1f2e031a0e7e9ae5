"""Shared helpers for the parity tests: seeded inputs, error metrics, configs."""
from __future__ import annotations

import math

import numpy as np

import synth

# Acceptance bar for bf16-in / fp32-accumulate attention against the float64
# oracle: max-abs error and relative L2 error over the compared outputs.
MAX_ABS_TOL = 1e-2
REL_L2_TOL = 5e-3
N_SAMPLED_ROWS = 1024


def errors(got: np.ndarray, want: np.ndarray):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    diff = got - want
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    den = float(np.linalg.norm(want.ravel()))
    rel = float(np.linalg.norm(diff.ravel()) / den) if den > 0 else float(np.linalg.norm(diff.ravel()))
    return max_abs, rel


# Outside the five stated configurations (edge shapes, other scales, plain
# GEMMs) outputs can exceed 2 in magnitude, where one bf16 rounding step of the
# output alone is up to 2^-8 |y| (0.0156 at |y| = 4). There the per-element
# bound adds that rounding term: |got - want| <= 1e-2 + 2^-8 |want|.
BF16_OUT_REL = 2.0 ** -8


def assert_close(got, want, what="", out_rounding=False):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    max_abs, rel = errors(got, want)
    assert np.all(np.isfinite(got)), "%s: non-finite output" % what
    if out_rounding:
        excess = np.abs(got - want) - (MAX_ABS_TOL + BF16_OUT_REL * np.abs(want))
        worst = float(excess.max()) if excess.size else 0.0
        assert worst <= 0 and rel <= REL_L2_TOL, \
            "%s: max_abs=%.3e exceeds 1e-2 + 2^-8|want| by %.3e; rel_l2=%.3e (tol %.0e)" % (
                what, max_abs, worst, rel, REL_L2_TOL)
    else:
        assert max_abs <= MAX_ABS_TOL and rel <= REL_L2_TOL, \
            "%s: max_abs=%.3e (tol %.0e) rel_l2=%.3e (tol %.0e)" % (what, max_abs, MAX_ABS_TOL, rel, REL_L2_TOL)
    return max_abs, rel


def assert_close_bound(got, want, bound, what=""):
    """Backward bar: per element |got - want| <= 2 * bound + 2^-8 |want| + 1e-6, where
    ``bound`` is the oracle's first-order rounding-error scale of a bf16-operand,
    fp32-accumulate backward (the factor 2 covers fp32 sums of up to 2^15
    terms and the exp2 / log-sum-exp approximations; 2^-8 |want| the bf16
    output rounding), and relative L2 <= 5e-3 as in the forward."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    max_abs, rel = errors(got, want)
    assert np.all(np.isfinite(got)), "%s: non-finite output" % what
    excess = np.abs(got - want) - (2.0 * bound + BF16_OUT_REL * np.abs(want) + 1e-6)
    worst = float(excess.max()) if excess.size else 0.0
    assert worst <= 0 and rel <= REL_L2_TOL, \
        "%s: max_abs=%.3e exceeds the rounding bound by %.3e; rel_l2=%.3e (tol %.0e)" % (
            what, max_abs, worst, rel, REL_L2_TOL)
    return max_abs, rel


def attn_inputs(B, N, H_q, H_kv, d, seed=0, factor=1.0, v_factor=None):
    """bf16 bit arrays q [B,N,H_q,d], k/v [B,N,H_kv,d] from the seeded generator."""
    q = synth.bf16_bits((B, N, H_q, d), seed, "q", factor)
    k = synth.bf16_bits((B, N, H_kv, d), seed, "k", factor)
    v = synth.bf16_bits((B, N, H_kv, d), seed, "v", factor if v_factor is None else v_factor)
    return q, k, v


def sampled_rows(B, N, seed, n=N_SAMPLED_ROWS):
    """>= n seeded flat positions b*N+t, always including the tile edges."""
    must = [0, N - 1, 127, 128]
    if N % 128:
        must.append(N - 1 - (N % 128))
    extra = []
    for b in range(B):
        extra += [b * N + t for t in must]
    return synth.sample_rows(n, B * N, seed ^ 0x5A17, must_include=extra)


# Config 5 grid: N x H_q x H_kv (H_kv <= H_q), row-major in the listed order;
# the position in this list is the seed.
def cost_sweep_grid():
    grid = []
    for N in (32768, 65536, 131072, 200000):
        for H_q in (32, 16, 8, 4):
            for H_kv in (8, 4, 1):
                if H_kv <= H_q:
                    grid.append((N, H_q, H_kv))
    return grid


HEAD_CONFIGS_32K = [("MHA", 16, 16), ("GQA", 16, 4), ("MQA", 16, 1), ("SQA", 8, 4), ("sSQA", 8, 8),
                    ("xSQA", 4, 4), ("xSMQA", 4, 1)]
LONG_HEAD_CONFIGS = [("MHA", 16, 16), ("SQA", 8, 4), ("xSQA", 4, 4)]


def default_scale(d):
    return 1.0 / math.sqrt(d)


# ---------------------------------------------------------------- GPU side
def to_device_bf16(bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def bf16_tensor_to_f64(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def run_attn(q_bits, k_bits, v_bits, causal, scale, d=None):
    """Run sqa_attn_fwd through the C ABI on device copies of the bit arrays."""
    import torch
    import reduced_query_head_b200 as sqa
    B, N, H_q, dd = q_bits.shape
    H_kv = k_bits.shape[2]
    q, k, v = to_device_bf16(q_bits), to_device_bf16(k_bits), to_device_bf16(v_bits)
    out = torch.full((B, N, H_q, dd), float("nan"), dtype=torch.bfloat16, device="cuda")
    sqa.sqa_attn_fwd(q, k, v, out, B, N, H_q, H_kv, dd, int(causal), scale)
    st = sqa.sqa_device_status()
    assert st == sqa.SQA_OK, sqa.sqa_status_string(st)
    return out
