"""The FMA-pipe exp2 of the attention kernels (exp2_poly2 in sm100.cuh).

At d = 128 the forward evaluates a share of the softmax's exponentials with
this polynomial instead of the hardware ex2 unit, so it is a step of the path
with its own error. Pinned here by:
  * the fitting script (Lawson IRLS for minimum maximum relative error)
    reproducing the coefficients written in the kernel source;
  * Chebyshev's alternation theorem: the minimax error of a degree-3 fit
    equioscillates at 5 points, so the source polynomial's relative error on
    [-1/2, 1/2] must peak 5 times with alternating signs and equal size;
  * a float32 emulation of the kernel's exact steps (clamp at -125, the
    1.5*2^23 shifter round, the polynomial as fused multiply-adds, the integer
    exponent insert) against float64 exp2 over every x the softmax can pass
    (-inf up to +8: the running maximum is allowed to lag by 2^8);
  * on the GPU, the device routine against this emulation and against CUDA's
    exp2f on a dense grid.
"""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "reduced_query_head_b200", "csrc")
MAX_REL = 7.5e-5           # stated bound of the polynomial on [-1/2, 1/2]
F32_SLACK = 2.0 ** -23     # the float32 steps after the polynomial (one rounding of p)


def source_coefficients():
    src = open(os.path.join(CSRC, "sm100.cuh")).read()
    body = src[src.index("exp2_poly2"):]
    vals = {}
    for name in ("c0", "c1", "c2", "c3"):
        m = re.search(r"\b%s\s*=\s*([0-9.eE+-]+)f" % name, body)
        assert m, name
        vals[name] = float(m.group(1))
    return np.array([vals["c0"], vals["c1"], vals["c2"], vals["c3"]])


def load_fit():
    spec = importlib.util.spec_from_file_location("_fit_exp2", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _fma32(a, b, c):
    # the product of two float32 values is exact in float64; one add, then round to float32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def emulate(x):
    """The kernel's float32 steps, in numpy float32 arithmetic."""
    c = source_coefficients().astype(np.float32)
    shift = np.float32(12582912.0)                    # 1.5 * 2^23
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = _fma32(f, np.full_like(f, c[3]), np.full_like(f, c[2]))
    p = _fma32(p, f, np.full_like(f, c[1]))
    p = _fma32(p, f, np.full_like(f, c[0]))
    bits = (t.view(np.uint32).astype(np.uint64) * np.uint64(1 << 23) + p.view(np.uint32).astype(np.uint64))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def x_grid():
    """Every region the softmax feeds: dense on [-130, 8], the integer and half-integer
    points where the rounding of n switches, and -inf (a masked score)."""
    dense = np.linspace(-130.0, 8.0, 1_000_003, dtype=np.float64).astype(np.float32)
    k = np.arange(-130, 9, dtype=np.float64)
    edges = np.concatenate([k, k + 0.5, k - 0.5, np.nextafter(k + 0.5, -np.inf), np.nextafter(k + 0.5, np.inf)])
    return np.concatenate([dense, edges.astype(np.float32), np.array([-np.inf, 0.0, -0.0], dtype=np.float32)])


def test_fit_script_reproduces_source_coefficients():
    fit, err = load_fit().fit()
    src = source_coefficients()
    assert np.max(np.abs(fit - src)) <= 2e-6, (fit, src)
    assert err <= MAX_REL


def test_source_polynomial_is_minimax():
    c = source_coefficients()
    f = np.linspace(-0.5, 0.5, 200_001)
    rel = (c[0] + f * (c[1] + f * (c[2] + f * c[3]))) / np.exp2(f) - 1.0
    assert np.max(np.abs(rel)) <= MAX_REL
    # local extrema of the error (interior sign changes of its slope, plus the two ends)
    d = np.diff(rel)
    idx = [0] + [i for i in range(1, len(d)) if np.sign(d[i]) != np.sign(d[i - 1])] + [len(rel) - 1]
    peaks = rel[idx]
    assert len(peaks) == 5, peaks
    assert np.all(np.sign(peaks[1:]) == -np.sign(peaks[:-1])), peaks
    assert np.max(np.abs(peaks)) / np.min(np.abs(peaks)) <= 1.01, peaks


def test_float32_steps_against_exp2():
    x = x_grid()
    got = emulate(x).astype(np.float64)
    want = np.exp2(np.maximum(x.astype(np.float64), -125.0))
    rel = np.abs(got / want - 1.0)
    assert np.all(np.isfinite(got)) and np.all(got > 0)
    assert float(rel.max()) <= MAX_REL + F32_SLACK, float(rel.max())
    # the shifter split is exact: n + f == x, |f| <= 1/2
    xc = np.maximum(x[np.isfinite(x)], np.float32(-125.0))
    t = (xc + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (xc - n).astype(np.float32)
    assert np.array_equal((n.astype(np.float64) + f.astype(np.float64)), xc.astype(np.float64))
    assert float(np.max(np.abs(f))) <= 0.5


def test_masked_score_gives_the_clamp_value():
    got = float(emulate(np.array([-np.inf, -1000.0, -125.0], dtype=np.float32))[0])
    assert got == float(emulate(np.array([-125.0], dtype=np.float32))[0])
    assert abs(got / 2.0 ** -125 - 1.0) <= MAX_REL + F32_SLACK


@pytest.mark.gpu
def test_device_polynomial_against_emulation_and_exp2f():
    import torch
    import reduced_query_head_b200 as sqa
    x = x_grid()
    xd = torch.from_numpy(x).cuda()
    poly = torch.full_like(xd, float("nan"))
    ref = torch.full_like(xd, float("nan"))
    sqa.sqa_check_exp2_poly(xd, poly, ref, x.size)
    torch.cuda.synchronize()
    got = poly.cpu().numpy()
    cuda_exp2 = ref.cpu().numpy().astype(np.float64)
    emu = emulate(x)
    # same steps in the same precision: equal up to the emulation's one double rounding
    ulps = np.abs(got.view(np.int32).astype(np.int64) - emu.view(np.int32).astype(np.int64))
    assert int(ulps.max()) <= 1, int(ulps.max())
    # against CUDA's exp2f where the clamp is not active (exp2f keeps going below 2^-125)
    live = x >= -125.0
    rel = np.abs(got[live].astype(np.float64) / cuda_exp2[live] - 1.0)
    assert float(rel.max()) <= MAX_REL + 2 * F32_SLACK, float(rel.max())
    with pytest.raises(sqa.SqaError):
        sqa.sqa_check_exp2_poly(xd, poly, ref, 0)
