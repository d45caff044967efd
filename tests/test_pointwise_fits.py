"""The kernels' pointwise approximations (csrc/pointwise.cuh).

CPU: the polynomial constants in pointwise.cuh are what csrc/fit_poly.py
derives (least-squares fits re-run here), and their float32 Horner evaluation
stays within the stated bounds (log(1 + e)/e on [0, 1]: 1.7e-7 relative;
2^f on [-0.5, 0.5]: 9.7e-8).

GPU: every function, evaluated by the device code the scans run, against
float64 over its whole input range.  The bounds follow from the parts: the
special-function unit's ex2 and rcp (relative error near 2^-22), the
polynomial fits above, and the rounding of the exponent argument -|x| log2(e),
an absolute error of about |x| 2^-24 in the exponent, i.e. a relative error
growing like 1e-7 |x| in e^-|x|.
"""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "selective_state_space_ss_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_poly", os.path.join(CSRC, "fit_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _header_constants(func_name):
    """The float literals of one function in pointwise.cuh, in source order."""
    text = open(os.path.join(CSRC, "pointwise.cuh")).read()
    start = text.index(func_name + "(")
    body = text[start:text.index("\n}\n", start)]
    return [float(v) for v in re.findall(r"(-?\d+\.\d+e[-+]\d+)f", body)]


def test_log1p_constants_match_the_fit():
    fp = _fit_module()
    c = fp.log1p_over_coeffs()  # increasing degree
    hdr = _header_constants("log1p_unit")  # Horner order: highest degree first
    assert len(hdr) == len(c) == 9
    np.testing.assert_array_equal(np.float32(hdr[::-1]), c)
    f = lambda e: np.where(e == 0, 1.0, np.log1p(e) / np.where(e == 0, 1.0, e))  # noqa: E731
    assert fp.max_rel_err(c, f, 0.0, 1.0) <= 1.7e-7


def test_packed_log1p_uses_the_same_constants():
    a = _header_constants("log1p_unit")
    b = _header_constants("log1p_unit2")
    # the packed form writes each constant twice (both halves of a pair)
    assert b[::2] == a and b[1::2] == a


def test_exp2_constants_match_the_fit():
    fp = _fit_module()
    c = fp.exp2_frac_coeffs()
    # the degree-6..1 literals come in pairs (packed); the constant term is
    # written 1.f, which is what the fit rounds to
    hdr = _header_constants("exp2_neg_fma2")[::2]
    assert len(hdr) == 6 and c[0] == np.float32(1.0)
    np.testing.assert_array_equal(np.float32(hdr[::-1]), c[1:])
    assert fp.max_rel_err(c, np.exp2, -0.5, 0.5) <= 9.7e-8


def test_rcp_seed_and_newton_steps():
    # seed 24/17 - 8/17 d has relative error <= 1/17 on [1, 2]; each Newton
    # step squares it: three steps reach (1/17)^8 ~ 1.4e-10, below fp32 rounding
    d = np.linspace(1.0, 2.0, 100001)
    r = 24.0 / 17.0 - 8.0 / 17.0 * d
    assert np.max(np.abs(1.0 - d * r)) <= 1.0 / 17.0 + 1e-15
    for _ in range(3):
        r = r + r * (1.0 - d * r)
    assert np.max(np.abs(1.0 - d * r)) <= 1.5e-10


# ------------------------------------------------------------------ GPU ----

def _gpu_eval(fn, x):
    import torch

    import selective_state_space_ss_b200 as ss

    y = ss._native.ss_debug_pointwise(fn, torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda())
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def _softplus64(x):
    return np.where(x > 30, x + np.log1p(np.exp(-np.abs(x))), np.log1p(np.exp(np.minimum(x, 30))))


def _silu64(x):
    return x / (1.0 + np.exp(-x))


def _grid(lo, hi, n=400001):
    x = np.linspace(lo, hi, n).astype(np.float32)
    return np.concatenate([x, np.float32([0.0, -0.0, lo, hi, 1e-30, -1e-30])])


@pytest.mark.gpu
@pytest.mark.parametrize("packed", [False, True])
def test_softplus_on_device(packed):
    from selective_state_space_ss_b200 import _native as N

    x = _grid(-100.0, 100.0)
    got = _gpu_eval(N.SS_PW_SOFTPLUS2 if packed else N.SS_PW_SOFTPLUS, x)
    ref = _softplus64(x.astype(np.float64))
    rel = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-300)
    # below e^-87 the flush-to-zero 2^x underflows: softplus(x) is then 0 or subnormal
    keep = x > -86.0
    bound = 6e-7 + 1.2e-7 * np.abs(x[keep].astype(np.float64))
    assert np.all(rel[keep] <= bound), float(np.max(rel[keep] / bound))
    assert np.all(np.abs(got[~keep]) <= 1e-37)


@pytest.mark.gpu
@pytest.mark.parametrize("packed", [False, True])
def test_silu_on_device(packed):
    from selective_state_space_ss_b200 import _native as N

    x = _grid(-100.0, 100.0)
    got = _gpu_eval(N.SS_PW_SILU2 if packed else N.SS_PW_SILU, x)
    ref = _silu64(x.astype(np.float64))
    keep = x > -86.0
    rel = np.abs(got[keep] - ref[keep]) / np.maximum(np.abs(ref[keep]), 1e-300)
    bound = 6e-7 + 1.2e-7 * np.abs(x[keep].astype(np.float64))
    assert np.all(rel <= bound), float(np.max(rel / bound))
    assert np.all(np.abs(got[~keep]) <= 1e-35)


@pytest.mark.gpu
def test_exp2_on_the_fma_pipe():
    from selective_state_space_ss_b200 import _native as N

    x = _grid(-125.0, 0.0)
    got = _gpu_eval(N.SS_PW_EXP2_NEG_FMA, x)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert np.max(rel) <= 3e-7, float(np.max(rel))
    # at and below -126 the result stands for 0: 2^-126 at most
    got_low = _gpu_eval(N.SS_PW_EXP2_NEG_FMA, np.float32([-126.0, -127.5, -300.0, -1e30]))
    assert np.all(got_low <= 2.0 ** -126 * 1.000001) and np.all(got_low >= 0)


@pytest.mark.gpu
def test_reciprocal_on_the_fma_pipe():
    from selective_state_space_ss_b200 import _native as N

    d = _grid(1.0, 2.0)
    d = d[(d >= 1.0) & (d <= 2.0)]
    got = _gpu_eval(N.SS_PW_RCP_1_2, d)
    rel = np.abs(got * d.astype(np.float64) - 1.0)
    assert np.max(rel) <= 2.5e-7, float(np.max(rel))


@pytest.mark.gpu
def test_special_function_unit_ex2():
    """The MUFU 2^x the recurrence uses: relative error near 2^-22 over the
    exponent range the decays take, flushing to zero below -126."""
    from selective_state_space_ss_b200 import _native as N

    x = _grid(-125.0, 0.0)
    got = _gpu_eval(N.SS_PW_EX2, x)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got - ref) / ref) <= 2.0 ** -21
