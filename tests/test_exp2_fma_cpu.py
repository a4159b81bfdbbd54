"""The FMA-pipe exponential of the tcgen05 softmax (exp2_fma2 in
sm100_ptx.cuh), emulated step by step in float32 on the CPU: its polynomial
is the minimax fit that exp2_poly_fit.py computes, its error stays within
that fit's bound against 2^x in float64, and clamped arguments give exactly
zero.  (The GPU parity tests check it inside the kernels.)"""
import importlib.util
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "attention_forward_20_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", os.path.join(CSRC, "exp2_poly_fit.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_coefficients():
    src = open(os.path.join(CSRC, "sm100_ptx.cuh")).read()
    m = re.search(r"c1 = ([0-9.eE+-]+)f, c2 = ([0-9.eE+-]+)f, c3 = ([0-9.eE+-]+)f", src)
    assert m, "coefficients not found in exp2_fma2"
    return [np.float32(float(g)) for g in m.groups()]


def emulate(x):
    """exp2_fma2 on float32 inputs, one step per device instruction."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-127.0))       # fmaxf
    shifter = np.float32(12582912.0)
    t = (shifter + np.floor(x.astype(np.float64))).astype(np.float32)          # add.rm: exact for |x| < 2^22
    j = (t - shifter).astype(np.float32)                                        # exact
    f = (x - j).astype(np.float32)                                              # exact
    c1, c2, c3 = _header_coefficients()
    fma = lambda a, b, c: (a.astype(np.float64) * b + c).astype(np.float32)    # noqa: E731 (single rounding)
    p = fma(f, c3, c2)
    p = fma(p, f, c1)
    p = fma(p, f, np.float32(1.0))
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_coefficients_are_the_minimax_fit():
    c, err = _fit_module().fit()
    assert err < 8.6e-5
    assert _header_coefficients() == [np.float32(v) for v in c]


def test_relative_error_within_the_fit_bound():
    x = np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float32)
    y = emulate(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 8.7e-5
    # integer arguments land on exact powers of two (p(0) = 1)
    k = np.arange(-126, 9, dtype=np.float32)
    assert np.array_equal(emulate(k), np.exp2(k.astype(np.float64)).astype(np.float32))


def test_clamped_arguments_give_zero():
    for v in (-127.0, -127.5, -200.0, -1e30, -np.inf):
        assert emulate(np.array([v]))[0] == 0.0
