"""The exp2 cubic that prefill attention evaluates on the FMA pipes
(``exp2_poly2`` in csrc/ptx.cuh): its fp32 coefficients are the Remez fit that
gated_mla_b200/fit_exp2_poly.py prints, and the whole kernel sequence (range
reduction by the 1.5 * 2^23 shift, fp32 Horner steps, exponent add), emulated
bit for bit in numpy, stays within the 7.5e-5 relative error the comment
states, against numpy's exp2 in fp64."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PTX = os.path.join(ROOT, "gated_mla_b200", "csrc", "ptx.cuh")
BOUND = 7.5e-5


def kernel_coefficients():
    src = open(PTX).read()
    body = src[src.index("void exp2_poly2"):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body)]
    # order in the Horner chain: c3, c2, c1, c0
    assert len(vals) == 4, vals
    c3, c2, c1, c0 = vals
    return c0, c1, c2, c3


def fma32(a, b, c):
    # an fp32 fused multiply-add: the fp64 product of two fp32 values is exact,
    # the sum is rounded once to fp64 and then to fp32 (a double rounding that
    # can only move the result by one fp32 ulp, far inside the bound)
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def kernel_exp2(x):
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n_f = (t - magic).astype(np.float32)
    f = (x - n_f).astype(np.float32)
    c0, c1, c2, c3 = (np.full_like(x, v) for v in kernel_coefficients())
    p = fma32(c3, f, c2)
    p = fma32(p, f, c1)
    p = fma32(p, f, c0)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23)))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_coefficients_are_the_remez_fit():
    spec = importlib.util.spec_from_file_location("fit", os.path.join(ROOT, "gated_mla_b200", "fit_exp2_poly.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c, E = fit.remez_relative()
    assert E < BOUND
    for got, want in zip(kernel_coefficients(), c):
        assert np.float32(got) == np.float32(want), (got, want)


def test_relative_error_within_the_stated_bound():
    rng = np.random.default_rng(0)
    xs = np.concatenate([
        np.linspace(-0.5, 0.5, 400001),                       # the reduced interval itself
        np.linspace(-30.0, 0.0, 600001),                      # the softmax range (x = s - m <= 0)
        rng.uniform(-124.0, 20.0, 400000),
        np.arange(-124, 21, dtype=np.float64) + 0.5,          # ties of the rounding to nearest
    ]).astype(np.float32)
    got = kernel_exp2(xs).astype(np.float64)
    ref = np.exp2(xs.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() <= BOUND, rel.max()
    # the bound is nearly attained, so the stated figure is the fit's, not a loose one
    assert rel.max() > 0.9 * BOUND


def test_clamp_below_minus_125():
    y = kernel_exp2(np.array([-200.0, -125.0], np.float32)).astype(np.float64)
    assert np.all(np.abs(y / 2.0 ** -125 - 1.0) <= BOUND)
