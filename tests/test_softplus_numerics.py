"""Error budget of the kernels' softplus on the CPU (no GPU).

The kernels form softplus(x) = max(x, 0) + log1p(e), e = 2^(-|x| log2 e) in (0, 1], with
log1p(e) = e * q(e) for a degree-7 polynomial q evaluated by fused multiply-adds (the
scalar helper and the packed four-at-a-time one use the same coefficients).  This file
reads the coefficients from the device header, checks that the two copies agree, redoes
the FMA chain in float32 (each step rounded once) and bounds its relative error against
fp64 log1p over (0, 1] -- the 3.3e-7 the kernels' softplus is documented to keep -- and
the resulting softplus against fp64 for x over the range the workloads' steps take.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "selective_state_space_56_b200", "csrc", "s6_device.cuh")
NUM = r"(-?\d+\.\d+e[-+]?\d+)f"


def _coefficients():
    src = open(HEADER).read()
    scalar = src[src.index("float log1p_over_x(float e)"):]
    scalar = scalar[:scalar.index("}")]
    packed = src[src.index("void softplus4("):]
    packed = packed[:packed.index("unpack2(r, out[q], out[q + 1]);")]
    a = [float(v) for v in re.findall(NUM, scalar)]
    b = [float(v) for v in re.findall(NUM, packed)]
    return a, b[::2]  # the packed form repeats each constant for both halves of a pair


def _log1p_over_x32(e, coefs):
    """Horner in the kernels' order: q = c0 e + c1, then q = q e + c_k, each fma rounded once."""
    e64 = e.astype(np.float64)
    q = (np.float64(np.float32(coefs[0])) * e64 + np.float64(np.float32(coefs[1]))).astype(np.float32)
    for c in coefs[2:]:
        q = (q.astype(np.float64) * e64 + np.float64(np.float32(c))).astype(np.float32)
    return q


def test_scalar_and_packed_coefficients_agree():
    a, b = _coefficients()
    assert len(a) == 8 and a == b, (a, b)


def test_log1p_polynomial_error_bound():
    coefs, _ = _coefficients()
    e = np.concatenate([np.logspace(-30, 0, 20001), np.linspace(1e-3, 1.0, 200001)]).astype(np.float32)
    q = _log1p_over_x32(e, coefs)
    approx = (e.astype(np.float64) * q.astype(np.float64)).astype(np.float32).astype(np.float64)
    exact = np.log1p(e.astype(np.float64))
    rel = np.abs(approx / exact - 1.0)
    assert rel.max() <= 3.3e-7 + 1.2e-7, rel.max()  # fit error plus one fp32 rounding


def test_softplus_error_on_the_step_range():
    coefs, _ = _coefficients()
    x = np.linspace(-30.0, 30.0, 600001).astype(np.float32)
    e = np.exp2(-np.abs(x.astype(np.float64)) * np.log2(np.e)).astype(np.float32)
    q = _log1p_over_x32(e, coefs)
    lp = (e.astype(np.float64) * q.astype(np.float64)).astype(np.float32)
    sp = (np.maximum(x, np.float32(0)).astype(np.float64) + lp.astype(np.float64)).astype(np.float32)
    exact = np.logaddexp(0.0, x.astype(np.float64))
    rel = np.abs(sp.astype(np.float64) / exact - 1.0)
    assert rel.max() <= 1e-6, rel.max()
