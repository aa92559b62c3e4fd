"""Error budget of the kernels' four-at-a-time SiLU on the CPU (no GPU).

The scan's output gate forms z * sigmoid(z) for four steps with one reciprocal between
them: d_q = 1 + 2^min(-z_q log2 e, 31), r = 1 / ((d0 d1)(d2 d3)), then
1/d0 = (r d2d3) d1, 1/d1 = (r d2d3) d0, 1/d2 = (r d0d1) d3, 1/d3 = (r d0d1) d2 and
out_q = z_q (1/d_q).  This file redoes that arithmetic in float32 (every operation rounded
once; the exponential and the reciprocal given the relative error their hardware
instructions are documented to stay within, 2^-22 and 2^-23, in the worst direction)
and bounds its error against fp64 z * sigmoid(z) wherever sigmoid(z) is above 2^-31 by
6e-7 + 1.2e-7 |z| relative -- the second term is the conditioning of 2^x for a rounded
argument x = -z log2 e (|dx| <= 2^-23 |x|), which the one-division form shares -- and
below that, where the cap takes over, by an absolute 5e-10 |z|.  The one-division form
z * (1 / (1 + e)) is checked against the same budget for comparison.
"""
import itertools

import numpy as np

F = np.float32


def _r(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def _silu4(z, ex2_err, rcp_err):
    """The kernel's sequence for z of shape (4, n) in float32, with relative perturbations
    ex2_err and rcp_err applied to the SFU results."""
    x = np.minimum(_r(-z.astype(np.float64) * np.float64(F(1.4426950408889634))), F(31.0))
    e = _r(np.exp2(x.astype(np.float64)) * (1.0 + ex2_err))
    d = _r(1.0 + e.astype(np.float64))
    p01 = _r(d[0].astype(np.float64) * d[1])
    p23 = _r(d[2].astype(np.float64) * d[3])
    p = _r(p01.astype(np.float64) * p23)
    r = _r((1.0 / p.astype(np.float64)) * (1.0 + rcp_err))
    r01 = _r(r.astype(np.float64) * p23)
    r23 = _r(r.astype(np.float64) * p01)
    inv = [_r(r01.astype(np.float64) * d[1]), _r(r01.astype(np.float64) * d[0]),
           _r(r23.astype(np.float64) * d[3]), _r(r23.astype(np.float64) * d[2])]
    return np.stack([_r(z[q].astype(np.float64) * inv[q]) for q in range(4)])


def _exact(z):
    z = z.astype(np.float64)
    return z / (1.0 + np.exp(-z))


def test_silu4_error_budget():
    rng = np.random.default_rng(7)
    zs = [rng.standard_normal((4, 200000)),                 # the workloads' gate values
          rng.uniform(-40.0, 40.0, (4, 200000)),            # far tails, cap engaged
          np.tile(np.linspace(-25.0, 25.0, 50001), (4, 1))]
    for z, ex2_err, rcp_err in itertools.product(zs, (-2.0 ** -22, 2.0 ** -22), (-2.0 ** -23, 2.0 ** -23)):
        z = z.astype(np.float32)
        got = _silu4(z, ex2_err, rcp_err).astype(np.float64)
        ref = _exact(z)
        sig = 1.0 / (1.0 + np.exp(-z.astype(np.float64)))
        normal = sig > 2.0 ** -31
        budget = 6e-7 + 1.2e-7 * np.abs(z.astype(np.float64))
        rel = np.abs(got - ref) / np.abs(ref).clip(1e-300)
        assert (rel[normal] <= budget[normal]).all(), (rel / budget)[normal].max()
        # the one-division form on the same inputs and perturbations
        x = np.minimum(_r(-z.astype(np.float64) * np.float64(F(1.4426950408889634))), F(31.0))
        e = _r(np.exp2(x.astype(np.float64)) * (1.0 + ex2_err))
        one = _r(z.astype(np.float64) * _r((1.0 / _r(1.0 + e.astype(np.float64)).astype(np.float64))
                                           * (1.0 + rcp_err)))
        rel1 = np.abs(one.astype(np.float64) - ref) / np.abs(ref).clip(1e-300)
        assert (rel1[normal] <= budget[normal]).all()
        absd = np.abs(got - ref)[~normal] / np.abs(z[~normal].astype(np.float64))
        assert absd.size == 0 or absd.max() <= 5e-10, absd.max()


def test_silu4_products_stay_finite():
    # every factor is at most 2^31 + 1, so the product of four is below 2^125
    z = np.full((4, 8), -1000.0, dtype=np.float32)
    got = _silu4(z, 2.0 ** -22, 2.0 ** -23)
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got) <= 1000.0 * 2.0 ** -30)
