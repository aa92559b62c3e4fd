"""Error budget of the exact-ZOH weight's derivative in A as the backward kernel evaluates
it (CPU, no GPU).

With the weight w = expm1(Delta A) / A (Mamba, "Method": Bbar = (Delta A)^-1
(exp(Delta A) - I) Delta B), dw/dA = Delta^2 psi(y), y = Delta A,
psi(y) = (y e^y - expm1(y)) / y^2 = 1/2 + y/3 + y^2/8 + y^3/30 + ...  The kernel forms it in
fp32 from x = y log2(e): where |y| < 1/2 as Delta^2 times the series truncated after y^7
(Horner in x, coefficients ln2^j times the above), elsewhere as (Delta e - w) / A with
e = 2^x from the SFU and w the weight as the forward forms it (its own switch is at
|y| = 1/16).  This file restates that arithmetic in numpy float32 (each fused multiply-add
rounded once, the SFU's 2^x off by up to 2^-22 relative) and checks psi's relative error
against fp64 over both branches.  Planted mistakes must fail: the switch moved down to the
weight's 1/16, where the closed form cancels, and the series cut after y^3 but kept to 1/2.
"""
import math

import numpy as np
import pytest

LN2 = np.log(2.0)
W_SWITCH = 1.0 / 16.0   # the weight's series / closed-form switch (forward's)
SWITCH = 0.5            # dw/dA's
SFU_REL = 2.0 ** -22
PSI_COEF = [LN2 ** j * (j + 1) / math.factorial(j + 2) for j in range(8)]  # in powers of x
W_COEF = [LN2 ** k / math.factorial(k + 1) for k in range(1, 4)]


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _f32(v):
    return np.float32(v)


def _kernel_dwda_over_delta2(x, delta, switch=SWITCH, sfu_err=0.0, terms=8):
    """dw/dA / Delta^2 (= psi) as the kernel forms it, from fp32 x and Delta."""
    x = x.astype(np.float32)
    delta = np.full_like(x, delta, dtype=np.float32)
    a = (x.astype(np.float64) / np.log2(np.e)).astype(np.float32) / delta  # A with x = Delta A log2 e
    inv_a = (1.0 / a.astype(np.float64)).astype(np.float32)
    e = (np.exp2(x.astype(np.float64)) * (1.0 + sfu_err)).astype(np.float32)
    # the weight as the forward forms it (series in x below the switch, (e - 1) / A above)
    p = _fma32(np.full_like(x, _f32(W_COEF[2])), x, np.full_like(x, _f32(W_COEF[1])))
    p = _fma32(p, x, np.full_like(x, _f32(W_COEF[0])))
    p = _fma32(p, x, np.ones_like(x))
    w_small = (delta * p).astype(np.float32)
    w_large = ((e - np.float32(1.0)) * inv_a).astype(np.float32)
    w = np.where(np.abs(x) < np.float32(W_SWITCH / LN2), w_small, w_large)
    small = np.abs(x) < np.float32(switch / LN2)
    # dw/dA: series (Delta^2 psi, Horner in x) or (Delta e - w) / A
    q = np.full_like(x, _f32(PSI_COEF[terms - 1]))
    for j in range(terms - 2, -1, -1):
        q = _fma32(q, x, np.full_like(x, _f32(PSI_COEF[j])))
    d_small = ((delta * delta).astype(np.float32) * q).astype(np.float32)
    d_large = (((delta * e).astype(np.float32) - w).astype(np.float32) * inv_a).astype(np.float32)
    d = np.where(small, d_small, d_large).astype(np.float64)
    return d / (delta.astype(np.float64) ** 2)


def _psi_exact(x):
    y = x.astype(np.float32).astype(np.float64) * LN2
    out = np.full_like(y, 0.5)
    big = np.abs(y) > 1e-4
    yb = y[big]
    out[big] = (yb * np.exp(yb) - np.expm1(yb)) / (yb * yb)
    ys = y[~big]
    out[~big] = 0.5 + ys / 3 + ys ** 2 / 8 + ys ** 3 / 30
    return out


def _grid():
    return np.concatenate([-np.logspace(-8, np.log10(40.0), 6001),
                           np.logspace(-8, np.log10(8.0), 3001),
                           np.linspace(-0.2, 0.2, 4001)]).astype(np.float32)


@pytest.mark.parametrize("sfu_err", [-SFU_REL, 0.0, SFU_REL])
@pytest.mark.parametrize("delta", [0.003, 0.1, 1.7])
def test_dwda_within_budget_on_both_branches(sfu_err, delta):
    x = _grid()
    x = x[x != 0]
    rel = np.abs(_kernel_dwda_over_delta2(x, delta, sfu_err=sfu_err) / _psi_exact(x) - 1.0)
    assert rel.max() <= 5e-6, rel.max()
    small = np.abs(x.astype(np.float64) * LN2) < SWITCH * 0.999
    assert rel[small].max() <= 1e-6, rel[small].max()


def test_planted_mistake_switch_at_the_weights_fails():
    x = _grid()
    x = x[x != 0]
    rel = np.abs(_kernel_dwda_over_delta2(x, 0.1, switch=W_SWITCH, sfu_err=SFU_REL) /
                 _psi_exact(x) - 1.0)
    assert rel.max() > 5e-5


def test_planted_mistake_short_series_fails():
    x = _grid()
    x = x[x != 0]
    rel = np.abs(_kernel_dwda_over_delta2(x, 0.1, terms=4) / _psi_exact(x) - 1.0)
    assert rel.max() > 1e-4
