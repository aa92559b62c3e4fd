"""Error budget of the exact-ZOH input weight as the kernels evaluate it (CPU, no GPU).

The weight (Mamba, "Method": per diagonal state Bbar_n = (exp(Delta A_n) - 1) / A_n B_n)
is formed in fp32 from x = Delta A log2(e): where |x| is below the switch point
(|Delta A| = 1/16) as Delta * phi(y), phi(y) = expm1(y) / y = sum_k y^k / (k+1)!
truncated after y^3 and evaluated by Horner's rule in x with coefficients
ln2^k / (k+1)!; elsewhere as (e - 1) / A with e = 2^x from the SFU.  This file
restates that arithmetic in numpy float32 -- every fused multiply-add rounded once,
the SFU's 2^x modelled as the exact value off by up to 2^-22 relative either way --
and checks the relative error of phi against fp64 expm1(y) / y over both branches.  A
planted mistake (the same three-term series kept up to |Delta A| = 1/2) must fail.
"""
import math

import numpy as np
import pytest

LN2 = np.log(2.0)
COEF = [LN2 ** k / math.factorial(k + 1) for k in range(1, 4)]  # c1, c2, c3
SWITCH = 1.0 / 16.0  # |Delta A| where the direct form takes over
SFU_REL = 2.0 ** -22


def _fma32(a, b, c):
    """fp32 fused multiply-add: the product and sum exact in fp64, rounded once."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _phi_kernel(x, switch=SWITCH, sfu_err=0.0):
    """phi(Delta A) as the kernels form it, from x = Delta A log2(e) (fp32)."""
    x = x.astype(np.float32)
    c1, c2, c3 = (np.full_like(x, c, dtype=np.float32) for c in COEF)
    p = _fma32(c3, x, c2)
    p = _fma32(p, x, c1)
    small = _fma32(p, x, np.ones_like(x))
    e = (np.exp2(x.astype(np.float64)) * (1.0 + sfu_err)).astype(np.float32)
    y = (x.astype(np.float64) * LN2)
    # the direct branch divides (e - 1) by A; as a factor of Delta that is (e - 1) / y
    with np.errstate(divide="ignore", invalid="ignore"):  # y = 0 takes the series
        large = (e - np.float32(1.0)).astype(np.float64) / y
    use_small = np.abs(x) < np.float32(switch / LN2)
    return np.where(use_small, small.astype(np.float64), large)


def _phi_exact(x):
    y = x.astype(np.float32).astype(np.float64) * LN2
    out = np.ones_like(y)
    nz = y != 0
    out[nz] = np.expm1(y[nz]) / y[nz]
    return out


def _grid():
    return np.concatenate([
        -np.logspace(-12, np.log10(60.0), 20001), np.logspace(-12, np.log10(12.0), 8001),
        np.linspace(-0.2, 0.2, 8001), [0.0]]).astype(np.float32)


@pytest.mark.parametrize("sfu_err", [-SFU_REL, 0.0, SFU_REL])
def test_weight_within_a_few_millionths_on_both_branches(sfu_err):
    x = _grid()
    rel = np.abs(_phi_kernel(x, sfu_err=sfu_err) / _phi_exact(x) - 1.0)
    assert rel.max() <= 5e-6, rel.max()
    # below the switch point only the truncation (< 1.3e-7) and fp32 rounding remain
    small = np.abs(x.astype(np.float64) * LN2) < SWITCH * 0.999
    assert rel[small].max() <= 5e-7, rel[small].max()


def test_planted_mistake_late_switch_fails():
    x = _grid()
    rel = np.abs(_phi_kernel(x, switch=0.5) / _phi_exact(x) - 1.0)
    assert rel.max() > 1e-4  # three terms are far too few out to |Delta A| = 1/2
