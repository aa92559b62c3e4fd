"""Tolerances for comparing the CUDA path with the fp64 oracle.

* fp32 inputs and output: per element |y - y_ref| <= 1e-4 * max(1, |y_ref|).
* bf16 inputs, fp32 output (isolates the kernel's arithmetic from output
  rounding): max |y - y_ref| <= 2e-2 * RMS(y_ref).
* bf16 output: per element |y - y_ref| <= 2e-2 * RMS(y_ref) + ulp_bf16(|y_ref|).
  Rounding an exact result to bf16 alone moves it by up to half a bf16 ulp
  (|y|/512), which for the heavy-tailed y of these workloads (max|y| ~ 50 RMS)
  exceeds 2e-2 RMS, so the plain bound cannot hold for any bf16 output; one ulp
  of slack at each element covers the rounding and one tie flip.
* fp32 state (last_state, decode state) after bf16 inputs: max |s - s_ref| <=
  2e-2 * RMS(s_ref); after fp32 inputs: the fp32 rule above.
The oracle always runs on the exact values the kernel read (bf16 inputs
widened without rounding).
"""
import numpy as np
import torch


def to64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def rms(x):
    x = np.asarray(x, dtype=np.float64)
    return float(np.sqrt(np.mean(x * x))) if x.size else 0.0


def ulp_bf16(x):
    ax = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


def check_fp32(got, ref, what="y", rel=1e-4):
    got, ref = to64(got), to64(ref)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    bound = rel * np.maximum(1.0, np.abs(ref))
    err = np.abs(got - ref)
    bad = err > bound
    assert not bad.any(), "%s: %d/%d elements beyond 1e-4*max(1,|ref|); worst %.3g at %s" % (
        what, int(bad.sum()), bad.size, float((err / bound).max()),
        np.unravel_index(int(np.argmax(err / bound)), err.shape))
    return float((err / bound).max()) if err.size else 0.0


def check_rms(got, ref, what="y", frac=2e-2, scale=None):
    got, ref = to64(got), to64(ref)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    r = rms(ref) if scale is None else scale
    err = float(np.abs(got - ref).max()) if got.size else 0.0
    assert err <= frac * r, "%s: max|err| %.4g > %.3g * RMS %.4g" % (what, err, frac, r)
    return err / r if r else 0.0


def check_bf16_out(got, ref, what="y", frac=2e-2, scale=None):
    """Per element: |y - ref| <= frac*RMS(ref) + ulp_bf16(|ref|).  Returns statistics."""
    got, ref = to64(got), to64(ref)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    r = rms(ref) if scale is None else scale
    err = np.abs(got - ref)
    bound = frac * r + ulp_bf16(ref)
    bad = err > bound
    assert not bad.any(), "%s: %d/%d elements beyond 2e-2*RMS + ulp; worst excess %.3g" % (
        what, int(bad.sum()), bad.size, float((err - bound).max()))
    literal = err > frac * r
    return dict(max_err_over_rms=float(err.max() / r) if r else 0.0,
                n_over_literal=int(literal.sum()), n=int(err.size))
