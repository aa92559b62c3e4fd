"""Pins for the oracle's backward: central finite differences of the forward oracle.

The loss is sum(y * dy) for a fixed random dy; every gradient entry the backward
returns (du, ddelta, dz, dA, dD, dbias, dB, dC) is compared with
(loss(x + eps) - loss(x - eps)) / (2 eps) computed from the forward oracle alone,
on tiny inputs in fp64.  The forward is itself pinned in test_oracle_pins.py.
"""
import numpy as np
import pytest

import oracle


def _problem(seed, b=2, d=3, N=3, L=7):
    rng = np.random.default_rng(seed)
    return dict(u=rng.standard_normal((b, d, L)), delta=rng.standard_normal((b, d, L)),
                A=-rng.uniform(0.3, 2.0, (d, N)), B=rng.standard_normal((b, N, L)),
                C=rng.standard_normal((b, N, L)), D=rng.standard_normal(d),
                z=rng.standard_normal((b, d, L)), delta_bias=rng.uniform(-2, 0.5, d)), \
        rng.standard_normal((b, d, L))


def _loss(p, dy, softplus):
    y, _ = oracle.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                                 delta_bias=p["delta_bias"], softplus=softplus)
    return float((y * dy).sum())


GRAD_OF = {"u": "du", "delta": "ddelta", "z": "dz", "A": "dA", "D": "dD",
           "delta_bias": "dbias", "B": "dB", "C": "dC"}


@pytest.mark.parametrize("variant", ["full", "no_softplus", "no_gate", "no_skip_no_bias"])
def test_backward_matches_finite_differences(variant):
    p, dy = _problem(seed=sum(map(ord, variant)))
    softplus = variant != "no_softplus"
    if variant == "no_softplus":
        p["delta"] = np.abs(p["delta"]) * 0.3 + 0.05   # keep steps positive
        p["delta_bias"] = np.full_like(p["delta_bias"], 0.02)
    if variant == "no_gate":
        p["z"] = None
    if variant == "no_skip_no_bias":
        p["D"] = None
        p["delta_bias"] = None
    g = oracle.selective_scan_backward(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"],
                                       z=p["z"], delta_bias=p["delta_bias"], softplus=softplus)
    eps = 1e-6
    for name, gname in GRAD_OF.items():
        if p.get(name) is None:
            continue
        base = p[name]
        num = np.empty_like(base)
        for idx in np.ndindex(base.shape):
            keep = base[idx]
            base[idx] = keep + eps
            lp = _loss(p, dy, softplus)
            base[idx] = keep - eps
            lm = _loss(p, dy, softplus)
            base[idx] = keep
            num[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(g[gname], num, rtol=1e-6, atol=1e-7, err_msg=gname)
    if p["z"] is None:
        assert np.all(g["dz"] == 0)


def test_backward_of_linear_readout_is_the_forward_state():
    """With C = 1 on one state, no skip and no gate, dC_t equals dy_t h_t summed over
    channels -- checked against the forward oracle's own states."""
    p, dy = _problem(seed=3, b=1, d=2, N=1, L=5)
    p["z"] = None
    p["D"] = None
    _, _, h = oracle.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=None, z=None,
                                    delta_bias=p["delta_bias"], return_states=True)
    g = oracle.selective_scan_backward(p["u"], p["delta"], p["A"], p["B"], p["C"], dy,
                                       delta_bias=p["delta_bias"])
    np.testing.assert_allclose(g["dC"][0, 0], (dy[0] * h[0, :, :, 0]).sum(0), rtol=1e-12)
