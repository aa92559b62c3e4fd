"""Pins for the oracle's backward: central finite differences of the forward oracle
(with the Delta * B input weight and with the exact ZOH weight).

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


def _loss(p, dy, softplus, zoh=False):
    y, _ = oracle.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                                 delta_bias=p["delta_bias"], softplus=softplus, zoh=zoh)
    return float((y * dy).sum())


GRAD_OF = {"u": "du", "delta": "ddelta", "z": "dz", "A": "dA", "D": "dD",
           "delta_bias": "dbias", "B": "dB", "C": "dC"}


@pytest.mark.parametrize("variant", ["full", "no_softplus", "no_gate", "no_skip_no_bias",
                                     "zoh", "zoh_small_and_zero_a", "zoh_no_softplus"])
def test_backward_matches_finite_differences(variant):
    """The exact-ZOH variants ("Mamba: Linear-Time Sequence Modeling with Selective State
    Spaces", Method: Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B) differentiate the ZOH
    forward; one of them puts A at 0, at +-1e-5 (the series side of dw/dA), and positive."""
    p, dy = _problem(seed=sum(map(ord, variant)))
    softplus = variant not in ("no_softplus", "zoh_no_softplus")
    zoh = variant.startswith("zoh")
    if variant == "zoh_small_and_zero_a":
        p["A"][0, 0] = 0.0
        p["A"][1, 1] = -1e-5
        p["A"][2, 2] = 1e-5
        p["A"][0, 2] = 0.4
    if variant in ("no_softplus", "zoh_no_softplus"):
        p["delta"] = np.abs(p["delta"]) * 0.3 + 0.05   # keep steps positive
        p["delta_bias"] = np.full_like(p["delta_bias"], 0.02)
    if variant == "no_gate":
        p["z"] = None
    if variant == "no_skip_no_bias":
        p["D"] = None
        p["delta_bias"] = None
    g = oracle.selective_scan_backward(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"],
                                       z=p["z"], delta_bias=p["delta_bias"], softplus=softplus,
                                       zoh=zoh)
    eps = 1e-6
    for name, gname in GRAD_OF.items():
        if p.get(name) is None:
            continue
        base = p[name]
        num = np.empty_like(base)
        for idx in np.ndindex(base.shape):
            keep = base[idx]
            base[idx] = keep + eps
            lp = _loss(p, dy, softplus, zoh)
            base[idx] = keep - eps
            lm = _loss(p, dy, softplus, zoh)
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


ZOH_BWD_MUTATIONS = {
    "weight_derivative_in_delta_is_one": ("ddt += gb * ut * abar;", "ddt += gb * ut;"),
    "psi_series_constant": ("return 0.5 + y * (1.0 / 3.0", "return 0.4 + y * (1.0 / 3.0"),
    "psi_closed_form_sign": ("return (y * exp(y) - expm1(y)) / (y * y);",
                             "return (y * exp(y) + expm1(y)) / (y * y);"),
    "du_uses_delta_not_weight": ("duw += gb * w;", "duw += gb * dt;"),
}


def _zoh_bwd_pins_pass():
    try:
        test_backward_matches_finite_differences("zoh")
        test_backward_matches_finite_differences("zoh_small_and_zero_a")
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("name", sorted(ZOH_BWD_MUTATIONS))
def test_planted_zoh_backward_mistake_fails_a_pin(name):
    import os
    from tests.test_oracle_pins import _mutated_oracle
    src = open(os.path.join(os.path.dirname(oracle.__file__), "s6_oracle.c")).read()
    old, new = ZOH_BWD_MUTATIONS[name]
    assert src.count(old) == 1, "mutation anchor not found: " + name
    with _mutated_oracle(src.replace(old, new)):
        assert not _zoh_bwd_pins_pass(), "planted mistake survived every pin: " + name
    assert _zoh_bwd_pins_pass()
