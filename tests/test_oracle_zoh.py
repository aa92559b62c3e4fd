"""Pins for the oracle's exact zero-order-hold variant (Bbar = (Delta A)^-1 (exp(Delta A) - I)
Delta B, the "Method" section of "Mamba: Linear-Time Sequence Modeling with Selective State
Spaces").  None of them reuses the oracle's formula:

* the gated-RNN identity of the same paper's discussion of the selection mechanism: with
  N = 1, A = -1, B = C = 1 the ZOH scan is h_t = (1 - g_t) h_{t-1} + g_t u_t with the
  sigmoid gate g_t = sigmoid(delta_t + bias);
* the continuous-time steady state: for constant inputs the state tends to -B u / A
  whatever the step size (the Delta * B reading tends to a Delta-dependent value);
* the solution of the continuous ODE h' = A h + B u with u held over each step, integrated
  numerically (RK4, many substeps) -- zero-order hold is exact for such inputs;
* the small-Delta limit (ZOH and Delta * B agree to first order) and A = 0 (Bbar = Delta B);
* decode steps reproduce the scan;
* planted mistakes in the ZOH weight fail one of these pins.
"""
import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import _mutated_oracle


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def test_gated_rnn_identity():
    rng = np.random.default_rng(11)
    nl, L = 3, 40
    u = rng.standard_normal((nl, L))
    dr = rng.standard_normal((nl, L)) * 2
    bias = rng.uniform(-1, 1, nl)
    ones = np.ones((1, 1, L))
    y, hl = oracle.scan_lanes(u, dr, -np.ones((nl, 1)), ones, ones, np.zeros(nl, dtype=np.int64),
                              delta_bias=bias, softplus=True, zoh=True)
    h = np.zeros(nl)
    for t in range(L):
        g = _sigmoid(dr[:, t] + bias)
        h = (1 - g) * h + g * u[:, t]
        np.testing.assert_allclose(y[:, t], h, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(hl[:, 0], h, rtol=1e-12)


@pytest.mark.parametrize("delta", [0.05, 0.3, 1.7])
def test_steady_state_is_minus_B_u_over_A(delta):
    N, L = 4, 4000
    A = -np.array([[0.5, 1.0, 2.0, 3.5]])
    Bv = np.array([0.7, -1.3, 2.0, 0.4])
    B = np.repeat(Bv[None, :, None], L, axis=2)
    C = np.ones((1, N, L))
    u = np.full((1, L), 1.9)
    dr = np.full((1, L), delta)
    _, hl = oracle.scan_lanes(u, dr, A, B, C, [0], softplus=False, zoh=True)
    np.testing.assert_allclose(hl[0], -Bv * 1.9 / A[0], rtol=1e-12)
    # the Delta * B reading settles elsewhere, and differently for each step size
    _, hl_plain = oracle.scan_lanes(u, dr, A, B, C, [0], softplus=False, zoh=False)
    np.testing.assert_allclose(hl_plain[0], delta * Bv * 1.9 / (1 - np.exp(delta * A[0])),
                               rtol=1e-12)


def _rk4_hold(h, a, b_u, dt, sub=400):
    """Integrate h' = a h + b_u for time dt (b_u constant), RK4 with `sub` substeps."""
    s = dt / sub
    f = lambda x: a * x + b_u  # noqa: E731
    for _ in range(sub):
        k1 = f(h)
        k2 = f(h + 0.5 * s * k1)
        k3 = f(h + 0.5 * s * k2)
        k4 = f(h + s * k3)
        h = h + s / 6 * (k1 + 2 * k2 + 2 * k3 + k4)
    return h


def test_zoh_solves_the_continuous_ode():
    rng = np.random.default_rng(5)
    nl, N, L = 2, 4, 7
    A = rng.uniform(-3.0, 0.5, (nl, N))
    A[0, 1] = 0.0  # pure integrator: h' = B u
    B = rng.standard_normal((1, N, L))
    C = rng.standard_normal((1, N, L))
    u = rng.standard_normal((nl, L))
    dt = rng.uniform(0.05, 0.8, (nl, L))
    _, _, hs = oracle.scan_lanes(u, dt, A, B, C, np.zeros(nl, dtype=np.int64), softplus=False,
                                 zoh=True, return_states=True)
    h = np.zeros((nl, N))
    for t in range(L):
        h = _rk4_hold(h, A, B[0, :, t][None, :] * u[:, t][:, None], dt[:, t][:, None])
        np.testing.assert_allclose(hs[:, t], h, rtol=1e-10, atol=1e-12)


def test_small_delta_limit_and_zero_A():
    rng = np.random.default_rng(8)
    nl, N, L = 2, 3, 20
    A = -rng.uniform(0.5, 4.0, (nl, N))
    B = rng.standard_normal((1, N, L))
    C = rng.standard_normal((1, N, L))
    u = rng.standard_normal((nl, L))
    dt = np.full((nl, L), 1e-6)
    lb = np.zeros(nl, dtype=np.int64)
    _, hz = oracle.scan_lanes(u, dt, A, B, C, lb, softplus=False, zoh=True)
    _, hp = oracle.scan_lanes(u, dt, A, B, C, lb, softplus=False, zoh=False)
    # (e^{Delta a} - 1)/a = Delta (1 + Delta a / 2 + ...): relative gap about Delta |a| / 2
    np.testing.assert_allclose(hz, hp, rtol=1e-5)
    assert not np.allclose(hz, hp, rtol=1e-9, atol=0)
    A0 = np.zeros((nl, N))
    dt = rng.uniform(0.1, 1.0, (nl, L))
    yz, hz = oracle.scan_lanes(u, dt, A0, B, C, lb, softplus=False, zoh=True)
    yp, hp = oracle.scan_lanes(u, dt, A0, B, C, lb, softplus=False, zoh=False)
    np.testing.assert_array_equal(yz, yp)
    np.testing.assert_array_equal(hz, hp)


def test_decode_steps_reproduce_the_zoh_scan():
    rng = np.random.default_rng(21)
    b, d, N, L = 2, 3, 4, 9
    u, dr, z = (rng.standard_normal((b, d, L)) for _ in range(3))
    A = -rng.uniform(0.3, 3.0, (d, N))
    B, C = rng.standard_normal((b, N, L)), rng.standard_normal((b, N, L))
    D, bias = rng.standard_normal(d), rng.uniform(-2, 0, d)
    y, hl = oracle.selective_scan(u, dr, A, B, C, D=D, z=z, delta_bias=bias, zoh=True)
    st = np.zeros((b, d, N))
    for t in range(L):
        st, yt = oracle.state_update(st, u[:, :, t], dr[:, :, t], A, B[:, :, t], C[:, :, t], D=D,
                                     z=z[:, :, t], delta_bias=bias, zoh=True)
        np.testing.assert_allclose(yt, y[:, :, t], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(st, hl, rtol=1e-12, atol=1e-13)


ZOH_MUTATIONS = {
    "missing_division_by_A": ("return expm1(dt * a) / a;", "return expm1(dt * a);"),
    "weight_is_abar_delta": ("return expm1(dt * a) / a;", "return dt * exp(dt * a);"),
    "wrong_sign": ("return expm1(dt * a) / a;", "return expm1(-dt * a) / a;"),
}


def _zoh_pins_pass():
    try:
        test_gated_rnn_identity()
        test_steady_state_is_minus_B_u_over_A(0.3)
        test_zoh_solves_the_continuous_ode()
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("name", sorted(ZOH_MUTATIONS))
def test_planted_zoh_mistake_fails_a_pin(name):
    import os
    src = open(os.path.join(os.path.dirname(oracle.__file__), "s6_oracle.c")).read()
    old, new = ZOH_MUTATIONS[name]
    assert src.count(old) == 1, "mutation anchor not found: " + name
    with _mutated_oracle(src.replace(old, new)):
        assert not _zoh_pins_pass(), "planted mistake survived every pin: " + name
    assert _zoh_pins_pass()
