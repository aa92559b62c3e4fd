"""Pins for the oracle's backward of the causal depthwise conv1d (+ SiLU): the gradients
of sum(out * dout) for x, the weight, the bias and the initial state.  The forward it
differentiates is the Mamba block's convolution step ("Mamba: Linear-Time Sequence
Modeling with Selective State Spaces", Mamba Block); the gradients are the chain rule of
that definition.  None of the pins reuses the oracle's loops:

* central finite differences of the oracle's forward, every entry of every input;
* without SiLU the map is linear, and the gradients have closed forms in numpy: dx is the
  full convolution of dout with the kernel (a correlation), dweight the dot products of
  dout with shifted inputs, dbias the sum of dout;
* the gradients are linear in dout;
* planted mistakes in the oracle's source (a dropped factor of SiLU's derivative, a
  shifted correlation, a shifted initial-state gradient) each fail one of the above.
"""
import os

import numpy as np
import pytest

import oracle


def _problem(seed, b=2, d=2, L=7, K=4, with_init=True, with_bias=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((b, d, L))
    w = rng.standard_normal((d, K))
    bias = rng.standard_normal(d) if with_bias else None
    init = rng.standard_normal((b, d, K - 1)) if (with_init and K > 1) else None
    dout = rng.standard_normal((b, d, L))
    return x, w, bias, init, dout


def _loss(x, w, bias, init, dout, silu):
    out, _ = oracle.causal_conv1d(x, w, bias, initial_state=init, silu=silu)
    return float((out * dout).sum())


def _fd(f, a, h=1e-6):
    g = np.zeros_like(a)
    it = np.nditer(a, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        keep = a[i]
        a[i] = keep + h
        fp = f()
        a[i] = keep - h
        fm = f()
        a[i] = keep
        g[i] = (fp - fm) / (2 * h)
    return g


def _check_fd(K, silu, with_init, with_bias, seed=0):
    x, w, bias, init, dout = _problem(seed + K, K=K, with_init=with_init, with_bias=with_bias)
    g = oracle.causal_conv1d_backward(x, w, dout, bias, init, silu=silu)
    f = lambda: _loss(x, w, bias, init, dout, silu)  # noqa: E731
    np.testing.assert_allclose(g["dx"], _fd(f, x), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(g["dweight"], _fd(f, w), rtol=1e-6, atol=1e-8)
    if bias is not None:
        np.testing.assert_allclose(g["dbias"], _fd(f, bias), rtol=1e-6, atol=1e-8)
    if init is not None:
        np.testing.assert_allclose(g["dinitial_state"], _fd(f, init), rtol=1e-6, atol=1e-8)
    else:
        assert g["dinitial_state"] is None


@pytest.mark.parametrize("K", [1, 2, 3, 4])
@pytest.mark.parametrize("silu", [True, False])
@pytest.mark.parametrize("with_init", [True, False])
def test_backward_matches_central_differences(K, silu, with_init):
    _check_fd(K, silu, with_init, with_bias=True)


def test_backward_without_bias_matches_central_differences():
    _check_fd(3, True, True, with_bias=False)


@pytest.mark.parametrize("K", [1, 2, 3, 4])
def test_linear_case_in_closed_form(K):
    x, w, bias, init, dout = _problem(40 + K, b=2, d=3, L=11, K=K)
    g = oracle.causal_conv1d_backward(x, w, dout, bias, init, silu=False)
    b, d, L = x.shape
    for i in range(b):
        for c in range(d):
            dx = np.convolve(dout[i, c], w[c], mode="full")[K - 1:K - 1 + L]
            np.testing.assert_allclose(g["dx"][i, c], dx, rtol=1e-12, atol=1e-12)
            if K > 1:
                lead = np.convolve(dout[i, c], w[c], mode="full")[:K - 1]
                np.testing.assert_allclose(g["dinitial_state"][i, c], lead, rtol=1e-12, atol=1e-12)
    xe = np.concatenate([init if K > 1 else np.zeros((2, 3, 0)), x], axis=2)
    dw = np.stack([(dout * xe[:, :, k:k + L]).sum(axis=(0, 2)) for k in range(K)], axis=1)
    np.testing.assert_allclose(g["dweight"], dw, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dbias"], dout.sum(axis=(0, 2)), rtol=1e-12, atol=1e-12)


def test_gradients_are_linear_in_dout():
    x, w, bias, init, d1 = _problem(7)
    d2 = np.random.default_rng(8).standard_normal(d1.shape)
    g1 = oracle.causal_conv1d_backward(x, w, d1, bias, init)
    g2 = oracle.causal_conv1d_backward(x, w, d2, bias, init)
    g3 = oracle.causal_conv1d_backward(x, w, 2.5 * d1 + d2, bias, init)
    for k in ("dx", "dweight", "dbias", "dinitial_state"):
        np.testing.assert_allclose(g3[k], 2.5 * g1[k] + g2[k], rtol=1e-12, atol=1e-12)


CONV_BWD_MUTATIONS = {
    "silu_derivative_drops_a_factor": ("d = sg * (1.0 + pre * (1.0 - sg));", "d = sg * (1.0 + pre);"),
    "correlation_off_by_one": ("long t = s + (K - 1) - k;\n", "long t = s + K - k;\n"),
    "initial_state_gradient_shifted": ("dinit[i * (K - 1) + (K - 1) + s] = acc;",
                                       "dinit[i * (K - 1) + (K - 2) + s + (s == -(K - 1))] = acc;"),
}


def _conv_bwd_pins_pass():
    try:
        _check_fd(4, True, True, with_bias=True)
        test_linear_case_in_closed_form(3)
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("name", sorted(CONV_BWD_MUTATIONS))
def test_planted_conv_backward_mistake_fails_a_pin(name):
    from tests.test_oracle_pins import _mutated_oracle
    src = open(os.path.join(os.path.dirname(oracle.__file__), "s6_oracle.c")).read()
    old, new = CONV_BWD_MUTATIONS[name]
    assert src.count(old) == 1, "mutation anchor not found: " + name
    with _mutated_oracle(src.replace(old, new)):
        assert not _conv_bwd_pins_pass(), "planted mistake survived every pin: " + name
    assert _conv_bwd_pins_pass()
