"""Pins for the oracle's causal depthwise conv1d (+ SiLU), the Mamba block's step before the
SSM ("Mamba" Q&A on the convolution before the SSM; "Mamba: Linear-Time Sequence Modeling
with Selective State Spaces", Mamba Block).  None reuses the oracle's loop:

* numpy's full convolution with the reversed kernel, truncated to the first L outputs;
* the impulse response is the reversed kernel, placed causally;
* causality: changing an input never changes an earlier output;
* chunked prefill (the second chunk starting from the first chunk's final state) equals
  one pass, and decode steps reproduce the prefill outputs and final state;
* the SiLU is x * sigmoid(x) (checked against numpy), and is off when asked.
"""
import numpy as np
import pytest

import oracle


def _sig(x):
    return 1.0 / (1.0 + np.exp(-x))


@pytest.mark.parametrize("K", [1, 2, 3, 4])
def test_matches_numpy_convolution(K):
    rng = np.random.default_rng(K)
    b, d, L = 2, 3, 37
    x = rng.standard_normal((b, d, L))
    w = rng.standard_normal((d, K))
    bias = rng.standard_normal(d)
    out, fin = oracle.causal_conv1d(x, w, bias, silu=False)
    outs, _ = oracle.causal_conv1d(x, w, bias, silu=True)
    for i in range(b):
        for c in range(d):
            ref = np.convolve(x[i, c], w[c, ::-1], mode="full")[:L] + bias[c]
            np.testing.assert_allclose(out[i, c], ref, rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(outs[i, c], ref * _sig(ref), rtol=1e-13, atol=1e-13)
            if K > 1:
                np.testing.assert_array_equal(fin[i, c], x[i, c, L - (K - 1):])


def test_impulse_response_is_the_reversed_kernel():
    K, L, t0 = 4, 12, 5
    w = np.array([[0.5, -1.0, 2.0, 3.0]])
    x = np.zeros((1, 1, L))
    x[0, 0, t0] = 1.0
    out, _ = oracle.causal_conv1d(x, w, silu=False)
    expect = np.zeros(L)
    expect[t0:t0 + K] = w[0, ::-1]
    np.testing.assert_array_equal(out[0, 0], expect)


def test_causality():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((1, 2, 30))
    w = rng.standard_normal((2, 4))
    base, _ = oracle.causal_conv1d(x, w, silu=True)
    for t in (0, 7, 29):
        x2 = x.copy()
        x2[:, :, t] += 5.0
        out, _ = oracle.causal_conv1d(x2, w, silu=True)
        np.testing.assert_array_equal(out[:, :, :t], base[:, :, :t])
        assert np.all(out[:, :, t] != base[:, :, t])


@pytest.mark.parametrize("split", [1, 2, 3, 10])
def test_chunked_prefill_and_decode(split):
    rng = np.random.default_rng(10 + split)
    b, d, L, K = 2, 3, 14, 4
    x = rng.standard_normal((b, d, L))
    w = rng.standard_normal((d, K))
    bias = rng.standard_normal(d)
    init = rng.standard_normal((b, d, K - 1))
    out, fin = oracle.causal_conv1d(x, w, bias, initial_state=init)
    o1, f1 = oracle.causal_conv1d(x[:, :, :split], w, bias, initial_state=init)
    o2, f2 = oracle.causal_conv1d(x[:, :, split:], w, bias, initial_state=f1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=2), out, rtol=1e-14, atol=1e-14)
    np.testing.assert_array_equal(f2, fin)
    st = init
    for t in range(L):
        st, o = oracle.causal_conv1d_update(st, x[:, :, t], w, bias)
        np.testing.assert_allclose(o, out[:, :, t], rtol=1e-14, atol=1e-14)
    np.testing.assert_array_equal(st, fin)


def test_short_sequence_final_state_keeps_the_initial_inputs():
    init = np.array([[[1.0, 2.0, 3.0]]])
    x = np.array([[[4.0]]])
    _, fin = oracle.causal_conv1d(x, np.ones((1, 4)), initial_state=init, silu=False)
    np.testing.assert_array_equal(fin, [[[2.0, 3.0, 4.0]]])
    _, fin0 = oracle.causal_conv1d(np.zeros((1, 1, 0)), np.ones((1, 4)), initial_state=init)
    np.testing.assert_array_equal(fin0, init)


CONV_MUTATIONS = {
    "kernel_not_reversed": ("acc += w[i * K + k] * v;", "acc += w[i * K + (K - 1 - k)] * v;"),
    "off_by_one_window": ("long s = t - (K - 1) + k;  /* position", "long s = t - K + k;  /* position"),
    "bias_after_activation": ("out[i * L + t] = silu_on ? silu(acc) : acc;",
                              "out[i * L + t] = (silu_on ? silu(acc - (bias ? bias[i] : 0.0)) : "
                              "acc - (bias ? bias[i] : 0.0)) + (bias ? bias[i] : 0.0);"),
}


def _conv_pins_pass():
    try:
        test_matches_numpy_convolution(4)
        test_impulse_response_is_the_reversed_kernel()
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("name", sorted(CONV_MUTATIONS))
def test_planted_conv_mistake_fails_a_pin(name):
    import os
    from tests.test_oracle_pins import _mutated_oracle
    src = open(os.path.join(os.path.dirname(oracle.__file__), "s6_oracle.c")).read()
    old, new = CONV_MUTATIONS[name]
    assert src.count(old) == 1, "mutation anchor not found: " + name
    with _mutated_oracle(src.replace(old, new)):
        assert not _conv_pins_pass(), "planted mistake survived every pin: " + name
    assert _conv_pins_pass()
