"""Pins for the fp64 oracle: each test checks it against something other than itself.

* hand-worked examples (tests/golden/s6_worked_examples.json);
* the associative combine of the parallel-scan derivation and three prefix
  algorithms over it, plus a brute-force product form, against the oracle's
  sequential states;
* the LTI convolution form when Delta, B and C do not vary in time;
* softplus against numpy's log-add-exp, Abar in (0, 1), the small- and
  large-Delta limits, the gated-RNN special case, decode steps against the scan;
* a mutation check: plausible mistakes planted in a copy of the oracle's C
  source must each fail at least one pin.
"""
import contextlib
import ctypes
import json
import math
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest
from scipy.special import expit

import oracle
from oracle import pscan

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "s6_worked_examples.json")
LN2 = math.log(2.0)


def _softplus_lib(x):
    return np.logaddexp(0.0, x)


def _silu_lib(z):
    return z * expit(z)


def _rand_lanes(rng, nl, N, L, nbatch=1):
    return dict(
        u=rng.standard_normal((nl, L)),
        delta_raw=rng.standard_normal((nl, L)),
        z=rng.standard_normal((nl, L)),
        A=-rng.uniform(0.5, 3.0, (nl, N)),
        D=rng.standard_normal(nl),
        delta_bias=rng.uniform(-4.0, -1.0, nl),
        B=rng.standard_normal((nbatch, N, L)),
        C=rng.standard_normal((nbatch, N, L)),
        lane_batch=rng.integers(0, nbatch, nl),
    )


def _run_golden_case(case):
    N, L = case["N"], case["L"]
    kw = dict(
        u=np.array([case["u"]], float), delta_raw=np.array([case["delta_raw"]], float),
        A=np.array([case["A"]], float), B=np.array([case["B"]], float),
        C=np.array([case["C"]], float), lane_batch=[0],
        D=np.array([case["D"]]), delta_bias=np.array([case["delta_bias"]]),
        z=None if case["z"] is None else np.array([case["z"]], float),
        softplus=case["softplus"])
    y, h = oracle.scan_lanes(**kw)
    assert y.shape == (1, L) and h.shape == (1, N)
    return y[0], h[0]


def check_golden():
    cases = json.load(open(GOLDEN))["cases"]
    for case in cases:
        y, h = _run_golden_case(case)
        if "y" in case:
            np.testing.assert_allclose(y, case["y"], rtol=1e-12, atol=1e-12, err_msg=case["name"])
            np.testing.assert_allclose(h, case["last_state"], rtol=1e-12, atol=1e-12,
                                       err_msg=case["name"])
        else:
            np.testing.assert_allclose(y, np.array(case["y_over_ln2"]) * LN2, rtol=1e-12,
                                       err_msg=case["name"])
            np.testing.assert_allclose(h, np.array(case["last_state_over_ln2"]) * LN2,
                                       rtol=1e-12, err_msg=case["name"])


def test_golden_worked_examples():
    check_golden()


def test_combine_is_associative():
    rng = np.random.default_rng(1)
    for _ in range(200):
        T = [(rng.uniform(0, 1, 8), rng.standard_normal(8)) for _ in range(3)]
        k, j, i = T
        lhs = pscan.combine(pscan.combine(k, j), i)
        rhs = pscan.combine(k, pscan.combine(j, i))
        for a, b in zip(lhs, rhs):
            np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-13)


def check_prefix_matches_states(seed=2, nl=5, N=4, L=37):
    rng = np.random.default_rng(seed)
    p = _rand_lanes(rng, nl, N, L, nbatch=2)
    y, h_last, h_all = oracle.scan_lanes(softplus=True, return_states=True, **p)
    delta, abar = oracle.discretize(p["delta_raw"], p["A"], p["delta_bias"], softplus=True)
    for i in range(nl):
        Bb = p["B"][p["lane_batch"][i]]
        Cb = p["C"][p["lane_batch"][i]]
        b = (delta[i] * p["u"][i])[:, None] * Bb.T          # step 1: b_t = Delta_t B_t x_t
        states = {
            "sequential": pscan.prefix_sequential(abar[i], b)[1],
            "hillis_steele": pscan.prefix_hillis_steele(abar[i], b)[1],
            "blelloch": pscan.prefix_blelloch(abar[i], b)[1],
        }
        for k in sorted({1, 7, 20, L - 1} & set(range(1, L))):
            states["split%d" % k] = pscan.prefix_split(abar[i], b, k)[1]
        # brute force: h_t = sum_{s<=t} (prod_{s<tau<=t} Abar_tau) b_s
        brute = np.zeros((L, N))
        for t in range(L):
            for s in range(t + 1):
                brute[t] += np.prod(abar[i, s + 1:t + 1], axis=0) * b[s]
        states["brute"] = brute
        for name, hs in states.items():
            np.testing.assert_allclose(h_all[i], hs, rtol=1e-12, atol=1e-12, err_msg=name)
        np.testing.assert_allclose(h_last[i], h_all[i, -1], rtol=0, atol=0)
        # readout reads the updated state; D skip and gate on top
        y_ref = ((Cb.T * states["blelloch"]).sum(1) + p["D"][i] * p["u"][i]) * _silu_lib(p["z"][i])
        np.testing.assert_allclose(y[i], y_ref, rtol=1e-12, atol=1e-12)


def test_prefix_algorithms_reproduce_states():
    check_prefix_matches_states()


def test_initial_state_enters_through_the_prefix():
    rng = np.random.default_rng(3)
    p = _rand_lanes(rng, 3, 4, 25)
    h0 = rng.standard_normal((3, 4))
    _, h_last, h_all = oracle.scan_lanes(softplus=True, h0=h0, return_states=True, **p)
    delta, abar = oracle.discretize(p["delta_raw"], p["A"], p["delta_bias"])
    for i in range(3):
        b = (delta[i] * p["u"][i])[:, None] * p["B"][0].T
        SA, SB = pscan.prefix_blelloch(abar[i], b)
        np.testing.assert_allclose(h_all[i], SA * h0[i] + SB, rtol=1e-12, atol=1e-12)


def check_lti_convolution(seed=4, nl=3, N=6, L=50):
    """Delta, B, C fixed in time: y = (K * u + D u) silu(z), K_k = sum_n C_n Abar_n^k Delta B_n."""
    rng = np.random.default_rng(seed)
    x = rng.uniform(-3, 1, nl)                       # raw step, constant in t
    A = -rng.uniform(0.2, 2.0, (nl, N))
    Bn = rng.standard_normal(N)
    Cn = rng.standard_normal(N)
    u = rng.standard_normal((nl, L))
    z = rng.standard_normal((nl, L))
    D = rng.standard_normal(nl)
    bias = rng.uniform(-1, 1, nl)
    y, _ = oracle.scan_lanes(u=u, delta_raw=np.repeat(x[:, None], L, 1), A=A,
                             B=np.repeat(Bn[None, :, None], L, 2),
                             C=np.repeat(Cn[None, :, None], L, 2), lane_batch=np.zeros(nl, int),
                             D=D, z=z, delta_bias=bias, softplus=True)
    for i in range(nl):
        dlt = _softplus_lib(x[i] + bias[i])
        abar = np.exp(dlt * A[i])
        K = np.array([(Cn * abar ** k * dlt * Bn).sum() for k in range(L)])
        conv = np.convolve(u[i], K)[:L]
        np.testing.assert_allclose(y[i], (conv + D[i] * u[i]) * _silu_lib(z[i]), rtol=1e-11,
                                   atol=1e-11)


def test_lti_convolution_form():
    check_lti_convolution()


def test_softplus_and_bias_order():
    xs = np.concatenate([np.linspace(-40, 40, 801), [-700.0, -50.0, 50.0, 700.0]])
    for x in xs:
        assert oracle.softplus(x) == pytest.approx(_softplus_lib(x), rel=1e-14, abs=1e-300)
    raw = np.linspace(-5, 5, 11)[None, :]
    bias = np.array([0.7])
    A = np.array([[-1.0, -2.0]])
    d_on, abar = oracle.discretize(raw, A, bias, softplus=True)
    np.testing.assert_allclose(d_on[0], _softplus_lib(raw[0] + 0.7), rtol=1e-14)
    np.testing.assert_allclose(abar[0], np.exp(d_on[0][:, None] * A[0]), rtol=1e-14)
    d_off, _ = oracle.discretize(raw, A, bias, softplus=False)
    np.testing.assert_allclose(d_off[0], raw[0] + 0.7, rtol=0, atol=1e-15)


def test_abar_in_unit_interval_on_workload_distribution():
    from selective_state_space_56_b200 import inputs
    p = inputs.scan_inputs(2, 64, 16, 256, seed=56002)
    dr = p["delta"].float().reshape(-1, 256)
    A = np.tile(p["A"].numpy(), (2, 1))
    bias = np.tile(p["delta_bias"].numpy(), 2)
    delta, abar = oracle.discretize(dr, A, bias, softplus=True)
    assert (delta > 0).all()
    assert (abar > 0).all() and (abar < 1).all()
    lo, hi = inputs.inverse_softplus_range()
    assert lo < bias.min() and bias.max() < hi


def test_small_delta_keeps_state():
    rng = np.random.default_rng(5)
    b, d, N = 2, 3, 4
    state = rng.standard_normal((b, d, N))
    u, z = rng.standard_normal((b, d)), rng.standard_normal((b, d))
    B, C = rng.standard_normal((b, N)), rng.standard_normal((b, N))
    A = -np.tile(np.arange(1.0, N + 1), (d, 1))
    D = rng.standard_normal(d)
    new, y = oracle.state_update(state, u, np.full((b, d), -30.0), A, B, C, D=D, z=z,
                                 softplus=True)
    np.testing.assert_allclose(new, state, rtol=0, atol=1e-12)
    y_ref = ((C[:, None, :] * state).sum(-1) + D * u) * _silu_lib(z)
    np.testing.assert_allclose(y, y_ref, rtol=1e-11, atol=1e-12)


def test_large_delta_forgets():
    rng = np.random.default_rng(6)
    b, d, N = 2, 3, 4
    state = rng.standard_normal((b, d, N))
    u = rng.standard_normal((b, d))
    B, C = rng.standard_normal((b, N)), rng.standard_normal((b, N))
    A = -np.tile(np.arange(1.0, N + 1), (d, 1))
    new, _ = oracle.state_update(state, u, np.full((b, d), 30.0), A, B, C, softplus=True)
    dlt = _softplus_lib(30.0)
    np.testing.assert_allclose(new, dlt * u[..., None] * B[:, None, :], rtol=1e-11, atol=1e-12)
    # same in the scan: with a huge step every state equals its own fresh input term
    L = 9
    uu = rng.standard_normal((1, L))
    Bs = rng.standard_normal((1, N, L))
    _, _, h_all = oracle.scan_lanes(uu, np.full((1, L), 30.0), A[:1], Bs, Bs, [0],
                                    softplus=True, return_states=True)
    np.testing.assert_allclose(h_all[0], dlt * uu[0][:, None] * Bs[0].T, rtol=1e-11, atol=1e-12)


def test_gated_rnn_special_case():
    """N = 1, A = -1: Abar_t = 1 - sigmoid(x_t), so h_t = (1 - g_t) h_{t-1} + Delta_t B_t x_t."""
    rng = np.random.default_rng(7)
    L = 40
    raw = rng.standard_normal((1, L)) * 2
    u = rng.standard_normal((1, L))
    Bs = rng.standard_normal((1, 1, L))
    _, abar = oracle.discretize(raw, np.array([[-1.0]]), None, softplus=True)
    g = expit(raw[0])
    np.testing.assert_allclose(abar[0, :, 0], 1.0 - g, rtol=1e-13, atol=1e-15)
    _, _, h_all = oracle.scan_lanes(u, raw, np.array([[-1.0]]), Bs, Bs, [0], softplus=True,
                                    return_states=True)
    h = 0.0
    for t in range(L):
        h = (1 - g[t]) * h + _softplus_lib(raw[0, t]) * Bs[0, 0, t] * u[0, t]
        assert h_all[0, t, 0] == pytest.approx(h, rel=1e-12, abs=1e-13)


def test_decode_steps_reproduce_scan():
    rng = np.random.default_rng(8)
    b, d, N, L = 2, 3, 4, 12
    u = rng.standard_normal((b, d, L))
    dr = rng.standard_normal((b, d, L))
    z = rng.standard_normal((b, d, L))
    A = -rng.uniform(0.5, 2, (d, N))
    B, C = rng.standard_normal((b, N, L)), rng.standard_normal((b, N, L))
    D, bias = rng.standard_normal(d), rng.uniform(-3, -1, d)
    y, hl = oracle.selective_scan(u, dr, A, B, C, D=D, z=z, delta_bias=bias)
    st = np.zeros((b, d, N))
    for t in range(L):
        st, yt = oracle.state_update(st, u[..., t], dr[..., t], A, B[..., t], C[..., t], D=D,
                                     z=z[..., t], delta_bias=bias)
        np.testing.assert_allclose(yt, y[..., t], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(st, hl, rtol=1e-13, atol=1e-13)


def test_batches_read_their_own_B_and_C():
    rng = np.random.default_rng(9)
    b, d, N, L = 3, 2, 4, 10
    args = dict(u=rng.standard_normal((b, d, L)), delta=rng.standard_normal((b, d, L)),
                A=-rng.uniform(0.5, 2, (d, N)), B=rng.standard_normal((b, N, L)),
                C=rng.standard_normal((b, N, L)), D=rng.standard_normal(d),
                z=rng.standard_normal((b, d, L)), delta_bias=rng.uniform(-3, -1, d))
    y, hl = oracle.selective_scan(**args)
    for bi in range(b):
        one = {k: (v[bi:bi + 1] if k in ("u", "delta", "B", "C", "z") else v)
               for k, v in args.items()}
        y1, h1 = oracle.selective_scan(**one)
        np.testing.assert_array_equal(y1[0], y[bi])
        np.testing.assert_array_equal(h1[0], hl[bi])


# --- mutation check -----------------------------------------------------------------------

MUTATIONS = {
    "drop_D_skip": ("acc += dskip * ut;", "acc += 0.0 * ut;"),
    "sign_of_exponent": ("exp(dt * A[i * N + n]);\n                double wt",
                         "exp(-dt * A[i * N + n]);\n                double wt"),
    "readout_before_update": (
        "hv[n] = abar * hv[n] + wt * Bb[n * L + t] * ut;\n                acc += Cb[n * L + t] * hv[n];",
        "acc += Cb[n * L + t] * hv[n];\n                hv[n] = abar * hv[n] + wt * Bb[n * L + t] * ut;"),
    "B_C_swapped": ("hv[n] = abar * hv[n] + wt * Bb[n * L + t] * ut;\n                acc += Cb[n * L + t]",
                    "hv[n] = abar * hv[n] + wt * Cb[n * L + t] * ut;\n                acc += Bb[n * L + t]"),
    "B_time_index_shift": ("wt * Bb[n * L + t] * ut", "wt * Bb[n * L + (t > 0 ? t - 1 : 0)] * ut"),
    "bias_after_softplus": ("double x = delta_raw + bias;\n    return softplus ? s6o_softplus(x) : x;",
                            "return softplus ? s6o_softplus(delta_raw) + bias : delta_raw + bias;"),
    "missing_delta_in_B": ("wt * Bb[n * L + t] * ut", "Bb[n * L + t] * ut"),
    "gate_is_sigmoid": ("if (z) acc *= silu(z[i * L + t]);",
                        "if (z) acc *= 1.0 / (1.0 + exp(-z[i * L + t]));"),
    "softplus_wrong_branch": ("if (x > 0.0) return x + log1p(exp(-x));",
                              "if (x > 0.0) return log1p(exp(-x));"),
}


@contextlib.contextmanager
def _mutated_oracle(src_text):
    d = tempfile.mkdtemp(prefix="s6o_mut_")
    try:
        c = os.path.join(d, "m.c")
        so = os.path.join(d, "m.so")
        open(c, "w").write(src_text)
        subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-o", so, c, "-lm"], check=True)
        real = oracle._load()
        lib = ctypes.CDLL(so)
        for name in ("s6o_softplus", "s6o_discretize", "s6o_scan", "s6o_state_update",
                     "s6o_scan_backward", "s6o_causal_conv1d", "s6o_causal_conv1d_update",
                     "s6o_causal_conv1d_backward"):
            getattr(lib, name).restype = getattr(real, name).restype
            getattr(lib, name).argtypes = getattr(real, name).argtypes
        lib.s6o_num_threads = real.s6o_num_threads
        saved = oracle._lib
        oracle._lib = lib
        try:
            yield
        finally:
            oracle._lib = saved
    finally:
        shutil.rmtree(d, ignore_errors=True)


def _pins_pass():
    try:
        check_golden()
        check_prefix_matches_states(nl=2, L=17)
        check_lti_convolution(nl=2, L=30)
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "s6_oracle.c")).read()
    old, new = MUTATIONS[name]
    assert src.count(old) == 1, "mutation anchor not found: " + name
    with _mutated_oracle(src.replace(old, new)):
        assert not _pins_pass(), "planted mistake survived every pin: " + name
    assert _pins_pass()
