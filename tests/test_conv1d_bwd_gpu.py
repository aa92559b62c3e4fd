"""Parity of the CUDA backward of the causal depthwise conv1d (+ SiLU) with the fp64
oracle's backward (pinned in test_oracle_conv_backward.py), through the C ABI.

Tolerances, from the kernel's fp32 arithmetic on the exact input values: with pre[t] the
value before the activation (at most five fp32 terms, error below 5 * 2^-24 Sp[t],
Sp = |bias| + sum_k |w_k x_k|) and SiLU's derivative from the SFU's 2^x and reciprocal
(relative error about 2^-21 (1 + |pre|)), each g[t] = dout[t] act'(pre[t]) is off by at
most E[t] = 4e-6 |dout[t]| (1 + Sp[t]) (act'' is below 0.6 in magnitude).  Then

* dx (and the initial state's gradient), K fp32 terms w_k g[.]:
  |dx - ref| <= ulp(|ref|) + sum_k |w_k| (E + 2e-6 |g|)[s + K-1-k], ulp of the output
  dtype (bf16 ulp; 2^-23 |ref| for fp32; one ulp allows a tie flip);
* dweight[k], dbias: sums over batch and steps formed per thread, per warp, per CTA and
  with atomics across CTAs: |err| <= 1e-5 sum_{b,t} (|g| + 4 |dout| (1 + Sp)) |xe_k|
  (xe_k = 1 for dbias), far above the tree-summation bound and below any real mistake.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_56_b200 import inputs, ops
from tests.s6_compare import to64, ulp_bf16

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _problem(b, d, L, K, dt, seed, init=False, bias=True):
    p = inputs.conv_inputs(b, d, L, K, dt, seed=seed, with_bias=bias, with_initial_state=init)
    g = torch.Generator().manual_seed(seed + 1)
    p["dout"] = torch.randn(b, d, L, generator=g).to(dt)
    return p


def _gpu(p, silu=True):
    c = {k: (None if v is None else v.to(DEV)) for k, v in p.items()}
    g = ops.causal_conv1d_bwd(c["x"], c["weight"], c["dout"], c["bias"], c["initial_state"],
                              silu=silu)
    torch.cuda.synchronize()
    return g


def _scales(p, silu):
    """E[t], |g[t]| and Sp[t] in fp64 from the exact inputs (the test's own error model)."""
    x, w = to64(p["x"]), to64(p["weight"])
    bias = None if p["bias"] is None else to64(p["bias"])
    init = None if p["initial_state"] is None else to64(p["initial_state"])
    dout = to64(p["dout"])
    pre, _ = oracle.causal_conv1d(x, w, bias, init, silu=False)
    sp, _ = oracle.causal_conv1d(np.abs(x), np.abs(w), None if bias is None else np.abs(bias),
                                 None if init is None else np.abs(init), silu=False)
    if silu:
        sg = 1.0 / (1.0 + np.exp(-pre))
        g = dout * sg * (1.0 + pre * (1.0 - sg))
    else:
        g = dout
    E = 4e-6 * np.abs(dout) * (1.0 + sp)
    return E, np.abs(g), sp


def _ulp(ref, dt):
    return ulp_bf16(ref) if dt == torch.bfloat16 else np.abs(ref) * 2.0 ** -23


def _check_dx(got, ref, p, E, ag, dt, what):
    w = np.abs(to64(p["weight"]))
    b, d, L = ref.shape
    K = w.shape[1]
    m = E + 2e-6 * ag
    tol = np.empty_like(ref)
    for i in range(b):
        for c in range(d):
            tol[i, c] = np.convolve(m[i, c], w[c], mode="full")[K - 1:K - 1 + L]
    g = to64(got)
    bound = _ulp(ref, dt) + tol
    bad = np.abs(g - ref) > bound
    assert not bad.any(), "%s: %d/%d beyond the bound; worst excess %.3g" % (
        what, int(bad.sum()), bad.size, float((np.abs(g - ref) - bound).max()))


def _check_dinit(got, ref, p, E, ag, dt):
    w = np.abs(to64(p["weight"]))
    b, d, Km1 = ref.shape
    m = E + 2e-6 * ag
    if m.shape[2] < Km1:  # g is zero past the sequence
        m = np.concatenate([m, np.zeros(m.shape[:2] + (Km1 - m.shape[2],))], axis=2)
    m = m[:, :, :Km1]
    tol = np.zeros_like(ref)
    for j in range(Km1):
        for k in range(j + 1):
            tol[:, :, j] += w[:, k][None, :] * m[:, :, j - k]
    bound = _ulp(ref, dt) + tol
    bad = np.abs(to64(got) - ref) > bound
    assert not bad.any(), "dinitial_state: %d/%d beyond the bound" % (int(bad.sum()), bad.size)


def _check_sums(got, p, ref, E, ag):
    x = to64(p["x"])
    b, d, L = x.shape
    K = ref["dweight"].shape[1]
    init = to64(p["initial_state"]) if p["initial_state"] is not None else np.zeros((b, d, K - 1))
    xe = np.abs(np.concatenate([init, x], axis=2))
    mag = ag + E / 1e-6  # |g| + 4 |dout| (1 + Sp), as E = 4e-6 |dout| (1 + Sp)
    sw = np.stack([(mag * xe[:, :, k:k + L]).sum(axis=(0, 2)) for k in range(K)], axis=1)
    err = np.abs(to64(got["dweight"]) - ref["dweight"])
    assert np.all(err <= 1e-5 * sw), "dweight: worst %.3g of its scale" % float((err / sw).max())
    if p["bias"] is not None:
        sb = mag.sum(axis=(0, 2))
        errb = np.abs(to64(got["dbias"]) - ref["dbias"])
        assert np.all(errb <= 1e-5 * sb), "dbias: worst %.3g of its scale" % float((errb / sb).max())
    else:
        assert got["dbias"] is None


def _compare(p, silu=True):
    dt = p["x"].dtype
    got = _gpu(p, silu)
    ref = oracle.causal_conv1d_backward(p["x"], p["weight"], p["dout"], p["bias"],
                                        p["initial_state"], silu=silu)
    E, ag, _ = _scales(p, silu)
    assert got["dx"].dtype == dt and got["dx"].shape == p["x"].shape
    _check_dx(got["dx"], ref["dx"], p, E, ag, dt, "dx")
    _check_sums(got, p, ref, E, ag)
    K = p["weight"].shape[1]
    if p["initial_state"] is not None and K > 1:
        _check_dinit(got["dinitial_state"], ref["dinitial_state"], p, E, ag, dt)
    else:
        assert got["dinitial_state"] is None


CASES = [(2, 40, 200, 4, torch.bfloat16), (1, 24, 77, 3, torch.float32),
         (3, 16, 130, 2, torch.float32), (2, 8, 64, 1, torch.bfloat16),
         (1, 33, 21, 4, torch.bfloat16), (2, 7, 96, 4, torch.float32),
         (1, 5, 2, 4, torch.bfloat16), (1, 5, 1, 3, torch.float32),
         (2, 3, 1040, 4, torch.bfloat16)]


@pytest.mark.parametrize("init", [False, True], ids=["zero_init", "init_state"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "%dx%dx%d_k%d_%s" % (
    c[0], c[1], c[2], c[3], str(c[4]).split(".")[1]))
def test_conv1d_backward_shapes(cuda_ok, case, init):
    b, d, L, K, dt = case
    _compare(_problem(b, d, L, K, dt, seed=b * 1000 + d * 10 + L, init=init))


@pytest.mark.parametrize("silu", [True, False])
@pytest.mark.parametrize("bias", [True, False])
def test_conv1d_backward_options(cuda_ok, silu, bias):
    _compare(_problem(2, 24, 64, 4, torch.float32, seed=5, init=True, bias=bias), silu=silu)


def test_conv1d_backward_many_channels(cuda_ok):
    """More channels than a grid's y extent: CTAs walk several rows."""
    _compare(_problem(1, 70000, 16, 4, torch.bfloat16, seed=11, init=True))


def test_conv1d_backward_empty_sequence(cuda_ok):
    p = _problem(2, 16, 0, 4, torch.bfloat16, seed=9, init=True)
    g = _gpu(p)
    assert g["dx"].shape == (2, 16, 0)
    assert float(g["dweight"].abs().max()) == 0.0 and float(g["dbias"].abs().max()) == 0.0
    assert float(g["dinitial_state"].float().abs().max()) == 0.0


def test_conv1d_backward_is_linear_in_dout(cuda_ok):
    p = _problem(2, 32, 96, 4, torch.float32, seed=21, init=True)
    q = dict(p)
    q["dout"] = (2.0 * p["dout"]).contiguous()
    g1, g2 = _gpu(p), _gpu(q)
    torch.testing.assert_close(g2["dx"], 2.0 * g1["dx"], rtol=0, atol=0)
    torch.testing.assert_close(g2["dweight"], 2.0 * g1["dweight"], rtol=1e-6, atol=0)


def test_conv1d_backward_m2p8b_layer(cuda_ok):
    """The backward of the 2.8B-shaped layer's conv: (4, 5120, 4096), K = 4, bf16, in full."""
    _compare(_problem(4, 5120, 4096, 4, torch.bfloat16, seed=2812))
