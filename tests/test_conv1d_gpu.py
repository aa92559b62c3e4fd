"""Parity of the CUDA causal depthwise conv1d (+ SiLU) and its decode update with the fp64
oracle (pinned in test_oracle_conv.py), through the C ABI.

Tolerances: fp32 outputs per element |o - ref| <= 1e-4 max(1, |ref|) (s6_compare's fp32
rule); bf16 outputs per element |o - ref| <= ulp_bf16(|ref|) + 1e-6 S, S = |bias| +
sum_k |w_k x_k| -- the kernel sums at most five fp32 terms (error below 5 * 2^-24 S, and
SiLU's slope is at most 1.1) and applies the SFU SiLU (relative error about 1e-6), then
rounds to bf16 (half an ulp, one ulp with a tie flip).  The S term matters only where the
terms cancel to a result much smaller than themselves.  Final conv states are copies of
inputs and must match bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_56_b200 import inputs, ops
from tests.s6_compare import check_fp32, to64, ulp_bf16

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _term_scale(p, x=None):
    """S = |bias| + sum_k |w_k x_k| per output (the oracle's conv of absolute values)."""
    xx = p["x"] if x is None else x
    s, _ = oracle.causal_conv1d(to64(xx).__abs__(), to64(p["weight"]).__abs__(),
                                None if p["bias"] is None else to64(p["bias"]).__abs__(),
                                None if p.get("initial_state") is None
                                else to64(p["initial_state"]).__abs__(), silu=False)
    return s


def _check(got, ref, what, scale=None):
    if got.dtype == torch.float32:
        check_fp32(got, ref, what)
        return
    g, r = to64(got), to64(ref)
    err = np.abs(g - r)
    bound = ulp_bf16(r) + (0.0 if scale is None else 1e-6 * scale)
    bad = err > bound
    assert not bad.any(), "%s: %d/%d elements beyond ulp_bf16 + 1e-6 S" % (
        what, int(bad.sum()), bad.size)


def _run(p, silu=True):
    g = {k: (None if v is None else v.to(DEV)) for k, v in p.items()}
    out, fin = ops.causal_conv1d_fwd(g["x"], g["weight"], g["bias"], g["initial_state"], silu=silu,
                                     return_final_state=True)
    torch.cuda.synchronize()
    return out, fin


def _ref(p, silu=True):
    return oracle.causal_conv1d(p["x"], p["weight"], p["bias"], p["initial_state"], silu=silu)


CASES = [(2, 40, 200, 4, torch.bfloat16), (1, 24, 77, 3, torch.float32),
         (3, 16, 130, 2, torch.float32), (2, 8, 64, 1, torch.bfloat16),
         (1, 33, 21, 4, torch.bfloat16), (2, 7, 96, 4, torch.float32),
         (1, 5, 2, 4, torch.bfloat16), (1, 5, 1, 3, torch.float32),
         (1, 70000, 16, 4, torch.bfloat16)]  # more channels than a grid's y extent


@pytest.mark.parametrize("init", [False, True], ids=["zero_init", "init_state"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "%dx%dx%d_k%d_%s" % (
    c[0], c[1], c[2], c[3], str(c[4]).split(".")[1]))
def test_conv1d_shapes(cuda_ok, case, init):
    b, d, L, K, dt = case
    p = inputs.conv_inputs(b, d, L, K, dt, seed=b * 1000 + d * 10 + L, with_initial_state=init)
    out, fin = _run(p)
    ref, fref = _ref(p)
    _check(out, ref, "out", _term_scale(p))
    if K > 1:
        np.testing.assert_array_equal(to64(fin), fref)


@pytest.mark.parametrize("silu", [True, False])
def test_conv1d_options(cuda_ok, silu):
    p = inputs.conv_inputs(2, 24, 64, 4, torch.float32, seed=5, with_bias=False)
    out, _ = _run(p, silu=silu)
    ref, _ = _ref(p, silu=silu)
    _check(out, ref, "out")


def test_conv1d_empty_sequence_passes_the_state(cuda_ok):
    p = inputs.conv_inputs(2, 16, 0, 4, torch.bfloat16, seed=9, with_initial_state=True)
    out, fin = _run(p)
    assert out.shape == (2, 16, 0)
    torch.testing.assert_close(fin.cpu(), p["initial_state"], rtol=0, atol=0)


def test_conv1d_m2p8b_layer(cuda_ok):
    """The producer of the 2.8B-shaped layer's u: (4, 5120, 4096), K = 4, bf16, in full."""
    p = inputs.conv_inputs(4, 5120, 4096, 4, torch.bfloat16)
    out, fin = _run(p)
    ref, fref = _ref(p)
    _check(out, ref, "out", _term_scale(p))
    np.testing.assert_array_equal(to64(fin), fref)


@pytest.mark.parametrize("b", [3, 6])
@pytest.mark.parametrize("d", [48, 45])
@pytest.mark.parametrize("K,dt", [(4, torch.bfloat16), (3, torch.float32), (2, torch.bfloat16),
                                  (1, torch.float32)])
def test_conv1d_decode_continues_the_prefill(cuda_ok, K, dt, d, b):
    """Decode steps after a prefill equal the prefill of the longer sequence (channel
    counts with and without a multiple-of-8 tail; 3 batch rows take one row per thread, 6
    take four rows per thread with the last slice ragged)."""
    L, steps = 20, 6
    p = inputs.conv_inputs(b, d, L + steps, K, dt, seed=77 + K, with_initial_state=True)
    full_ref, _ = _ref(p)
    pre = dict(p)
    pre["x"] = p["x"][:, :, :L].contiguous()
    g = {k: (None if v is None else v.to(DEV)) for k, v in pre.items()}
    out, state = ops.causal_conv1d_fwd(g["x"], g["weight"], g["bias"], g["initial_state"],
                                       return_final_state=True)
    scale = _term_scale(p)
    _check(out, full_ref[:, :, :L], "prefill", scale[:, :, :L])
    st_ref = oracle.causal_conv1d(pre["x"], p["weight"], p["bias"], p["initial_state"])[1]
    if K == 1:
        state = torch.empty((b, d, 0), dtype=dt, device=DEV)
    for s in range(steps):
        xt = p["x"][:, :, L + s].contiguous()
        o = ops.causal_conv1d_update(state, xt.to(DEV), g["weight"], g["bias"])
        st_ref, o_ref = oracle.causal_conv1d_update(st_ref, xt, p["weight"], p["bias"])
        torch.cuda.synchronize()
        _check(o, o_ref, "decode step %d" % s, scale[:, :, L + s])
        _check(o, full_ref[:, :, L + s], "decode vs prefill step %d" % s, scale[:, :, L + s])
        np.testing.assert_array_equal(to64(state), st_ref)
