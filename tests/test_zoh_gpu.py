"""Parity of the exact zero-order-hold variant (MAMBA_FLAG_EXACT_ZOH) with the fp64 oracle's
ZOH scan (pinned in test_oracle_zoh.py), through the C ABI.  Bbar = (exp(Delta A) - 1) / A * B
replaces Delta * B (Mamba, "Method" section); the kernels evaluate the weight from the same
exponential as Abar where |Delta A| >= 1/16 and from the series of expm1(y) / y below, so the
cases cover both branches (small, mixed and large steps), A = 0 and A > 0, a split sequence
(segment aggregates with the ZOH weight), and the decode step.  Tolerances are those of the
plain scan (s6_compare).
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_56_b200 import inputs, ops
from tests.s6_compare import check_bf16_out, check_fp32, check_rms

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gpu(p, out_dtype=None, softplus=True):
    g = {k: (None if v is None else v.to(DEV)) for k, v in p.items()}
    y, st = ops.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                                   delta_bias=g["delta_bias"], delta_softplus=softplus,
                                   out_dtype=out_dtype, return_last_state=True, exact_zoh=True)
    torch.cuda.synchronize()
    return y, st


def _ref(p, softplus=True):
    return oracle.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                                 delta_bias=p["delta_bias"], softplus=softplus, zoh=True)


def test_tiny_fp32_workload_zoh(cuda_ok):
    w = inputs.SCAN_WORKLOADS["tiny_fp32"]
    p = inputs.workload_inputs(w)
    y, st = _gpu(p)
    y_ref, st_ref = _ref(p)
    check_fp32(y, y_ref, "y")
    check_fp32(st, st_ref, "last_state")


@pytest.mark.parametrize("regime", ["small_steps", "mixed", "large_steps"])
@pytest.mark.parametrize("shape", [(2, 40, 16, 200), (1, 24, 8, 77), (3, 16, 4, 130)],
                         ids=lambda s: "x".join(map(str, s)))
def test_zoh_fp32_regimes(cuda_ok, shape, regime):
    b, d, N, L = shape
    p = inputs.scan_inputs(b, d, N, L, torch.float32, seed=sum(shape) + len(regime))
    # step bias: Delta ~ 1e-4 (every |Delta A| < 1/16), the recipe's [0.001, 0.1] (both
    # branches), or Delta ~ 3 (most |Delta A| >= 1/16)
    shift = {"small_steps": -9.0, "mixed": 0.0, "large_steps": 3.0}[regime]
    p["delta"] = p["delta"] * 0.3
    p["delta_bias"] = p["delta_bias"] + shift
    y, st = _gpu(p)
    y_ref, st_ref = _ref(p)
    check_fp32(y, y_ref, "y")
    check_fp32(st, st_ref, "last_state")


def test_zoh_zero_and_positive_A(cuda_ok):
    b, d, N, L = 2, 20, 16, 96
    p = inputs.scan_inputs(b, d, N, L, torch.float32, seed=77)
    A = p["A"].clone()
    A[:, 0] = 0.0       # pure integrator
    A[:, 1] = 0.25      # mildly unstable
    A[::3, 5] = -1e-3   # near zero
    p["A"] = A
    y, st = _gpu(p)
    y_ref, st_ref = _ref(p)
    check_fp32(y, y_ref, "y")
    check_fp32(st, st_ref, "last_state")


def test_zoh_bf16_m130m_layer(cuda_ok):
    w = inputs.SCAN_WORKLOADS["m130m"]
    p = inputs.workload_inputs(w)
    y32, st = _gpu(p, out_dtype=torch.float32)
    y_ref, st_ref = _ref(p)
    check_rms(y32, y_ref, "y (fp32 out)")
    check_rms(st, st_ref, "last_state")
    y16, _ = _gpu(p)
    check_bf16_out(y16, y_ref, "y (bf16 out)")


def test_zoh_split_sequence(cuda_ok):
    """Few channels and a long sequence: the scan runs as segment aggregates, the carry
    across segments and a rescan, all with the ZOH weight."""
    b, d, N, L = 1, 64, 16, 40000
    assert ops.selective_scan_workspace_size(b, d, N, L) > 0
    p = inputs.scan_inputs(b, d, N, L, torch.bfloat16, seed=4242)
    y, st = _gpu(p, out_dtype=torch.float32)
    y_ref, st_ref = _ref(p)
    check_rms(y, y_ref, "y")
    check_rms(st, st_ref, "last_state")


def test_zoh_differs_from_delta_B(cuda_ok):
    p = inputs.scan_inputs(1, 16, 16, 64, torch.float32, seed=3)
    y_z, _ = _gpu(p)
    g = {k: (None if v is None else v.to(DEV)) for k, v in p.items()}
    y_p = ops.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=None, z=None,
                                 delta_bias=g["delta_bias"])
    y_z2 = ops.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=None, z=None,
                                  delta_bias=g["delta_bias"], exact_zoh=True)
    gap = (y_z2 - y_p).abs().max().item()
    assert gap > 1e-3 * y_p.abs().max().item()
    assert y_z.shape == y_p.shape


@pytest.mark.parametrize("N,dtype", [(16, torch.bfloat16), (16, torch.float32), (5, torch.float32),
                                     (8, torch.bfloat16)])
def test_zoh_decode_steps(cuda_ok, N, dtype):
    b, d, steps = 3, 96, 6
    gen = torch.Generator().manual_seed(900 + N)
    A = -torch.rand(d, N, generator=gen) * 3 - 0.05
    A[:, 0] = 0.0
    D = torch.randn(d, generator=gen)
    bias = torch.rand(d, generator=gen) * 2 - 4
    state0 = 0.1 * torch.randn(b, d, N, generator=gen)
    st_gpu = state0.to(DEV)
    st_ref = state0.double().numpy()
    tol = check_fp32 if dtype == torch.float32 else check_rms
    for k in range(steps):
        u, dr, z = (torch.randn(b, d, generator=gen).to(dtype) for _ in range(3))
        Bm, Cm = (torch.randn(b, N, generator=gen).to(dtype) for _ in range(2))
        y = ops.selective_state_update(st_gpu, u.to(DEV), dr.to(DEV), A.to(DEV), Bm.to(DEV),
                                       Cm.to(DEV), D=D.to(DEV), z=z.to(DEV),
                                       delta_bias=bias.to(DEV), exact_zoh=True)
        st_ref, y_ref = oracle.state_update(st_ref, u, dr, A, Bm, Cm, D=D, z=z, delta_bias=bias,
                                            zoh=True)
        torch.cuda.synchronize()
        if dtype == torch.float32:
            check_fp32(y, y_ref, "y step %d" % k)
        else:
            check_bf16_out(y, y_ref, "y step %d" % k)
        tol(st_gpu, st_ref, "state step %d" % k)
    assert np.isfinite(st_ref).all()
