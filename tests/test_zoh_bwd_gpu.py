"""Parity of the exact-ZOH backward (mamba_selective_scan_bwd_ex with MAMBA_FLAG_EXACT_ZOH)
with the fp64 oracle's ZOH backward (pinned by central differences of the ZOH forward in
test_oracle_backward.py), through the C ABI.  The weight w = expm1(Delta A) / A (Mamba,
"Method" section) and its derivative in A, Delta^2 psi(Delta A), switch between a series
and the closed form at |Delta A| = 1/16, so the cases cover small, mixed and large steps,
A = 0, A > 0 and A near zero, ragged shapes and both dtypes.  Tolerances are those of the
plain backward (test_scan_bwd_gpu.py): the bf16-output rule for bf16 gradients, and
|g - ref| <= rel (|ref| + RMS(ref)) for fp32 gradients, rel = 1e-3 (bf16 inputs) or 1e-4
(fp32 inputs); the weight's fp32 evaluation (a few millionths relative, up to about 1e-5
for dw/dA next to the switch, where its closed form cancels) sits well inside them.
"""
import pytest
import torch

import oracle
from selective_state_space_56_b200 import inputs, ops
from tests.test_scan_bwd_gpu import GRADS, _compare, _grad_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gpu_bwd_zoh(p, dy, softplus=True):
    c = {k: (None if v is None else v.to(DEV)) for k, v in p.items()}
    g = ops.selective_scan_bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], dy.to(DEV), D=c["D"],
                               z=c["z"], delta_bias=c["delta_bias"], delta_softplus=softplus,
                               exact_zoh=True)
    torch.cuda.synchronize()
    return g


def _oracle_bwd_zoh(p, dy, softplus=True):
    return oracle.selective_scan_backward(p["u"], p["delta"], p["A"], p["B"], p["C"], dy,
                                          D=p["D"], z=p["z"], delta_bias=p["delta_bias"],
                                          softplus=softplus, zoh=True)


def test_tiny_fp32_workload_zoh_backward(cuda_ok):
    w = inputs.SCAN_WORKLOADS["tiny_fp32"]
    p, dy = _grad_inputs(w.batch, w.dim, w.dstate, w.seqlen, w.in_dtype, w.seed)
    _compare(_gpu_bwd_zoh(p, dy), _oracle_bwd_zoh(p, dy), p, w.in_dtype)


@pytest.mark.parametrize("regime", ["small_steps", "mixed", "large_steps"])
@pytest.mark.parametrize("shape", [(2, 40, 16, 200), (3, 24, 16, 77), (2, 33, 5, 130)],
                         ids=lambda s: "x".join(map(str, s)))
def test_zoh_backward_fp32_regimes(cuda_ok, shape, regime):
    b, d, N, L = shape
    p, dy = _grad_inputs(b, d, N, L, torch.float32, seed=sum(shape) + len(regime))
    shift = {"small_steps": -9.0, "mixed": 0.0, "large_steps": 3.0}[regime]
    p["delta"] = p["delta"] * 0.3
    p["delta_bias"] = p["delta_bias"] + shift
    _compare(_gpu_bwd_zoh(p, dy), _oracle_bwd_zoh(p, dy), p, torch.float32)


def test_zoh_backward_zero_positive_and_small_A(cuda_ok):
    p, dy = _grad_inputs(2, 20, 16, 96, torch.float32, seed=77)
    A = p["A"].clone()
    A[:, 0] = 0.0       # pure integrator: w = Delta, dw/dA = Delta^2 / 2
    A[:, 1] = 0.25      # mildly unstable
    A[::3, 5] = -1e-3   # near zero
    p["A"] = A
    _compare(_gpu_bwd_zoh(p, dy), _oracle_bwd_zoh(p, dy), p, torch.float32)


@pytest.mark.parametrize("shape,dtype", [((2, 40, 16, 200), torch.bfloat16),
                                         ((1, 16, 16, 1), torch.float32),
                                         ((2, 24, 8, 64), torch.bfloat16)],
                         ids=lambda v: "x".join(map(str, v)) if isinstance(v, tuple) else str(v))
def test_zoh_backward_shapes(cuda_ok, shape, dtype):
    b, d, N, L = shape
    p, dy = _grad_inputs(b, d, N, L, dtype, seed=L + d)
    _compare(_gpu_bwd_zoh(p, dy), _oracle_bwd_zoh(p, dy), p, dtype)


@pytest.mark.parametrize("variant", ["no_softplus", "no_gate_no_skip_no_bias"])
def test_zoh_backward_options(cuda_ok, variant):
    softplus = variant != "no_softplus"
    p, dy = _grad_inputs(2, 24, 16, 64, torch.float32, seed=31,
                         with_z=variant == "no_softplus", with_d=variant == "no_softplus",
                         with_bias=variant == "no_softplus")
    if not softplus:  # positive steps without the softplus
        p["delta"] = p["delta"].abs() * 0.05 + 0.01
        p["delta_bias"] = torch.full_like(p["delta_bias"], 0.02)
    _compare(_gpu_bwd_zoh(p, dy, softplus), _oracle_bwd_zoh(p, dy, softplus), p, torch.float32)


def test_zoh_backward_m130m_layer(cuda_ok):
    """The 130M-shaped layer (8, 1536, 16, 2048) in bf16 with the exact ZOH weight: every
    gradient in full."""
    w = inputs.SCAN_WORKLOADS["m130m"]
    p, dy = _grad_inputs(w.batch, w.dim, w.dstate, w.seqlen, w.in_dtype, w.seed)
    _compare(_gpu_bwd_zoh(p, dy), _oracle_bwd_zoh(p, dy), p, w.in_dtype)


def test_zoh_backward_flag_zero_is_the_plain_backward(cuda_ok):
    p, dy = _grad_inputs(2, 16, 16, 48, torch.float32, seed=5)
    c = {k: (None if v is None else v.to(DEV)) for k, v in p.items()}
    args = (c["u"], c["delta"], c["A"], c["B"], c["C"], dy.to(DEV))
    kw = dict(D=c["D"], z=c["z"], delta_bias=c["delta_bias"])
    g0 = ops.selective_scan_bwd(*args, **kw)
    g1 = ops.selective_scan_bwd(*args, **kw, exact_zoh=False)
    torch.cuda.synchronize()
    for name, _ in GRADS:
        if g0[name] is not None and name in ("du", "ddelta", "dz"):
            assert torch.equal(g0[name], g1[name]), name


def test_zoh_backward_of_a_split_sequence(cuda_ok):
    """The exact-ZOH backward of a sequence swept in segments (checkpoint pass with the ZOH
    weight from each segment's true start, adjoint summaries and their fold)."""
    p, dy = _grad_inputs(1, 40, 16, 20000, torch.float32, seed=9)
    _compare(_gpu_bwd_zoh(p, dy), _oracle_bwd_zoh(p, dy), p, torch.float32)
