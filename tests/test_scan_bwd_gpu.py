"""Parity of the CUDA backward of the selective scan with the fp64 oracle (needs a B200).

The oracle's backward is pinned to finite differences of the forward oracle
(test_oracle_backward.py); here every gradient the library writes (du, ddelta, dz,
dA, dB, dC, dD, ddelta_bias) is compared with it on the same inputs, through the C
ABI.  Tolerances:

* bf16 gradients (du, ddelta, dz after bf16 inputs): the bf16-output rule of
  s6_compare (2e-2 RMS + one bf16 ulp per element).
* fp32 gradients: per element |g - ref| <= rel * (|ref| + RMS(ref)), rel = 1e-3.
  The kernel runs entirely in fp32 on the exact input values; each gradient is a
  sum of at most a few thousand products (over steps, or channels for dB / dC),
  so its rounding error is a few hundred fp32 ulps of the summed magnitude, well
  under 1e-3 of it.  RMS(ref) in the scale absorbs entries that cancel to near zero.
* fp32 inputs: the same rule with rel = 1e-4 for every gradient (short sequences).
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_56_b200 import inputs, ops
from tests.s6_compare import check_bf16_out, rms, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
GRADS = (("du", "du"), ("ddelta", "ddelta"), ("dz", "dz"), ("dA", "dA"), ("dB", "dB"),
         ("dC", "dC"), ("dD", "dD"), ("ddelta_bias", "dbias"))


def check_scaled(got, ref, what, rel):
    got, ref = to64(got), to64(ref)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    if not got.size:
        return 0.0
    scale = rel * (np.abs(ref) + rms(ref))
    err = np.abs(got - ref)
    worst = float((err / np.maximum(scale, 1e-300)).max())
    assert np.all(err <= scale), "%s: %d/%d beyond %.0e*(|ref|+RMS); worst ratio %.3g" % (
        what, int((err > scale).sum()), err.size, rel, worst)
    return worst


def _grad_inputs(b, d, N, L, dtype, seed, with_z=True, with_d=True, with_bias=True):
    p = inputs.scan_inputs(b, d, N, L, dtype, seed=seed, with_z=with_z, with_d=with_d,
                           with_bias=with_bias)
    g = torch.Generator().manual_seed(seed + 7)
    dy = torch.randn(b, d, L, generator=g).to(dtype)
    return p, dy


def _gpu_bwd(p, dy, softplus=True):
    c = {k: (None if v is None else v.to(DEV)) for k, v in p.items()}
    g = ops.selective_scan_bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], dy.to(DEV), D=c["D"],
                               z=c["z"], delta_bias=c["delta_bias"], delta_softplus=softplus)
    torch.cuda.synchronize()
    return g


def _oracle_bwd(p, dy, softplus=True):
    return oracle.selective_scan_backward(p["u"], p["delta"], p["A"], p["B"], p["C"], dy,
                                          D=p["D"], z=p["z"], delta_bias=p["delta_bias"],
                                          softplus=softplus)


def _compare(got, ref, p, dtype):
    for gname, oname in GRADS:
        if got[gname] is None:
            present = {"dz": "z", "dD": "D", "ddelta_bias": "delta_bias"}[gname]
            assert p[present] is None, gname
            continue
        if dtype == torch.float32:
            check_scaled(got[gname], ref[oname], gname, 1e-4)
        elif got[gname].dtype == torch.bfloat16:
            check_bf16_out(got[gname], ref[oname], gname)
        else:
            check_scaled(got[gname], ref[oname], gname, 1e-3)


def test_tiny_fp32_workload_backward(cuda_ok):
    w = inputs.SCAN_WORKLOADS["tiny_fp32"]
    p, dy = _grad_inputs(w.batch, w.dim, w.dstate, w.seqlen, w.in_dtype, w.seed)
    _compare(_gpu_bwd(p, dy), _oracle_bwd(p, dy), p, w.in_dtype)


# several channel tiles with a ragged last one, several chunks with a ragged tail,
# every supported state width class
SHAPES = [(2, 40, 16, 200), (1, 24, 8, 77), (3, 16, 4, 130), (2, 33, 16, 300), (1, 16, 16, 32),
          (2, 17, 5, 1), (1, 48, 12, 129)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["fp32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_backward_shapes(cuda_ok, shape, dtype):
    b, d, N, L = shape
    p, dy = _grad_inputs(b, d, N, L, dtype, seed=sum(shape) * 31)
    _compare(_gpu_bwd(p, dy), _oracle_bwd(p, dy), p, dtype)


@pytest.mark.parametrize("variant", ["no_gate", "no_skip", "no_bias", "no_softplus", "bare"])
def test_backward_options(cuda_ok, variant):
    b, d, N, L = 2, 24, 16, 100
    p, dy = _grad_inputs(b, d, N, L, torch.float32, seed=sum(map(ord, variant)),
                         with_z=variant not in ("no_gate", "bare"),
                         with_d=variant not in ("no_skip", "bare"),
                         with_bias=variant not in ("no_bias", "bare"))
    softplus = variant not in ("no_softplus", "bare")
    if not softplus:
        # raw steps must be positive without the softplus: draw them in (0.001, 0.1)
        gen = torch.Generator().manual_seed(5)
        p["delta"] = 0.001 + 0.099 * torch.rand(b, d, L, generator=gen)
        if p["delta_bias"] is not None:
            p["delta_bias"] = torch.zeros(d)
    _compare(_gpu_bwd(p, dy, softplus), _oracle_bwd(p, dy, softplus), p, torch.float32)


def test_backward_empty_sequence(cuda_ok):
    b, d, N = 2, 20, 16
    p, _ = _grad_inputs(b, d, N, 0, torch.bfloat16, seed=3)
    dy = torch.empty(b, d, 0, dtype=torch.bfloat16)
    g = _gpu_bwd(p, dy)
    for k in ("dA", "dD", "ddelta_bias"):
        assert torch.count_nonzero(g[k]).item() == 0, k
    assert g["du"].shape == (b, d, 0) and g["dB"].shape == (b, N, 0)


def test_backward_is_linear_in_dy(cuda_ok):
    """Doubling dy doubles every gradient (exactly up to rounding: the sweep is linear in
    dy), and dy = 0 gives all-zero gradients."""
    p, dy = _grad_inputs(1, 32, 16, 96, torch.float32, seed=11)
    g1 = _gpu_bwd(p, dy)
    g2 = _gpu_bwd(p, 2 * dy)
    for k, _ in GRADS:
        torch.testing.assert_close(g2[k], 2 * g1[k], rtol=1e-5, atol=1e-6)
    g0 = _gpu_bwd(p, torch.zeros_like(dy))
    for k, _ in GRADS:
        assert torch.count_nonzero(g0[k]).item() == 0, k


def test_m130m_layer_backward_full(cuda_ok):
    """The 130M-shaped layer (8, 1536, 16, 2048) in bf16, every gradient in full; dB and dC
    are sums over all 1536 channels of a batch."""
    w = inputs.SCAN_WORKLOADS["m130m"]
    p, dy = _grad_inputs(w.batch, w.dim, w.dstate, w.seqlen, w.in_dtype, w.seed)
    _compare(_gpu_bwd(p, dy), _oracle_bwd(p, dy), p, w.in_dtype)


def test_m2p8b_layer_backward_full(cuda_ok):
    """The 2.8B-shaped layer (4, 5120, 16, 4096) in bf16 at full size: every gradient of
    every channel, batch and step against the oracle (about 25 s of single-thread fp64);
    dB and dC are sums over all 5120 channels of a batch, built by the kernel across 160
    CTAs with atomics."""
    w = inputs.SCAN_WORKLOADS["m2p8b"]
    p, dy = _grad_inputs(w.batch, w.dim, w.dstate, w.seqlen, w.in_dtype, w.seed)
    _compare(_gpu_bwd(p, dy), _oracle_bwd(p, dy), p, w.in_dtype)


@pytest.mark.parametrize("shape,dtype", [((1, 64, 16, 40000), torch.bfloat16),
                                         ((2, 33, 5, 20000), torch.float32),
                                         ((1, 40, 16, 65536), torch.bfloat16),
                                         ((1, 24, 8, 131072), torch.float32)],
                         ids=lambda v: "x".join(map(str, v)) if isinstance(v, tuple) else str(v))
def test_backward_of_a_split_sequence(cuda_ok, shape, dtype):
    """Long sequences over few channels are swept in segments side by side: checkpoints
    from each segment's true start, the adjoint entering each segment from a summary pass
    and its fold (the last segment ragged here); every gradient against the oracle.  The
    last two shapes (L * N = 2^20) keep their checkpoints tile-major, with a partly filled
    tile (N = 8: element-wise staging of the states, 64-step blocks)."""
    b, d, N, L = shape
    ws = ops.selective_scan_bwd_workspace_size(b, d, N, L)
    ck = (b * -(-d // 32) * 32 * -(-L // 4) * N + 63) // 64 * 64 * 4  # the checkpoints alone
    assert ws > ck, "this shape should be swept in segments"
    p, dy = _grad_inputs(b, d, N, L, dtype, seed=L + d)
    _compare(_gpu_bwd(p, dy), _oracle_bwd(p, dy), p, dtype)
