"""The training path (needs a B200): a forward that records the backward's checkpoints
(mamba_selective_scan_fwd_train) and the backward that reads them
(mamba_selective_scan_bwd_from_checkpoints).  The forward's outputs must equal the plain
forward's bit for bit when the sequence is scanned in one pass; a sequence long enough to
be split is scanned by the plain forward in one pass over all segments from zero plus a
correction from each segment's true start, while the training forward rescans every
segment from its start (so its checkpoints are true states), and the two agree to
rounding.  The gradients must equal those of the recomputing backward:
bit for bit where no atomics are involved, when the sequence is scanned in one pass; dA,
dB, dC, dD and ddelta_bias are sums formed with atomics, whose order varies, so they are
compared to 1e-5 relative.  A sequence long enough to be split has its segment starts
folded from segment summaries in the training forward but recomputed straight through by
the backward's own pass, so the states -- and the gradients that depend on them -- agree
to rounding there (du, which depends on no state, still bit for bit)."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_56_b200 import inputs, ops
from tests.s6_compare import check_fp32, check_rms

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("shape,dtype", [((2, 40, 16, 200), torch.bfloat16),
                                         ((1, 64, 16, 40000), torch.bfloat16),  # split plan
                                         ((2, 33, 5, 130), torch.float32),      # 64-step blocks
                                         ((3, 24, 16, 77), torch.float32),      # ragged, no TMA
                                         ((1, 16, 16, 1), torch.float32)],
                         ids=lambda v: "x".join(map(str, v)) if isinstance(v, tuple) else str(v))
def test_training_forward_and_backward_match(cuda_ok, shape, dtype):
    b, d, N, L = shape
    p = inputs.scan_inputs(b, d, N, L, dtype, seed=L + d, device=DEV)
    gen = torch.Generator(device=DEV).manual_seed(3)
    dy = torch.randn(b, d, L, generator=gen, device=DEV).to(dtype)
    ck = torch.empty(ops.selective_scan_bwd_workspace_size(b, d, N, L), dtype=torch.uint8,
                     device=DEV)
    y_t, st_t = ops.selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"],
                                       z=p["z"], delta_bias=p["delta_bias"],
                                       return_last_state=True, checkpoints=ck)
    y_p, st_p = ops.selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"],
                                       z=p["z"], delta_bias=p["delta_bias"],
                                       return_last_state=True)
    torch.cuda.synchronize()
    split = ops.selective_scan_workspace_size(b, d, N, L) > 0
    if not split:
        assert torch.equal(y_t, y_p) and torch.equal(st_t, st_p)
    else:
        # Both are within the bf16-output bound of the exact result (2e-2 RMS + one ulp per
        # element); the plain forward rounds a bf16 y twice, first at the first pass's
        # value, which can exceed |y| where that value and the correction partly cancel.
        yt, yp = y_t.double(), y_p.double()
        mag = torch.maximum(yt.abs(), yp.abs()).clamp_min(2.0 ** -126)
        ulp = torch.exp2(torch.floor(torch.log2(mag)) - (7 if dtype == torch.bfloat16 else 23))
        tol = 2 * ulp + 2 * 2e-2 * yp.pow(2).mean().sqrt()
        assert bool(((yt - yp).abs() <= tol).all())
        torch.testing.assert_close(st_t, st_p, rtol=1e-4, atol=1e-6 * st_p.abs().max().item())
    g_c = ops.selective_scan_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"],
                                 z=p["z"], delta_bias=p["delta_bias"], checkpoints=ck)
    g_r = ops.selective_scan_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"],
                                 z=p["z"], delta_bias=p["delta_bias"])
    torch.cuda.synchronize()
    assert torch.equal(g_c["du"], g_r["du"])
    for k in ("ddelta", "dz"):
        if not split:
            assert torch.equal(g_c[k], g_r[k]), k
        else:  # within one unit of the output dtype's rounding of the larger value
            diff = (g_c[k].float() - g_r[k].float()).abs()
            tol = (g_r[k].float().abs() * (2.0 ** -7 if dtype == torch.bfloat16 else 1e-5) +
                   1e-6 * g_r[k].float().abs().max())
            assert bool((diff <= tol).all()), k
    for k in ("dA", "dB", "dC", "dD", "ddelta_bias"):
        torch.testing.assert_close(g_c[k], g_r[k], rtol=1e-4 if split else 1e-5,
                                   atol=1e-6 * g_r[k].abs().max().item())
    ops.check_device_error()


def test_training_forward_rejects_an_initial_state(cuda_ok):
    p = inputs.scan_inputs(1, 8, 16, 16, torch.float32, seed=1, device=DEV)
    ck = torch.empty(ops.selective_scan_bwd_workspace_size(1, 8, 16, 16), dtype=torch.uint8,
                     device=DEV)
    h0 = torch.zeros(1, 8, 16, device=DEV)
    with pytest.raises(ValueError):
        ops.selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], checkpoints=ck,
                               initial_state=h0)


@pytest.mark.parametrize("shape,dtype", [((2, 40, 16, 200), torch.float32),
                                         ((2, 24, 16, 77), torch.bfloat16),
                                         ((1, 64, 16, 40000), torch.bfloat16),  # split plan
                                         ((2, 33, 5, 130), torch.float32)],
                         ids=lambda v: "x".join(map(str, v)) if isinstance(v, tuple) else str(v))
def test_exact_zoh_training_pair(cuda_ok, shape, dtype):
    """The training pair with the exact-ZOH weight: the forward's outputs equal the exact-ZOH
    forward's (bit for bit in one pass; a split sequence's to the bf16-output bound, as for
    the Delta * B pair), and the gradients from its checkpoints equal the recomputing
    exact-ZOH backward's (du, ddelta, dz bit for bit in one pass; sums to 1e-5)."""
    b, d, N, L = shape
    p = inputs.scan_inputs(b, d, N, L, dtype, seed=L + d + 1, device=DEV)
    gen = torch.Generator(device=DEV).manual_seed(4)
    dy = torch.randn(b, d, L, generator=gen, device=DEV).to(dtype)
    ck = torch.empty(ops.selective_scan_bwd_workspace_size(b, d, N, L), dtype=torch.uint8,
                     device=DEV)
    kw = dict(D=p["D"], z=p["z"], delta_bias=p["delta_bias"], exact_zoh=True)
    y_t, st_t = ops.selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"],
                                       return_last_state=True, checkpoints=ck, **kw)
    y_p, st_p = ops.selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"],
                                       return_last_state=True, **kw)
    torch.cuda.synchronize()
    split = ops.selective_scan_workspace_size(b, d, N, L) > 0
    if not split:
        assert torch.equal(y_t, y_p) and torch.equal(st_t, st_p)
    else:
        yt, yp = y_t.double(), y_p.double()
        mag = torch.maximum(yt.abs(), yp.abs()).clamp_min(2.0 ** -126)
        ulp = torch.exp2(torch.floor(torch.log2(mag)) - (7 if dtype == torch.bfloat16 else 23))
        tol = 2 * ulp + 2 * 2e-2 * yp.pow(2).mean().sqrt()
        assert bool(((yt - yp).abs() <= tol).all())
        torch.testing.assert_close(st_t, st_p, rtol=1e-4, atol=1e-6 * st_p.abs().max().item())
    g_c = ops.selective_scan_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, checkpoints=ck,
                                 **kw)
    g_r = ops.selective_scan_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, **kw)
    torch.cuda.synchronize()
    for k in ("du", "ddelta", "dz"):
        if not split:
            assert torch.equal(g_c[k], g_r[k]), k
        else:
            diff = (g_c[k].float() - g_r[k].float()).abs()
            tol = (g_r[k].float().abs() * (2.0 ** -7 if dtype == torch.bfloat16 else 1e-5) +
                   1e-6 * g_r[k].float().abs().max())
            assert bool((diff <= tol).all()), k
    for k in ("dA", "dB", "dC", "dD", "ddelta_bias"):
        torch.testing.assert_close(g_c[k], g_r[k], rtol=1e-4 if split else 1e-5,
                                   atol=1e-6 * g_r[k].abs().max().item())
    ops.check_device_error()


@pytest.mark.parametrize("shape,dtype", [((2, 40, 16, 200), torch.float32),
                                         ((2, 24, 16, 77), torch.bfloat16),
                                         ((1, 70, 5, 130), torch.float32),
                                         ((1, 40, 16, 65536), torch.float32),
                                         ((1, 24, 8, 131072), torch.bfloat16)],
                         ids=lambda v: "x".join(map(str, v)) if isinstance(v, tuple) else str(v))
def test_checkpoints_are_the_group_entry_states(cuda_ok, shape, dtype):
    """The recorded checkpoints are the layout the header documents: the state entering
    every group of 4 steps, h_{4g-1} (zero for g = 0), fp32, per channel
    ([batch][dim][group][N]) while L * N < 2^20 and tile-major beyond ([batch][tile of 32
    channels][group][channel in tile][N]; the last shape, a split sequence).  Compared with
    the oracle's states under the last_state tolerances (fp32 inputs per element, bf16
    inputs against the RMS)."""
    b, d, N, L = shape
    p = inputs.scan_inputs(b, d, N, L, dtype, seed=4 * L + N)
    g = {k: (None if v is None else v.to(DEV)) for k, v in p.items()}
    ck = torch.zeros(ops.selective_scan_bwd_workspace_size(b, d, N, L), dtype=torch.uint8,
                     device=DEV)
    ops.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                           delta_bias=g["delta_bias"], checkpoints=ck)
    torch.cuda.synchronize()
    G = (L + 3) // 4
    if L * N >= 1 << 20:
        nt = (d + 31) // 32
        tiled = ck[: b * nt * G * 32 * N * 4].view(torch.float32).reshape(b, nt, G, 32, N)
        got = tiled.permute(0, 1, 3, 2, 4).reshape(b, nt * 32, G, N)[:, :d]
    else:
        got = ck[: b * d * G * N * 4].view(torch.float32).reshape(b, d, G, N)
    _, _, hs = oracle.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"],
                                     z=p["z"], delta_bias=p["delta_bias"], return_states=True)
    ref = np.zeros((b, d, G, N))
    ref[:, :, 1:, :] = hs[:, :, 3:4 * (G - 1):4, :]
    assert float(got[:, :, 0].abs().max()) == 0.0
    if dtype == torch.float32:
        check_fp32(got, ref, "checkpoints")
    else:
        check_rms(got, ref, "checkpoints")
