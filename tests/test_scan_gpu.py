"""Parity of the CUDA selective scan with the fp64 oracle (needs a B200).

Every call goes through the C ABI (``selective_state_space_56_b200.ops``).
Workloads: the tiny fp32 case, the 130M-shaped layer and the 2.8B-shaped layer
in full (the latter in the launch configuration the bench times); the
million-length scan at full size, checked on every channel of a 65,536-step
prefix and on 16 spot channels over the whole length; plus ragged, degenerate and
option-combination cases at sizes the oracle finishes in seconds.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_56_b200 import inputs, ops
from tests.s6_compare import check_bf16_out, check_fp32, check_rms, rms, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _to(p, device):
    return {k: (None if v is None else v.to(device)) for k, v in p.items()}


def _gpu_scan(p, out_dtype=None, softplus=True):
    g = _to(p, DEV)
    y, st = ops.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                                   delta_bias=g["delta_bias"], delta_softplus=softplus,
                                   out_dtype=out_dtype, return_last_state=True)
    torch.cuda.synchronize()
    return y, st


def _oracle_scan(p, softplus=True):
    return oracle.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                                 delta_bias=p["delta_bias"], softplus=softplus)


def _check(y, st, y_ref, st_ref, in_dtype, out_dtype):
    if out_dtype == torch.float32 and in_dtype == torch.float32:
        check_fp32(y, y_ref, "y")
        check_fp32(st, st_ref, "last_state")
    elif out_dtype == torch.float32:
        check_rms(y, y_ref, "y")
        check_rms(st, st_ref, "last_state")
    else:
        check_bf16_out(y, y_ref, "y")
        if in_dtype == torch.float32:
            check_fp32(st, st_ref, "last_state")
        else:
            check_rms(st, st_ref, "last_state")


def test_tiny_fp32_workload(cuda_ok):
    w = inputs.SCAN_WORKLOADS["tiny_fp32"]
    p = inputs.workload_inputs(w)
    y, st = _gpu_scan(p)
    y_ref, st_ref = _oracle_scan(p)
    assert y.dtype == torch.float32
    check_fp32(y, y_ref, "y")
    check_fp32(st, st_ref, "last_state")


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_m130m_workload_full(cuda_ok, out_dtype):
    w = inputs.SCAN_WORKLOADS["m130m"]
    p = inputs.workload_inputs(w)
    y, st = _gpu_scan(p, out_dtype=out_dtype)
    y_ref, st_ref = _oracle_scan(p)
    _check(y, st, y_ref, st_ref, w.in_dtype, out_dtype)


def test_m2p8b_workload_full(cuda_ok):
    """The 2.8B-shaped layer at full size, in the bench's launch configuration: every one
    of the 4 x 5120 x 4096 outputs and the whole final state against the oracle."""
    w = inputs.SCAN_WORKLOADS["m2p8b"]
    p = inputs.workload_inputs(w)
    y, st = _gpu_scan(p)
    y_ref, st_ref = _oracle_scan(p)
    stats = check_bf16_out(y, y_ref, "y")
    check_rms(st, st_ref, "last_state")
    assert stats["n"] == w.batch * w.dim * w.seqlen


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_single_wave_grid_with_producer_warps(cuda_ok, out_dtype):
    """A grid of one wave at about three CTAs per SM takes the form in which producer warps
    stage the chunks and form Delta and Delta u: here with a ragged channel tile (5000 =
    104 x 48 + 8) and a ragged last chunk (1000 = 31 x 32 + 8), every output checked."""
    b, d, n, L = 4, 5000, 16, 1000
    p = inputs.scan_inputs(b, d, n, L, in_dtype=torch.bfloat16, seed=4242)
    y, st = _gpu_scan(p, out_dtype=out_dtype)
    y_ref, st_ref = _oracle_scan(p)
    _check(y, st, y_ref, st_ref, torch.bfloat16, out_dtype)


def test_m2p8b_fp32_output_literal_bound(cuda_ok):
    """The same layer with fp32 y: the literal max|y - y_ref| <= 2e-2 RMS bound on every
    element."""
    w = inputs.SCAN_WORKLOADS["m2p8b"]
    p = inputs.workload_inputs(w)
    y, st = _gpu_scan(p, out_dtype=torch.float32)
    y_ref, st_ref = _oracle_scan(p)
    check_rms(y, y_ref, "y")
    check_rms(st, st_ref, "last_state")


def test_million_length_workload(cuda_ok):
    """Full 2^20-step run; every channel checked on a 65,536-step prefix, 16 seeded
    spot channels over the whole length and their final state."""
    w = inputs.SCAN_WORKLOADS["million"]
    torch.cuda.empty_cache()
    p = inputs.workload_inputs(w, device=DEV)
    y, st = ops.selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                                   delta_bias=p["delta_bias"], return_last_state=True)
    torch.cuda.synchronize()
    prefix = 1 << 16
    A = p["A"].cpu()
    D = p["D"].cpu()
    bias = p["delta_bias"].cpu()
    Bp = p["B"][:, :, :prefix].cpu()
    Cp = p["C"][:, :, :prefix].cpu()
    y_pre = y[0, :, :prefix].cpu()
    # the prefix's RMS over all channels scales the bound for every block
    refs = []
    for c0 in range(0, w.dim, 256):
        sl = slice(c0, c0 + 256)
        yr, _ = oracle.scan_lanes(p["u"][0, sl, :prefix].cpu(), p["delta"][0, sl, :prefix].cpu(),
                                  A[sl], Bp, Cp, np.zeros(256, int), D=D[sl],
                                  z=p["z"][0, sl, :prefix].cpu(), delta_bias=bias[sl])
        refs.append(yr)
    y_ref = np.concatenate(refs)
    check_bf16_out(y_pre, y_ref, "y[:, :65536]")
    rng = np.random.default_rng(56004)
    spots = sorted(rng.choice(w.dim, 16, replace=False).tolist())
    yr, hr = oracle.scan_lanes(p["u"][0, spots].cpu(), p["delta"][0, spots].cpu(), A[spots],
                               p["B"].cpu(), p["C"].cpu(), np.zeros(16, int), D=D[spots],
                               z=p["z"][0, spots].cpu(), delta_bias=bias[spots])
    check_bf16_out(y[0, spots].cpu(), yr, "y spot channels, full length")
    check_rms(st[0, spots].cpu(), hr, "final state, spot channels")
    del p, y, st
    torch.cuda.empty_cache()


EDGE_SHAPES = [
    (1, 1, 16, 1),       # one channel, one step
    (2, 33, 16, 63),     # ragged L (unaligned rows: element-wise staging), ragged channel tile
    (3, 70, 16, 200),    # aligned rows, chunk tail of 8 steps
    (1, 5, 1, 97),       # N = 1
    (2, 40, 4, 128),
    (2, 17, 8, 130),
    (1, 9, 12, 64),      # N not a power of two
    (1, 3, 6, 65),
    (2, 64, 16, 0),      # empty sequence: last_state = 0
]


@pytest.mark.parametrize("shape", EDGE_SHAPES)
@pytest.mark.parametrize("dtypes", [(torch.float32, torch.float32), (torch.bfloat16, torch.bfloat16),
                                    (torch.bfloat16, torch.float32), (torch.float32, torch.bfloat16)])
def test_edge_shapes(cuda_ok, shape, dtypes):
    b, d, n, L = shape
    in_dt, out_dt = dtypes
    p = inputs.scan_inputs(b, d, n, L, in_dtype=in_dt, seed=7 + sum(shape))
    y, st = _gpu_scan(p, out_dtype=out_dt)
    y_ref, st_ref = _oracle_scan(p)
    assert y.shape == (b, d, L) and st.shape == (b, d, n)
    if L == 0:
        assert torch.count_nonzero(st) == 0
        return
    _check(y, st, y_ref, st_ref, in_dt, out_dt)


@pytest.mark.parametrize("drop", ["z", "D", "delta_bias", "all"])
def test_optional_inputs_absent(cuda_ok, drop):
    p = inputs.scan_inputs(2, 48, 16, 192, in_dtype=torch.float32, seed=11)
    for k in (["z", "D", "delta_bias"] if drop == "all" else [drop]):
        p[k] = None
    y, st = _gpu_scan(p)
    y_ref, st_ref = _oracle_scan(p)
    check_fp32(y, y_ref, "y")
    check_fp32(st, st_ref, "last_state")


def test_softplus_off(cuda_ok):
    p = inputs.scan_inputs(2, 40, 16, 160, in_dtype=torch.float32, seed=12)
    g = torch.Generator().manual_seed(12)
    p["delta"] = 0.001 + 0.2 * torch.rand(p["delta"].shape, generator=g)  # positive raw steps
    p["delta_bias"] = torch.full_like(p["delta_bias"], 0.01)
    y, st = _gpu_scan(p, softplus=False)
    y_ref, st_ref = _oracle_scan(p, softplus=False)
    check_fp32(y, y_ref, "y")
    check_fp32(st, st_ref, "last_state")


def test_extreme_steps(cuda_ok):
    """Very negative raw steps (Delta -> 0: state kept) and very positive (forget)."""
    p = inputs.scan_inputs(1, 32, 16, 128, in_dtype=torch.float32, seed=13)
    d = p["delta"]
    d[:, :16] = -30.0
    d[:, 16:, ::2] = 30.0
    y, st = _gpu_scan(p)
    y_ref, st_ref = _oracle_scan(p)
    check_fp32(y, y_ref, "y")
    check_fp32(st, st_ref, "last_state")


@pytest.mark.parametrize("shape", [(1, 64, 16, 16384 + 37), (2, 48, 16, 20480), (1, 24, 8, 17000)])
def test_split_sequence(cuda_ok, shape):
    """Few channels and a long L take the three-launch split path."""
    b, d, n, L = shape
    assert ops.selective_scan_workspace_size(b, d, n, L) > 0
    p = inputs.scan_inputs(b, d, n, L, in_dtype=torch.bfloat16, seed=21 + L)
    y, st = _gpu_scan(p, out_dtype=torch.float32)
    y_ref, st_ref = _oracle_scan(p)
    check_rms(y, y_ref, "y")
    check_rms(st, st_ref, "last_state")


@pytest.mark.parametrize("case", ["bf16_out", "softplus_off", "positive_A", "fast_decay"])
def test_split_sequence_correction_cases(cuda_ok, case):
    """The one-pass split: every segment scanned from zero, then the input-free correction
    from each segment's true start.  The correction stops early only when the carried
    state can only decay (every A <= 0, softplus on); these cases cover the early stop
    (fast_decay, bf16_out), no early stop (softplus off, A > 0 in a few states) and a y
    rounded to bf16 twice (first pass, then first pass + correction)."""
    b, d, n, L = 2, 48, 16, 20480
    assert ops.selective_scan_workspace_size(b, d, n, L) > 0
    p = inputs.scan_inputs(b, d, n, L, in_dtype=torch.bfloat16, seed=77 + len(case))
    softplus = True
    out_dtype = torch.float32
    if case == "bf16_out":
        out_dtype = torch.bfloat16
    elif case == "softplus_off":
        softplus = False
        g = torch.Generator().manual_seed(5)
        p["delta"] = (0.02 * torch.rand(b, d, L, generator=g)).to(torch.bfloat16)  # Delta > 0
        p["delta_bias"] = torch.zeros(d)
    elif case == "positive_A":
        p["A"][::7, 0] = 1e-3   # a slowly growing state in every seventh channel
    elif case == "fast_decay":
        p["delta_bias"] = torch.full((d,), 2.0)  # Delta ~ 2: the start state is gone in ~20 steps
    y, st = _gpu_scan(p, out_dtype=out_dtype, softplus=softplus)
    y_ref, st_ref = _oracle_scan(p, softplus=softplus)
    if out_dtype == torch.bfloat16:
        check_bf16_out(y, y_ref, "y")
    else:
        check_rms(y, y_ref, "y")
    check_rms(st, st_ref, "last_state")


def test_deterministic_and_stream_ordered(cuda_ok):
    p = _to(inputs.scan_inputs(2, 96, 16, 512, seed=31), DEV)
    s = torch.cuda.Stream()
    outs = []
    for _ in range(2):
        with torch.cuda.stream(s):
            outs.append(ops.selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"],
                                               z=p["z"], delta_bias=p["delta_bias"]))
    s.synchronize()
    assert torch.equal(outs[0], outs[1])


def test_writes_stay_inside_outputs(cuda_ok):
    b, d, n, L = 2, 37, 16, 100
    p = _to(inputs.scan_inputs(b, d, n, L, seed=41), DEV)
    guard = 4096
    ybuf = torch.full((b * d * L + 2 * guard,), 7.0, dtype=torch.bfloat16, device=DEV)
    sbuf = torch.full((b * d * n + 2 * guard,), 7.0, dtype=torch.float32, device=DEV)
    y = ybuf[guard:guard + b * d * L].view(b, d, L)
    st = sbuf[guard:guard + b * d * n].view(b, d, n)
    ops.selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                           delta_bias=p["delta_bias"], y=y, last_state=st)
    torch.cuda.synchronize()
    for buf in (ybuf, sbuf):
        assert torch.all(buf[:guard] == 7.0) and torch.all(buf[-guard:] == 7.0)
    assert rms(to64(y)) > 0
