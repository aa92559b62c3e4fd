"""The L-sharded scan's kernels on one GPU (needs a B200), ranks emulated in sequence.

Each building block against the fp64 oracle: the segment summary (the state after a
segment from zero, and its summed step), the fold of summaries (the state after several
segments, with and without a starting state), the scan from an initial state; then the
whole composition (summary per shard -> stacked as an all-gather would -> fold -> scan
per shard) against the oracle's unsplit scan, including shards long enough to be split
again inside the library and the exact-ZOH variant.  Emulating ranks in sequence runs no
kernels that wait on each other.  Tolerances as in s6_compare.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_56_b200 import inputs, ops, sharded
from tests.s6_compare import check_fp32, check_rms, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dev(p):
    return {k: (None if v is None else v.to(DEV)) for k, v in p.items()}


def _shard(p, lo, hi):
    out = dict(p)
    for k in ("u", "delta", "z", "B", "C"):
        if p[k] is not None:
            out[k] = p[k][:, :, lo:hi].contiguous()
    return out


@pytest.mark.parametrize("dtype,shape", [(torch.float32, (2, 24, 16, 150)),
                                         (torch.bfloat16, (1, 64, 16, 40000)),
                                         (torch.float32, (3, 10, 5, 33))])
def test_summary_matches_the_oracle(cuda_ok, dtype, shape):
    b, d, N, L = shape
    p = inputs.scan_inputs(b, d, N, L, dtype, seed=L + N)
    g = _dev(p)
    h_end, dsum = ops.selective_scan_summary(g["u"], g["delta"], g["A"], g["B"], g["C"],
                                             delta_bias=g["delta_bias"])
    torch.cuda.synchronize()
    _, h_ref = oracle.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"],
                                     delta_bias=p["delta_bias"])
    delta_ref, _ = oracle.discretize(to64(p["delta"]).reshape(b * d, L),
                                     np.tile(to64(p["A"]), (b, 1)),
                                     np.tile(to64(p["delta_bias"]), b))
    s_ref = delta_ref.sum(axis=1).reshape(b, d)
    if dtype == torch.float32 and L < 1000:
        check_fp32(h_end, h_ref, "h_end")
    else:
        check_rms(h_end, h_ref, "h_end")
    np.testing.assert_allclose(to64(dsum), s_ref, rtol=2e-5 if L < 1000 else 1e-4)


def test_fold_and_initial_state_match_the_oracle(cuda_ok):
    b, d, N, L, R = 2, 20, 16, 240, 3
    p = inputs.scan_inputs(b, d, N, L, torch.float32, seed=31)
    g = _dev(p)
    h0 = 0.3 * torch.randn(b, d, N, generator=torch.Generator().manual_seed(2))
    Ls = L // R
    hs, ss = [], []
    for r in range(R):
        q = _shard(g, r * Ls, (r + 1) * Ls)
        h, s = ops.selective_scan_summary(q["u"], q["delta"], q["A"], q["B"], q["C"],
                                          delta_bias=q["delta_bias"])
        hs.append(h)
        ss.append(s)
    H, S = torch.stack(hs), torch.stack(ss)
    # the state after all segments, from h0, equals the oracle's scan from h0
    h_all, s_all = ops.selective_scan_fold(H, S, g["A"], h0.to(DEV), return_delta_sum=True)
    _, h_ref = oracle.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"],
                                     delta_bias=p["delta_bias"], h0=h0)
    torch.cuda.synchronize()
    check_fp32(h_all, h_ref, "fold from h0")
    np.testing.assert_allclose(to64(s_all), to64(S).sum(0), rtol=1e-6)
    # count 0 returns the starting state
    h_same = ops.selective_scan_fold(H[:0], S[:0], g["A"], h0.to(DEV))
    torch.testing.assert_close(h_same.cpu(), h0, rtol=0, atol=0)
    # the scan from an initial state
    y, last = ops.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"],
                                     z=g["z"], delta_bias=g["delta_bias"], return_last_state=True,
                                     initial_state=h0.to(DEV))
    y_ref, last_ref = oracle.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"],
                                            z=p["z"], delta_bias=p["delta_bias"], h0=h0)
    torch.cuda.synchronize()
    check_fp32(y, y_ref, "y from h0")
    check_fp32(last, last_ref, "last_state from h0")


def _emulated_sharded_scan(p, R, exact_zoh=False, out_dtype=None):
    """Ranks 0..R-1 in sequence: summaries, stacked as the all-gather returns them, then
    every shard's fold + scan."""
    g = _dev(p)
    L = p["u"].shape[2]
    Ls = L // R
    bounds = [(r * Ls, (r + 1) * Ls if r < R - 1 else L) for r in range(R)]
    hs, ss = [], []
    for lo, hi in bounds:
        q = _shard(g, lo, hi)
        h, s = sharded.shard_summary(q["u"], q["delta"], q["A"], q["B"], q["C"], q["delta_bias"],
                                     exact_zoh=exact_zoh)
        hs.append(h)
        ss.append(s)
    H, S = torch.stack(hs), torch.stack(ss)
    ys, last = [], None
    for r, (lo, hi) in enumerate(bounds):
        q = _shard(g, lo, hi)
        y, last = sharded.shard_scan(r, H, S, q["u"], q["delta"], q["A"], q["B"], q["C"], D=q["D"],
                                     z=q["z"], delta_bias=q["delta_bias"], out_dtype=out_dtype,
                                     exact_zoh=exact_zoh)
        ys.append(y)
    torch.cuda.synchronize()
    return torch.cat(ys, dim=2), last


@pytest.mark.parametrize("R", [2, 3, 4])
def test_sharded_scan_fp32(cuda_ok, R):
    p = inputs.scan_inputs(2, 24, 16, 300, torch.float32, seed=40 + R)
    y, last = _emulated_sharded_scan(p, R)
    y_ref, last_ref = oracle.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"],
                                            z=p["z"], delta_bias=p["delta_bias"])
    check_fp32(y, y_ref, "y")
    check_fp32(last, last_ref, "last_state")


def test_sharded_scan_zoh(cuda_ok):
    p = inputs.scan_inputs(1, 16, 8, 200, torch.float32, seed=7)
    y, last = _emulated_sharded_scan(p, 4, exact_zoh=True)
    y_ref, last_ref = oracle.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"],
                                            z=p["z"], delta_bias=p["delta_bias"], zoh=True)
    check_fp32(y, y_ref, "y")
    check_fp32(last, last_ref, "last_state")


def test_sharded_long_sequence_with_inner_splits(cuda_ok):
    """(1, 2048, 16, 65536) bf16 over 4 shards of 16,384 steps: every shard is long enough
    (with few channels) for the library to split it again into segments, so the summary
    folds segment aggregates and the scan carries from the initial state.  Checked against
    the one-call GPU scan everywhere and against the oracle on 16 channels."""
    p = inputs.scan_inputs(1, 2048, 16, 65536, torch.bfloat16, seed=65536)
    assert ops.selective_scan_workspace_size(1, 2048, 16, 16384) > 0
    y, last = _emulated_sharded_scan(p, 4, out_dtype=torch.float32)
    g = _dev(p)
    y1, last1 = ops.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"],
                                       z=g["z"], delta_bias=g["delta_bias"],
                                       out_dtype=torch.float32, return_last_state=True)
    torch.cuda.synchronize()
    check_rms(y, to64(y1), "y vs one call")
    check_rms(last, to64(last1), "last_state vs one call")
    ch = np.sort(np.random.default_rng(4).choice(2048, 16, replace=False))
    sub = dict(p)
    for k in ("u", "delta", "z"):
        sub[k] = p[k][:, ch]
    sub["A"], sub["D"], sub["delta_bias"] = p["A"][ch], p["D"][ch], p["delta_bias"][ch]
    y_ref, last_ref = oracle.selective_scan(sub["u"], sub["delta"], sub["A"], sub["B"], sub["C"],
                                            D=sub["D"], z=sub["z"], delta_bias=sub["delta_bias"])
    check_rms(y[:, ch], y_ref, "y vs oracle")
    check_rms(last[:, ch], last_ref, "last_state vs oracle")
