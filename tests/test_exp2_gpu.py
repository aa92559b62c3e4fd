"""The FMA-pipe 2^x the scan uses for part of its Abar factors, against fp64 and CUDA.

Bound: relative error <= 4e-7 (about 3 fp32 ulps) on the range the recurrence uses
(x = Delta * A * log2(e) <= 0, down to the clamp at -126), the same order as the
SFU's ex2.approx; checked against numpy's fp64 exp2 and against CUDA's exp2f.
"""
import numpy as np
import pytest
import torch

from selective_state_space_56_b200 import ops

pytestmark = pytest.mark.gpu


def test_exp2_polynomial_error_bound(cuda_ok):
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125.9, 0.0, 400001), -rng.exponential(2.0, 200000),
                        np.linspace(0.0, 20.0, 20001), [-0.5, 0.5, -1e-30, 0.0, -3.25]])
    x = x.astype(np.float32)
    f, s, lib = (t.cpu().numpy().astype(np.float64) for t in ops.diag_exp2(torch.from_numpy(x).cuda()))
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(f - ref) / ref
    assert rel.max() <= 4e-7, rel.max()
    rel_lib = np.abs(f - lib) / lib
    assert rel_lib.max() <= 4e-7, rel_lib.max()
    # same order as the SFU instruction it stands in for
    rel_sfu = np.abs(s - ref) / ref
    assert rel.max() <= 4 * max(rel_sfu.max(), 1e-7)


def test_exp2_polynomial_clamps(cuda_ok):
    x = torch.tensor([-1000.0, -200.0, -127.0, -126.0, 126.5, 127.0, 300.0], device="cuda")
    f, _, _ = ops.diag_exp2(x)
    f = f.cpu().numpy()
    assert (f[:4] >= 0).all() and (f[:4] < 1.2e-38).all()   # underflow stays tiny, never negative
    assert np.isfinite(f).all() and f[-1] == pytest.approx(2.0 ** 127, rel=1e-6)
