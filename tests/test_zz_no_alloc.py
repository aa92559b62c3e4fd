"""mamba_selective_scan_fwd_noalloc: the scan for callers that cannot allocate.

Callers such as plug-ins inside a framework that owns all device memory, or code
that cannot afford a synchronising cudaMalloc, get their segment scratch from a
fixed array inside the library.  These checks call the entry point through the C
ABI (ctypes, no Python wrapper) and compare it with mamba_selective_scan_fwd on the
same inputs, twice in a row, so a second call that reuses the array's old contents
is covered.  This file is collected last on purpose; it also passes on its own.
"""
import ctypes

import pytest
import torch

from selective_state_space_56_b200 import inputs, ops
from tests.s6_compare import check_bf16_out, check_fp32, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
ERR_WORKSPACE = -5


def _noalloc_fn():
    lib = ops.load_library()
    f = lib.mamba_selective_scan_fwd_noalloc
    vp = ctypes.c_void_p
    f.restype = ctypes.c_int
    f.argtypes = [vp] * 8 + [ctypes.c_int, vp, vp, ops.ScanDims, ctypes.c_int, ctypes.c_int, vp]
    return f


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(p, y, st, out_dtype):
    b, d, L = p["u"].shape
    n = p["A"].shape[1]
    f = _noalloc_fn()
    rc = f(_p(p["u"]), _p(p["delta"]), _p(p["A"]), _p(p["B"]), _p(p["C"]), _p(p["D"]), _p(p["z"]),
           _p(p["delta_bias"]), 1, _p(y), _p(st), ops.ScanDims(b, d, n, L),
           ops.MAMBA_BF16 if p["u"].dtype == torch.bfloat16 else ops.MAMBA_F32,
           ops.MAMBA_BF16 if out_dtype == torch.bfloat16 else ops.MAMBA_F32,
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc


@pytest.mark.parametrize("shape,in_dt,out_dt", [
    ((1, 64, 16, 16384 + 37), torch.bfloat16, torch.float32),   # split, unaligned rows
    ((2, 48, 16, 20480), torch.bfloat16, torch.bfloat16),       # split, TMA path
    ((1, 24, 8, 17000), torch.float32, torch.float32),          # split, N = 8
    ((2, 96, 16, 512), torch.bfloat16, torch.bfloat16),         # no split: no scratch used
])
def test_noalloc_matches_regular_entry_point_twice(cuda_ok, shape, in_dt, out_dt):
    b, d, n, L = shape
    ref_p = {k: (None if v is None else v.to(DEV)) for k, v in
             inputs.scan_inputs(b, d, n, L, in_dtype=in_dt, seed=900 + L).items()}
    y_ref, st_ref = ops.selective_scan_fwd(ref_p["u"], ref_p["delta"], ref_p["A"], ref_p["B"],
                                           ref_p["C"], D=ref_p["D"], z=ref_p["z"],
                                           delta_bias=ref_p["delta_bias"], out_dtype=out_dt,
                                           return_last_state=True)
    torch.cuda.synchronize()
    for call in range(2):
        y = torch.full((b, d, L), float("nan"), dtype=out_dt, device=DEV)
        st = torch.full((b, d, n), float("nan"), dtype=torch.float32, device=DEV)
        assert _noalloc(ref_p, y, st, out_dt) == 0, "call %d" % call
        torch.cuda.synchronize()
        if out_dt == torch.float32:
            check_fp32(y.cpu(), to64(y_ref.cpu()), "y, call %d" % call)
        else:
            check_bf16_out(y.cpu(), to64(y_ref.cpu()), "y, call %d" % call)
        check_fp32(st.cpu(), to64(st_ref.cpu()), "last_state, call %d" % call)
    ops.check_device_error(clear=True)


def test_noalloc_just_under_its_limit_is_bit_identical(cuda_ok):
    # 1 x 3300 channels, L = 40960: ten segments, 2.24 MB of scratch (95% of the array).
    b, d, n, L = 1, 3300, 16, 40960
    assert (9 << 18) * 0.9 < ops.selective_scan_workspace_size(b, d, n, L) <= (9 << 18)
    p = inputs.scan_inputs(b, d, n, L, in_dtype=torch.bfloat16, seed=905, device=DEV)
    y_ref, st_ref = ops.selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"],
                                           z=p["z"], delta_bias=p["delta_bias"],
                                           return_last_state=True)
    for call in range(2):
        y = torch.full_like(y_ref, float("nan"))
        st = torch.full_like(st_ref, float("nan"))
        assert _noalloc(p, y, st, torch.bfloat16) == 0, "call %d" % call
        torch.cuda.synchronize()
        # the same plan and kernels on the same inputs: identical bits
        assert torch.equal(y, y_ref), "y, call %d" % call
        assert torch.equal(st, st_ref), "last_state, call %d" % call
    ops.check_device_error(clear=True)


def test_noalloc_rejects_scratch_beyond_its_limit(cuda_ok):
    # 1 x 4095 channels, L = 65536: the split plan needs ~2.4 MiB > 2.25 MiB.
    assert ops.selective_scan_workspace_size(1, 4095, 16, 65536) > (9 << 18)
    small = torch.zeros(16, device=DEV)
    f = _noalloc_fn()
    rc = f(*([_p(small)] * 5), None, None, None, 1, _p(small), None, ops.ScanDims(1, 4095, 16, 65536),
           ops.MAMBA_BF16, ops.MAMBA_BF16, None)
    assert rc == ERR_WORKSPACE
