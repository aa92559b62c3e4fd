"""CPU-side checks of the C ABI: the library loads, exports every declared symbol,
and rejects bad arguments on the host before anything is launched.

No compute call is made here (there is no GPU): every call below fails
validation, which runs before the library touches the CUDA runtime.  Fake
pointers are small integers that are never dereferenced.
"""
import ctypes
import os
import re

import pytest

from selective_state_space_56_b200 import build as s6build
from selective_state_space_56_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, ERR_NULL, ERR_DIMS, ERR_ALIGN, ERR_DTYPE, ERR_WORKSPACE = 0, -1, -2, -3, -4, -5


@pytest.fixture(scope="module")
def lib():
    s6build.build()
    return ops.load_library()


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(mamba_\w+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert {"mamba_selective_scan_fwd", "mamba_selective_state_update",
            "mamba_selective_scan_workspace_size", "mamba_status_string"} <= set(names)
    for n in names:
        assert hasattr(lib, n), "symbol %s declared in include/ but not exported" % n


def test_built_for_sm100a_only():
    assert "arch=compute_100a,code=sm_100a" in " ".join(s6build.ARCH)


def test_status_strings(lib):
    for code in range(-8, 1):
        assert ops.status_string(code) and ops.status_string(code) != "unknown status"
    assert ops.status_string(-99) == "unknown status"
    assert lib.mamba_abi_version() >= 100


def _dims(b=2, d=64, n=16, L=128):
    return ops.ScanDims(b, d, n, L)


A16 = 16 * 1024  # a fake, 16-byte aligned, never dereferenced address


def _scan(lib, **kw):
    args = dict(u=A16, delta=A16, A=A16, B=A16, C=A16, D=None, z=None, bias=None, sp=1, y=A16,
                last=None, dims=_dims(), i=0, o=0, ws=None, wsb=0)
    args.update(kw)
    vp = lambda v: None if v is None else ctypes.c_void_p(v)  # noqa: E731
    return lib.mamba_selective_scan_fwd(
        vp(args["u"]), vp(args["delta"]), vp(args["A"]), vp(args["B"]), vp(args["C"]),
        vp(args["D"]), vp(args["z"]), vp(args["bias"]), args["sp"], vp(args["y"]),
        vp(args["last"]), args["dims"], args["i"], args["o"], vp(args["ws"]), args["wsb"], None)


@pytest.mark.parametrize("field", ["u", "delta", "A", "B", "C", "y"])
def test_scan_null_required_pointer(lib, field):
    assert _scan(lib, **{field: None}) == ERR_NULL


@pytest.mark.parametrize("dims", [(0, 64, 16, 8), (2, 0, 16, 8), (2, 64, 0, 8), (2, 64, 17, 8),
                                  (2, 64, 16, -1), (70000, 4, 16, 8), (1 << 40, 1 << 40, 16, 8)])
def test_scan_bad_dims(lib, dims):
    assert _scan(lib, dims=_dims(*dims)) == ERR_DIMS


@pytest.mark.parametrize("i,o", [(2, 0), (0, 7), (-1, 1)])
def test_scan_bad_dtype(lib, i, o):
    assert _scan(lib, i=i, o=o) == ERR_DTYPE


@pytest.mark.parametrize("field", ["u", "delta", "A", "B", "C", "D", "z", "bias", "y", "last"])
def test_scan_misaligned_pointer(lib, field):
    assert _scan(lib, **{field: A16 + 4}) == ERR_ALIGN


def test_scan_workspace_checks(lib):
    long_dims = _dims(1, 64, 16, 1 << 16)  # few channels, long L: the split plan needs scratch
    need = lib.mamba_selective_scan_workspace_size(long_dims)
    assert need > 0 and need % 256 == 0
    assert _scan(lib, dims=long_dims) == ERR_WORKSPACE
    assert _scan(lib, dims=long_dims, ws=A16, wsb=need - 1) == ERR_WORKSPACE
    assert _scan(lib, dims=long_dims, ws=A16 + 8, wsb=need) == ERR_ALIGN


def test_workspace_plan(lib):
    ws = lambda *d: lib.mamba_selective_scan_workspace_size(_dims(*d))  # noqa: E731
    assert ws(4, 5120, 16, 4096) == 0          # enough channels: one pass
    assert ws(8, 1536, 16, 2048) == 0
    assert ws(1, 2048, 16, 1 << 20) > 0        # million-length: split
    assert ws(1, 2048, 16, 1 << 20) < 64 << 20
    # the no-allocation entry point's fixed 2.25 MiB scratch covers the million-length layer
    assert ws(1, 2048, 16, 1 << 20) <= 9 << 18
    assert ws(1, 3300, 16, 40960) <= 9 << 18 < ws(1, 3300, 16, 40960) * 1.06  # just under it
    assert ws(0, 2048, 16, 1 << 20) == 0       # invalid dims report 0


def _upd(lib, **kw):
    args = dict(state=A16, u=A16, delta=A16, A=A16, B=A16, C=A16, D=None, z=None, bias=None,
                sp=1, y=A16, b=4, d=64, n=16, io=1)
    args.update(kw)
    vp = lambda v: None if v is None else ctypes.c_void_p(v)  # noqa: E731
    return lib.mamba_selective_state_update(
        vp(args["state"]), vp(args["u"]), vp(args["delta"]), vp(args["A"]), vp(args["B"]),
        vp(args["C"]), vp(args["D"]), vp(args["z"]), vp(args["bias"]), args["sp"], vp(args["y"]),
        args["b"], args["d"], args["n"], args["io"], None)


@pytest.mark.parametrize("field", ["state", "u", "delta", "A", "B", "C", "y"])
def test_update_null(lib, field):
    assert _upd(lib, **{field: None}) == ERR_NULL


def test_update_dims_dtype_align(lib):
    assert _upd(lib, b=0) == ERR_DIMS
    assert _upd(lib, n=17) == ERR_DIMS
    assert _upd(lib, d=-3) == ERR_DIMS
    assert _upd(lib, io=5) == ERR_DTYPE
    for f in ("state", "u", "delta", "A", "B", "C", "D", "z", "bias", "y"):
        assert _upd(lib, **{f: A16 + 2}) == ERR_ALIGN, f


def test_binding_rejects_cpu_tensors():
    import torch
    u = torch.zeros(1, 2, 8)
    with pytest.raises(ValueError):
        ops.selective_scan_fwd(u, u, torch.zeros(2, 4), torch.zeros(1, 4, 8), torch.zeros(1, 4, 8))


def _bwd(lib, **kw):
    args = dict(u=A16, delta=A16, A=A16, B=A16, C=A16, D=None, z=None, bias=None, sp=1, dy=A16,
                du=A16, ddelta=A16, dz=None, dA=A16, dB=A16, dC=A16, dD=None, dbias=None,
                dims=_dims(), i=1, ws=A16, wsb=1 << 30)
    args.update(kw)
    vp = lambda v: None if v is None else ctypes.c_void_p(v)  # noqa: E731
    names = ("u", "delta", "A", "B", "C", "D", "z", "bias")
    grads = ("dy", "du", "ddelta", "dz", "dA", "dB", "dC", "dD", "dbias")
    return lib.mamba_selective_scan_bwd(*[vp(args[n]) for n in names], args["sp"],
                                        *[vp(args[n]) for n in grads], args["dims"], args["i"],
                                        vp(args["ws"]), args["wsb"], None)


@pytest.mark.parametrize("field", ["u", "delta", "A", "B", "C", "dy", "du", "ddelta", "dA",
                                   "dB", "dC"])
def test_bwd_null_required_pointer(lib, field):
    assert _bwd(lib, **{field: None}) == ERR_NULL


@pytest.mark.parametrize("inp,grad", [("D", "dD"), ("z", "dz"), ("bias", "dbias")])
def test_bwd_gradient_present_iff_input_present(lib, inp, grad):
    assert _bwd(lib, **{inp: A16}) == ERR_NULL       # input without its gradient
    assert _bwd(lib, **{grad: A16}) == ERR_NULL      # gradient without its input


def test_bwd_dims_dtype_align_workspace(lib):
    assert _bwd(lib, dims=_dims(2, 64, 17, 8)) == ERR_DIMS
    assert _bwd(lib, i=3) == ERR_DTYPE
    for f in ("u", "delta", "A", "B", "C", "dy", "du", "ddelta", "dA", "dB", "dC"):
        assert _bwd(lib, **{f: A16 + 4}) == ERR_ALIGN, f
    need = lib.mamba_selective_scan_bwd_workspace_size(_dims())
    assert _bwd(lib, ws=None, wsb=0) == ERR_WORKSPACE
    assert _bwd(lib, wsb=need - 1) == ERR_WORKSPACE
    assert _bwd(lib, ws=A16 + 8, wsb=need) == ERR_ALIGN


def test_bwd_workspace_is_one_checkpoint_per_group(lib):
    ws = lambda *d: lib.mamba_selective_scan_bwd_workspace_size(_dims(*d))  # noqa: E731
    # the state entering every group of 4 steps, fp32, for every dstate; channels in tiles
    # of 32 (3 channels take one whole tile)
    assert ws(4, 5120, 16, 4096) == 4 * 5120 * 1024 * 16 * 4
    assert ws(2, 64, 16, 33) == 2 * 64 * 9 * 16 * 4
    assert ws(2, 64, 8, 64) == 2 * 64 * 16 * 8 * 4
    assert ws(1, 3, 5, 65) == (1 * 32 * 17 * 5 * 4 + 255) // 256 * 256
    assert ws(2, 40, 16, 8) == 2 * 64 * 2 * 16 * 4
    assert ws(2, 64, 16, 0) == 0
    assert ws(2, 64, 17, 8) == 0


def test_bwd_workspace_of_a_split_sequence(lib):
    """A long sequence over few channels is swept in segments: after the checkpoints
    (rounded up to 64 floats) the workspace holds each segment's adjoint summary and summed
    step, S x batch x dim x (N + 1) floats.  Without a GPU the plan assumes 148 SMs: the
    million-length layer (1, 2048, 16, 2^20) has 64 CTAs of 32 channels, so S = 740 // 64 = 11
    segments of 95,360 steps."""
    ws = lambda *d: lib.mamba_selective_scan_bwd_workspace_size(_dims(*d))  # noqa: E731
    b, d, N, L = 1, 2048, 16, 1 << 20
    ck = (b * d * (L // 4) * N + 63) // 64 * 64
    assert ws(b, d, N, L) == ((ck + 11 * b * d * (N + 1)) * 4 + 255) // 256 * 256
    # enough channels (640 CTAs for the 2.8B-shaped layer), or a short sequence: no split
    assert ws(4, 5120, 16, 1 << 15) == 4 * 5120 * (1 << 13) * 16 * 4
    assert ws(1, 64, 16, 8192) == 64 * 2048 * 16 * 4


ERR_FLAGS = -8


def test_ex_entry_points_reject_unknown_flags(lib):
    vp = lambda v: None if v is None else ctypes.c_void_p(v)  # noqa: E731
    scan_args = [vp(A16)] * 5 + [None, None, None, 1, vp(A16), None, _dims(), 0, 0, None, 0]
    for flags in (2, 0x80000000, 3):
        assert lib.mamba_selective_scan_fwd_ex(*scan_args, flags, None) == ERR_FLAGS
    # known flags go on to the ordinary checks
    assert lib.mamba_selective_scan_fwd_ex(*([None] + scan_args[1:]), 1, None) == ERR_NULL
    assert lib.mamba_selective_scan_fwd_ex(*scan_args[:11], _dims(2, 64, 17, 8), 0, 0, None, 0,
                                           1, None) == ERR_DIMS
    # the training pair's flags forms: unknown bits refused, known ones reach the usual checks
    need = lib.mamba_selective_scan_bwd_workspace_size(_dims())
    for flags in (2, 0x80000000):
        assert lib.mamba_selective_scan_fwd_train_ex(*scan_args, vp(A16), need, flags,
                                                     None) == ERR_FLAGS
    assert lib.mamba_selective_scan_fwd_train_ex(*scan_args, None, need, 1, None) == ERR_NULL
    assert lib.mamba_selective_scan_fwd_train_ex(*scan_args, vp(A16), need - 1, 1,
                                                 None) == ERR_WORKSPACE
    bw = [vp(A16)] * 5 + [None, None, None, 1] + [vp(A16)] * 3 + [None] + [vp(A16)] * 3 + \
        [None, None, _dims(), 1]
    assert lib.mamba_selective_scan_bwd_from_checkpoints_ex(*bw, vp(A16), need, 2,
                                                            None) == ERR_FLAGS
    assert lib.mamba_selective_scan_bwd_from_checkpoints_ex(*bw, vp(A16), need - 1, 1,
                                                            None) == ERR_WORKSPACE
    upd = [vp(A16)] * 6 + [None, None, None, 1, vp(A16), 4, 64, 16, 1]
    assert lib.mamba_selective_state_update_ex(*upd, 4, None) == ERR_FLAGS
    assert lib.mamba_selective_state_update_ex(*([None] + upd[1:]), 1, None) == ERR_NULL
    assert ops.status_string(ERR_FLAGS) == "unknown flag bits"


def _conv(lib, **kw):
    args = dict(x=A16, w=A16, bias=None, init=None, out=A16, fin=None, b=2, d=64, L=128, K=4,
                silu=1, dt=1)
    args.update(kw)
    vp = lambda v: None if v is None else ctypes.c_void_p(v)  # noqa: E731
    return lib.mamba_causal_conv1d_fwd(vp(args["x"]), vp(args["w"]), vp(args["bias"]),
                                       vp(args["init"]), vp(args["out"]), vp(args["fin"]),
                                       args["b"], args["d"], args["L"], args["K"], args["silu"],
                                       args["dt"], None)


def test_conv1d_host_checks(lib):
    for f in ("x", "w", "out"):
        assert _conv(lib, **{f: None}) == ERR_NULL, f
    for kw in (dict(K=0), dict(K=5), dict(b=0), dict(d=0), dict(L=-1)):
        assert _conv(lib, **kw) == ERR_DIMS, kw
    assert _conv(lib, dt=2) == ERR_DTYPE
    for f in ("x", "w", "bias", "init", "out", "fin"):
        assert _conv(lib, **{f: A16 + 2}) == ERR_ALIGN, f
    vp = ctypes.c_void_p
    upd = lib.mamba_causal_conv1d_update
    assert upd(None, vp(A16), vp(A16), None, vp(A16), 2, 64, 4, 1, 1, None) == ERR_NULL
    assert upd(vp(A16), vp(A16), vp(A16), None, vp(A16), 2, 64, 7, 1, 1, None) == ERR_DIMS
    assert upd(vp(A16), vp(A16), vp(A16), None, vp(A16), 70000, 4, 4, 1, 1, None) == ERR_DIMS
    assert upd(vp(A16), vp(A16 + 4), vp(A16), None, vp(A16), 2, 64, 4, 1, 1, None) == ERR_ALIGN


def test_diag_wait_timeout_rejects_bad_limits(lib):
    assert lib.mamba_diag_wait_timeout(0, None) == ERR_DIMS
    assert lib.mamba_diag_wait_timeout(-5, None) == ERR_DIMS
    assert lib.mamba_diag_wait_timeout(5_000_000_000, None) == ERR_DIMS


def test_diag_throughput_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    probe = lib.mamba_diag_throughput
    probe.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, vp, vp]
    assert probe(0, 8, 16, None, None) == ERR_NULL
    for kind, blocks, iters in ((3, 8, 16), (-1, 8, 16), (0, 0, 16), (0, 1 << 21, 16),
                                (0, 8, 0), (0, 8, 1 << 25), (0, 1 << 20, 1 << 9),
                                (1, 1 << 5, 1 << 24)):  # the last two: blocks x iters > 2^28
        assert probe(kind, blocks, iters, vp(A16), None) == ERR_DIMS, (kind, blocks, iters)


def test_diag_throughput_binding_checks_its_sink():
    import torch
    with pytest.raises(ValueError):
        ops.diag_throughput("sfu_ex2", 1, 1, torch.empty(256))  # host tensor
    with pytest.raises(KeyError):
        ops.diag_throughput("dfma", 1, 1, torch.empty(256))
    assert set(ops.THROUGHPUT_KINDS) == {"sfu_ex2", "ffma", "ffma2"}


def test_training_entry_points_check_the_checkpoint_buffer(lib):
    vp = ctypes.c_void_p
    need = lib.mamba_selective_scan_bwd_workspace_size(_dims())
    base = [vp(A16)] * 5 + [None, None, None, 1, vp(A16), None, _dims(), 0, 0, None, 0]
    assert lib.mamba_selective_scan_fwd_train(*base, None, 0, None) == ERR_NULL
    assert lib.mamba_selective_scan_fwd_train(*base, vp(A16), need - 1, None) == ERR_WORKSPACE
    assert lib.mamba_selective_scan_fwd_train(*base, vp(A16 + 8), need, None) == ERR_ALIGN
    bw = [vp(A16)] * 5 + [None, None, None, 1] + [vp(A16)] * 3 + [None] + [vp(A16)] * 3 + \
        [None, None, _dims(), 1]
    assert lib.mamba_selective_scan_bwd_from_checkpoints(*bw, vp(A16), need - 1, None) == \
        ERR_WORKSPACE
    assert lib.mamba_selective_scan_bwd_from_checkpoints(*bw, None, need, None) == ERR_WORKSPACE
