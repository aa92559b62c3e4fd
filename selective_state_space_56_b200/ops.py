"""Thin ctypes binding over the C ABI in include/mamba_s6.h (argument marshalling only).

Every function here checks that its tensors sit on one CUDA device with the
layouts the ABI expects, allocates any output the caller did not pass (with
torch), and forwards raw device pointers plus the current torch stream to
``libmamba_s6.so``.  All arithmetic runs in the library's CUDA kernels; there is
no fallback: if the library is missing or the ABI rejects the call, a
``MambaError`` is raised.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmamba_s6.so")

MAMBA_F32, MAMBA_BF16 = 0, 1
MAMBA_FLAG_EXACT_ZOH = 1
_DTYPES = {torch.float32: MAMBA_F32, torch.bfloat16: MAMBA_BF16}


class MambaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (where, status_string(status), status))


class ScanDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("dim", ctypes.c_int64), ("dstate", ctypes.c_int64),
                ("seqlen", ctypes.c_int64)]


_lock = threading.Lock()
_lib = None


def load_library():
    """Load libmamba_s6.so (build it first with ``python -m selective_state_space_56_b200.build``)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError("libmamba_s6.so is not built (run: python -m "
                                  "selective_state_space_56_b200.build)")
            lib = ctypes.CDLL(LIB_PATH)
            vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
            lib.mamba_selective_scan_workspace_size.restype = ctypes.c_size_t
            lib.mamba_selective_scan_workspace_size.argtypes = [ScanDims]
            lib.mamba_selective_scan_fwd.restype = i32
            lib.mamba_selective_scan_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp,
                                                     ScanDims, i32, i32, vp, ctypes.c_size_t, vp]
            lib.mamba_selective_scan_bwd_workspace_size.restype = ctypes.c_size_t
            lib.mamba_selective_scan_bwd_workspace_size.argtypes = [ScanDims]
            lib.mamba_selective_scan_bwd.restype = i32
            lib.mamba_selective_scan_bwd.argtypes = [vp] * 8 + [i32] + [vp] * 9 + [
                ScanDims, i32, vp, ctypes.c_size_t, vp]
            lib.mamba_selective_scan_bwd_ex.restype = i32
            lib.mamba_selective_scan_bwd_ex.argtypes = [vp] * 8 + [i32] + [vp] * 9 + [
                ScanDims, i32, vp, ctypes.c_size_t, ctypes.c_uint, vp]
            u32 = ctypes.c_uint
            lib.mamba_selective_scan_fwd_ex.restype = i32
            lib.mamba_selective_scan_fwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, vp,
                                                        vp, ScanDims, i32, i32, vp,
                                                        ctypes.c_size_t, u32, vp]
            lib.mamba_selective_scan_fwd_train.restype = i32
            lib.mamba_selective_scan_fwd_train.argtypes = [vp] * 8 + [i32, vp, vp, ScanDims, i32,
                                                               i32, vp, ctypes.c_size_t, vp,
                                                               ctypes.c_size_t, vp]
            lib.mamba_selective_scan_bwd_from_checkpoints.restype = i32
            lib.mamba_selective_scan_bwd_from_checkpoints.argtypes = [vp] * 8 + [i32] + [vp] * 9 + [
                ScanDims, i32, vp, ctypes.c_size_t, vp]
            lib.mamba_selective_scan_fwd_train_ex.restype = i32
            lib.mamba_selective_scan_fwd_train_ex.argtypes = [vp] * 8 + [
                i32, vp, vp, ScanDims, i32, i32, vp, ctypes.c_size_t, vp, ctypes.c_size_t, u32, vp]
            lib.mamba_selective_scan_bwd_from_checkpoints_ex.restype = i32
            lib.mamba_selective_scan_bwd_from_checkpoints_ex.argtypes = [vp] * 8 + [i32] + [vp] * 9 + [
                ScanDims, i32, vp, ctypes.c_size_t, u32, vp]
            lib.mamba_selective_scan_fwd_init.restype = i32
            lib.mamba_selective_scan_fwd_init.argtypes = [vp] * 8 + [i32] + [vp] * 3 + [
                ScanDims, i32, i32, vp, ctypes.c_size_t, u32, vp]
            lib.mamba_selective_scan_summary.restype = i32
            lib.mamba_selective_scan_summary.argtypes = [vp] * 6 + [i32, vp, vp, ScanDims, i32, vp,
                                                                 ctypes.c_size_t, u32, vp]
            lib.mamba_selective_scan_fold.restype = i32
            lib.mamba_selective_scan_fold.argtypes = [vp] * 4 + [i64] * 4 + [vp, vp, vp]
            lib.mamba_selective_state_update_ex.restype = i32
            lib.mamba_selective_state_update_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                                            i32, vp, i64, i64, i64, i32, u32, vp]
            lib.mamba_causal_conv1d_fwd.restype = i32
            lib.mamba_causal_conv1d_fwd.argtypes = [vp] * 6 + [i64, i64, i64, i32, i32, i32, vp]
            lib.mamba_causal_conv1d_update.restype = i32
            lib.mamba_causal_conv1d_update.argtypes = [vp] * 5 + [i64, i64, i32, i32, i32, vp]
            lib.mamba_causal_conv1d_bwd.restype = i32
            lib.mamba_causal_conv1d_bwd.argtypes = [vp] * 9 + [i64, i64, i64, i32, i32, i32, vp]
            lib.mamba_selective_state_update.restype = i32
            lib.mamba_selective_state_update.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32,
                                                         vp, i64, i64, i64, i32, vp]
            lib.mamba_status_string.restype = ctypes.c_char_p
            lib.mamba_status_string.argtypes = [i32]
            lib.mamba_check_device_error.restype = i32
            lib.mamba_check_device_error.argtypes = [i32, vp]
            lib.mamba_diag_wait_timeout.restype = i32
            lib.mamba_diag_wait_timeout.argtypes = [i64, vp]
            lib.mamba_diag_exp2.restype = i32
            lib.mamba_diag_exp2.argtypes = [vp, vp, vp, vp, i64, vp]
            lib.mamba_diag_throughput.restype = i32
            lib.mamba_diag_throughput.argtypes = [i32, i64, i64, vp, vp]
            lib.mamba_abi_version.restype = i32
            lib.mamba_abi_version.argtypes = []
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    try:
        return load_library().mamba_status_string(int(status)).decode()
    except ImportError:
        return "status %d" % status


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(t, name, device, shape=None, dtypes=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError("%s has dtype %s, expected one of %s" % (name, t.dtype, dtypes))


def check_device_error(clear: bool = True, device=None) -> None:
    """Raise MambaError if a bounded device-side wait gave up since the last clear."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        rc = load_library().mamba_check_device_error(int(bool(clear)), _stream_handle(dev))
    if rc != 0:
        raise MambaError(rc, "mamba_check_device_error")


def diag_wait_timeout(limit_cycles: int = 2_000_000, device=None) -> None:
    """Launch one bounded device wait that nothing completes (it gives up after
    limit_cycles SM clocks and sets the device error word); for testing detection."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        rc = load_library().mamba_diag_wait_timeout(int(limit_cycles), _stream_handle(dev))
    if rc != 0:
        raise MambaError(rc, "mamba_diag_wait_timeout")


def diag_exp2(x):
    """2^x of a float32 CUDA tensor via (FMA-pipe polynomial, SFU ex2.approx, exp2f)."""
    if x.dtype != torch.float32 or x.device.type != "cuda" or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 CUDA tensor")
    outs = [torch.empty_like(x) for _ in range(3)]
    with torch.cuda.device(x.device):
        rc = load_library().mamba_diag_exp2(_ptr(x), _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]),
                                            x.numel(), _stream_handle(x.device))
    if rc != 0:
        raise MambaError(rc, "mamba_diag_exp2")
    return tuple(outs)


THROUGHPUT_KINDS = {"sfu_ex2": 0, "ffma": 1, "ffma2": 2}


def diag_throughput(kind: str, blocks: int, iters: int, sink):
    """Launch the pipe-throughput probe (kind "sfu_ex2", "ffma" or "ffma2") on the current
    stream; sink is a float32 CUDA tensor of at least blocks * 256 elements.  Returns the
    number of fp32 results the launch computes (the caller times it)."""
    k = THROUGHPUT_KINDS[kind]
    if sink.dtype != torch.float32 or sink.device.type != "cuda" or sink.numel() < blocks * 256:
        raise ValueError("sink must be a float32 CUDA tensor of at least blocks * 256 elements")
    with torch.cuda.device(sink.device):
        rc = load_library().mamba_diag_throughput(k, int(blocks), int(iters), _ptr(sink),
                                                  _stream_handle(sink.device))
    if rc != 0:
        raise MambaError(rc, "mamba_diag_throughput")
    return blocks * 256 * iters * (16 if k == 2 else 8)


def selective_scan_workspace_size(batch: int, dim: int, dstate: int, seqlen: int) -> int:
    """Bytes of workspace ``mamba_selective_scan_fwd`` needs for these sizes (0 if none)."""
    return int(load_library().mamba_selective_scan_workspace_size(
        ScanDims(batch, dim, dstate, seqlen)))


def selective_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
                       out_dtype=None, y=None, last_state=None, return_last_state=False,
                       workspace=None, exact_zoh=False, initial_state=None, checkpoints=None):
    """Fused selective scan.  u, delta, z: (batch, dim, L); A: (dim, N) fp32;
    B, C: (batch, N, L); D, delta_bias: (dim) fp32.  Returns y (batch, dim, L)
    [and last_state (batch, dim, N) fp32].  exact_zoh: Bbar = (exp(Delta A) - 1) / A * B
    instead of Delta * B.  initial_state: (batch, dim, N) fp32 state before the sequence
    (zero when None).  checkpoints: a uint8 CUDA tensor of at least
    selective_scan_bwd_workspace_size(...) bytes to record the backward's checkpoints in
    (a training forward, also with exact_zoh; not with initial_state)."""
    if not isinstance(u, torch.Tensor) or u.dim() != 3:
        raise ValueError("u must be a (batch, dim, L) tensor")
    dev = u.device
    if dev.type != "cuda":
        raise ValueError("selective_scan_fwd runs on CUDA tensors only")
    b, d, L = u.shape
    N = A.shape[1] if A.dim() == 2 else -1
    in_dt = u.dtype
    if in_dt not in _DTYPES:
        raise ValueError("unsupported input dtype %s" % in_dt)
    out_dt = in_dt if out_dtype is None else out_dtype
    if out_dt not in _DTYPES:
        raise ValueError("unsupported output dtype %s" % out_dt)
    _check(u, "u", dev, (b, d, L), (in_dt,))
    _check(delta, "delta", dev, (b, d, L), (in_dt,))
    _check(z, "z", dev, (b, d, L), (in_dt,))
    _check(A, "A", dev, (d, N), (torch.float32,))
    _check(B, "B", dev, (b, N, L), (in_dt,))
    _check(C, "C", dev, (b, N, L), (in_dt,))
    _check(D, "D", dev, (d,), (torch.float32,))
    _check(delta_bias, "delta_bias", dev, (d,), (torch.float32,))
    if y is None:
        y = torch.empty((b, d, L), dtype=out_dt, device=dev)
    _check(y, "y", dev, (b, d, L), (out_dt,))
    if last_state is None and return_last_state:
        last_state = torch.empty((b, d, N), dtype=torch.float32, device=dev)
    _check(last_state, "last_state", dev, (b, d, N), (torch.float32,))
    _check(initial_state, "initial_state", dev, (b, d, N), (torch.float32,))
    lib = load_library()
    dims = ScanDims(b, d, N, L)
    need = int(lib.mamba_selective_scan_workspace_size(dims))
    if need > 0 and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    args = (_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
            int(bool(delta_softplus)), _ptr(y), _ptr(last_state), dims, _DTYPES[in_dt],
            _DTYPES[out_dt], _ptr(workspace), ws_bytes)
    flags = MAMBA_FLAG_EXACT_ZOH if exact_zoh else 0
    if checkpoints is not None and initial_state is not None:
        raise ValueError("checkpoints are recorded by a forward from h = 0 only")
    with torch.cuda.device(dev):
        if checkpoints is not None:
            _check(checkpoints, "checkpoints", dev)
            rc = lib.mamba_selective_scan_fwd_train_ex(
                *args, _ptr(checkpoints), checkpoints.numel() * checkpoints.element_size(),
                flags, _stream_handle(dev))
        elif initial_state is not None:
            rc = lib.mamba_selective_scan_fwd_init(*args[:9], _ptr(initial_state), *args[9:], flags,
                                                   _stream_handle(dev))
        elif exact_zoh:
            rc = lib.mamba_selective_scan_fwd_ex(*args, flags, _stream_handle(dev))
        else:
            rc = lib.mamba_selective_scan_fwd(*args, _stream_handle(dev))
    if rc != 0:
        raise MambaError(rc, "mamba_selective_scan_fwd")
    if return_last_state:
        return y, last_state
    return y


def selective_scan_bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None,
                       delta_softplus=True, workspace=None, checkpoints=None, exact_zoh=False):
    """Gradients of ``selective_scan_fwd`` for the upstream gradient dy (batch, dim, L),
    in the inputs' dtype.  Returns a dict with du, ddelta, dz (input dtype, dz None
    without a gate), dA (dim, N), dB, dC (batch, N, L), dD, ddelta_bias (dim) in fp32
    (None where the input is None).  checkpoints: the buffer a training forward
    (selective_scan_fwd(..., checkpoints=...)) filled for the same inputs; the backward
    then skips its own checkpointing pass (with the exact_zoh the forward used).
    exact_zoh: the gradients of the exact zero-order-hold forward
    (``selective_scan_fwd(..., exact_zoh=True)``)."""
    if not isinstance(u, torch.Tensor) or u.dim() != 3:
        raise ValueError("u must be a (batch, dim, L) tensor")
    dev = u.device
    if dev.type != "cuda":
        raise ValueError("selective_scan_bwd runs on CUDA tensors only")
    b, d, L = u.shape
    N = A.shape[1] if A.dim() == 2 else -1
    dt = u.dtype
    if dt not in _DTYPES:
        raise ValueError("unsupported input dtype %s" % dt)
    for t, name, shape, dts in ((u, "u", (b, d, L), (dt,)), (delta, "delta", (b, d, L), (dt,)),
                                (z, "z", (b, d, L), (dt,)), (dy, "dy", (b, d, L), (dt,)),
                                (A, "A", (d, N), (torch.float32,)), (B, "B", (b, N, L), (dt,)),
                                (C, "C", (b, N, L), (dt,)), (D, "D", (d,), (torch.float32,)),
                                (delta_bias, "delta_bias", (d,), (torch.float32,))):
        _check(t, name, dev, shape, dts)
    f32 = torch.float32
    g = dict(du=torch.empty((b, d, L), dtype=dt, device=dev),
             ddelta=torch.empty((b, d, L), dtype=dt, device=dev),
             dz=None if z is None else torch.empty((b, d, L), dtype=dt, device=dev),
             dA=torch.empty((d, N), dtype=f32, device=dev),
             dB=torch.empty((b, N, L), dtype=f32, device=dev),
             dC=torch.empty((b, N, L), dtype=f32, device=dev),
             dD=None if D is None else torch.empty(d, dtype=f32, device=dev),
             ddelta_bias=None if delta_bias is None else torch.empty(d, dtype=f32, device=dev))
    lib = load_library()
    dims = ScanDims(b, d, N, L)
    if checkpoints is not None:
        _check(checkpoints, "checkpoints", dev)
        with torch.cuda.device(dev):
            rc = lib.mamba_selective_scan_bwd_from_checkpoints_ex(
                _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                _ptr(delta_bias), int(bool(delta_softplus)), _ptr(dy), _ptr(g["du"]),
                _ptr(g["ddelta"]), _ptr(g["dz"]), _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]),
                _ptr(g["dD"]), _ptr(g["ddelta_bias"]), dims, _DTYPES[dt], _ptr(checkpoints),
                checkpoints.numel() * checkpoints.element_size(),
                MAMBA_FLAG_EXACT_ZOH if exact_zoh else 0, _stream_handle(dev))
        if rc != 0:
            raise MambaError(rc, "mamba_selective_scan_bwd_from_checkpoints")
        return g
    need = int(lib.mamba_selective_scan_bwd_workspace_size(dims))
    if need > 0 and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        rc = lib.mamba_selective_scan_bwd_ex(
            _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
            int(bool(delta_softplus)), _ptr(dy), _ptr(g["du"]), _ptr(g["ddelta"]), _ptr(g["dz"]),
            _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dD"]), _ptr(g["ddelta_bias"]),
            dims, _DTYPES[dt], _ptr(workspace), ws_bytes,
            MAMBA_FLAG_EXACT_ZOH if exact_zoh else 0, _stream_handle(dev))
    if rc != 0:
        raise MambaError(rc, "mamba_selective_scan_bwd_ex")
    return g


def selective_scan_bwd_workspace_size(batch: int, dim: int, dstate: int, seqlen: int) -> int:
    """Bytes of workspace ``mamba_selective_scan_bwd`` needs (the chunk checkpoints)."""
    return int(load_library().mamba_selective_scan_bwd_workspace_size(
        ScanDims(batch, dim, dstate, seqlen)))


def selective_state_update(state, u, delta, A, B, C, D=None, z=None, delta_bias=None,
                           delta_softplus=True, y=None, exact_zoh=False):
    """One decode token, in place on ``state`` (batch, dim, N) fp32.
    u, delta, z: (batch, dim); B, C: (batch, N); A: (dim, N).  Returns y (batch, dim).
    exact_zoh: Bbar = (exp(Delta A) - 1) / A * B instead of Delta * B."""
    if not isinstance(state, torch.Tensor) or state.dim() != 3:
        raise ValueError("state must be a (batch, dim, N) tensor")
    dev = state.device
    if dev.type != "cuda":
        raise ValueError("selective_state_update runs on CUDA tensors only")
    b, d, N = state.shape
    io_dt = u.dtype
    if io_dt not in _DTYPES:
        raise ValueError("unsupported dtype %s" % io_dt)
    _check(state, "state", dev, (b, d, N), (torch.float32,))
    _check(u, "u", dev, (b, d), (io_dt,))
    _check(delta, "delta", dev, (b, d), (io_dt,))
    _check(z, "z", dev, (b, d), (io_dt,))
    _check(A, "A", dev, (d, N), (torch.float32,))
    _check(B, "B", dev, (b, N), (io_dt,))
    _check(C, "C", dev, (b, N), (io_dt,))
    _check(D, "D", dev, (d,), (torch.float32,))
    _check(delta_bias, "delta_bias", dev, (d,), (torch.float32,))
    if y is None:
        y = torch.empty((b, d), dtype=io_dt, device=dev)
    _check(y, "y", dev, (b, d), (io_dt,))
    args = (_ptr(state), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
            _ptr(delta_bias), int(bool(delta_softplus)), _ptr(y), b, d, N, _DTYPES[io_dt])
    lib = load_library()
    with torch.cuda.device(dev):
        if exact_zoh:
            rc = lib.mamba_selective_state_update_ex(*args, MAMBA_FLAG_EXACT_ZOH,
                                                     _stream_handle(dev))
        else:
            rc = lib.mamba_selective_state_update(*args, _stream_handle(dev))
    if rc != 0:
        raise MambaError(rc, "mamba_selective_state_update")
    return y


def causal_conv1d_fwd(x, weight, bias=None, initial_state=None, silu=True, out=None,
                      return_final_state=False):
    """Causal depthwise conv1d (+ SiLU).  x: (batch, dim, L) bf16/fp32; weight: (dim, K)
    fp32, 1 <= K <= 4; bias: (dim) fp32; initial_state: (batch, dim, K-1) x.dtype.
    Returns out (batch, dim, L) [and the final state (batch, dim, K-1)]."""
    if not isinstance(x, torch.Tensor) or x.dim() != 3:
        raise ValueError("x must be a (batch, dim, L) tensor")
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("causal_conv1d_fwd runs on CUDA tensors only")
    b, d, L = x.shape
    K = weight.shape[1] if weight.dim() == 2 else -1
    dt = x.dtype
    if dt not in _DTYPES:
        raise ValueError("unsupported dtype %s" % dt)
    _check(x, "x", dev, (b, d, L), (dt,))
    _check(weight, "weight", dev, (d, K), (torch.float32,))
    _check(bias, "bias", dev, (d,), (torch.float32,))
    _check(initial_state, "initial_state", dev, (b, d, K - 1), (dt,))
    if out is None:
        out = torch.empty((b, d, L), dtype=dt, device=dev)
    _check(out, "out", dev, (b, d, L), (dt,))
    fin = None
    if return_final_state and K > 1:
        fin = torch.empty((b, d, K - 1), dtype=dt, device=dev)
    with torch.cuda.device(dev):
        rc = load_library().mamba_causal_conv1d_fwd(
            _ptr(x), _ptr(weight), _ptr(bias), _ptr(initial_state), _ptr(out), _ptr(fin),
            b, d, L, K, int(bool(silu)), _DTYPES[dt], _stream_handle(dev))
    if rc != 0:
        raise MambaError(rc, "mamba_causal_conv1d_fwd")
    if return_final_state:
        return out, fin
    return out


def causal_conv1d_update(conv_state, x, weight, bias=None, silu=True, out=None):
    """One decode token: conv_state (batch, dim, K-1) is updated in place; x (batch, dim).
    Returns out (batch, dim)."""
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise ValueError("x must be a (batch, dim) tensor")
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("causal_conv1d_update runs on CUDA tensors only")
    b, d = x.shape
    K = weight.shape[1] if weight.dim() == 2 else -1
    dt = x.dtype
    if dt not in _DTYPES:
        raise ValueError("unsupported dtype %s" % dt)
    _check(x, "x", dev, (b, d), (dt,))
    _check(weight, "weight", dev, (d, K), (torch.float32,))
    _check(bias, "bias", dev, (d,), (torch.float32,))
    _check(conv_state, "conv_state", dev, (b, d, K - 1), (dt,))
    if out is None:
        out = torch.empty((b, d), dtype=dt, device=dev)
    _check(out, "out", dev, (b, d), (dt,))
    with torch.cuda.device(dev):
        rc = load_library().mamba_causal_conv1d_update(
            _ptr(conv_state), _ptr(x), _ptr(weight), _ptr(bias), _ptr(out), b, d, K,
            int(bool(silu)), _DTYPES[dt], _stream_handle(dev))
    if rc != 0:
        raise MambaError(rc, "mamba_causal_conv1d_update")
    return out


def causal_conv1d_bwd(x, weight, dout, bias=None, initial_state=None, silu=True):
    """Gradients of sum(out * dout) for ``causal_conv1d_fwd`` with the same x, weight, bias,
    initial_state and silu.  Returns a dict: dx (batch, dim, L) x.dtype, dweight (dim, K)
    fp32, dbias (dim) fp32 (None without a bias), dinitial_state (batch, dim, K-1) x.dtype
    (None without an initial state)."""
    if not isinstance(x, torch.Tensor) or x.dim() != 3:
        raise ValueError("x must be a (batch, dim, L) tensor")
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("causal_conv1d_bwd runs on CUDA tensors only")
    b, d, L = x.shape
    K = weight.shape[1] if weight.dim() == 2 else -1
    dt = x.dtype
    if dt not in _DTYPES:
        raise ValueError("unsupported dtype %s" % dt)
    _check(x, "x", dev, (b, d, L), (dt,))
    _check(dout, "dout", dev, (b, d, L), (dt,))
    _check(weight, "weight", dev, (d, K), (torch.float32,))
    _check(bias, "bias", dev, (d,), (torch.float32,))
    _check(initial_state, "initial_state", dev, (b, d, K - 1), (dt,))
    g = dict(dx=torch.empty((b, d, L), dtype=dt, device=dev),
             dweight=torch.empty((d, K), dtype=torch.float32, device=dev),
             dbias=None if bias is None else torch.empty(d, dtype=torch.float32, device=dev),
             dinitial_state=None if (initial_state is None or K < 2)
             else torch.empty((b, d, K - 1), dtype=dt, device=dev))
    with torch.cuda.device(dev):
        rc = load_library().mamba_causal_conv1d_bwd(
            _ptr(x), _ptr(weight), _ptr(bias), _ptr(initial_state), _ptr(dout), _ptr(g["dx"]),
            _ptr(g["dweight"]), _ptr(g["dbias"]), _ptr(g["dinitial_state"]), b, d, L, K,
            int(bool(silu)), _DTYPES[dt], _stream_handle(dev))
    if rc != 0:
        raise MambaError(rc, "mamba_causal_conv1d_bwd")
    return g


def selective_scan_summary(u, delta, A, B, C, delta_bias=None, delta_softplus=True,
                           exact_zoh=False, workspace=None):
    """Summary of a sequence segment for the associative combine: (h_end (batch, dim, N),
    delta_sum (batch, dim)), the state after the segment from zero and its summed step."""
    if not isinstance(u, torch.Tensor) or u.dim() != 3:
        raise ValueError("u must be a (batch, dim, L) tensor")
    dev = u.device
    if dev.type != "cuda":
        raise ValueError("selective_scan_summary runs on CUDA tensors only")
    b, d, L = u.shape
    N = A.shape[1] if A.dim() == 2 else -1
    dt = u.dtype
    if dt not in _DTYPES:
        raise ValueError("unsupported input dtype %s" % dt)
    for t, name, shape, dts in ((u, "u", (b, d, L), (dt,)), (delta, "delta", (b, d, L), (dt,)),
                                (A, "A", (d, N), (torch.float32,)), (B, "B", (b, N, L), (dt,)),
                                (C, "C", (b, N, L), (dt,)),
                                (delta_bias, "delta_bias", (d,), (torch.float32,))):
        _check(t, name, dev, shape, dts)
    h_end = torch.empty((b, d, N), dtype=torch.float32, device=dev)
    dsum = torch.empty((b, d), dtype=torch.float32, device=dev)
    lib = load_library()
    dims = ScanDims(b, d, N, L)
    need = int(lib.mamba_selective_scan_workspace_size(dims))
    if need > 0 and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        rc = lib.mamba_selective_scan_summary(
            _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(delta_bias),
            int(bool(delta_softplus)), _ptr(h_end), _ptr(dsum), dims, _DTYPES[dt],
            _ptr(workspace), ws_bytes, MAMBA_FLAG_EXACT_ZOH if exact_zoh else 0,
            _stream_handle(dev))
    if rc != 0:
        raise MambaError(rc, "mamba_selective_scan_summary")
    return h_end, dsum


def selective_scan_fold(h_ends, delta_sums, A, h0=None, return_delta_sum=False):
    """Apply summaries h_ends (count, batch, dim, N), delta_sums (count, batch, dim) in order
    to h0 (batch, dim, N) or zero; returns the resulting state [and the total step]."""
    dev = A.device
    if dev.type != "cuda":
        raise ValueError("selective_scan_fold runs on CUDA tensors only")
    cnt, b, d, N = h_ends.shape
    _check(h_ends, "h_ends", dev, (cnt, b, d, N), (torch.float32,))
    _check(delta_sums, "delta_sums", dev, (cnt, b, d), (torch.float32,))
    _check(A, "A", dev, (d, N), (torch.float32,))
    _check(h0, "h0", dev, (b, d, N), (torch.float32,))
    h_out = torch.empty((b, d, N), dtype=torch.float32, device=dev)
    s_out = torch.empty((b, d), dtype=torch.float32, device=dev) if return_delta_sum else None
    with torch.cuda.device(dev):
        rc = load_library().mamba_selective_scan_fold(
            _ptr(h_ends) if cnt else None, _ptr(delta_sums) if cnt else None, _ptr(A), _ptr(h0),
            cnt, b, d, N, _ptr(h_out), _ptr(s_out), _stream_handle(dev))
    if rc != 0:
        raise MambaError(rc, "mamba_selective_scan_fold")
    return (h_out, s_out) if return_delta_sum else h_out
