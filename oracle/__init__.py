"""Sequential fp64 CPU oracle for the selective scan (S6) and its decode step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library and never imports it; the CUDA path never imports this.

The arithmetic lives in ``s6_oracle.c`` (plain C, IEEE double, libm exp/log1p,
no fast-math), compiled on first use into ``libs6_oracle.so`` beside it.  This
module only marshals numpy arrays.  The definitions it follows:

* Mamba: Linear-Time Sequence Modeling with Selective State Spaces (page
  "xyznot.com/ar/paper/2312.00752"), section "Method": ZOH discretisation
  Abar = exp(Delta A); recurrence h_t = Abar h_{t-1} + Bbar x_t; readout
  y_t = C h_t.  Section "Selection mechanism (S6)": B_t, C_t per token, shared
  over channels; Delta = softplus(Parameter + s_Delta(x)).
* Page "yongjin360.com/news/29389": the serial "MambaMini" scan, initial state
  h_{-1} = 0, Bbar formed as the element-wise product of Delta and B, the
  state shape (batch, d_inner, d_state) and the SiLU gate.
* With ``zoh=True``: the exact zero-order-hold Bbar = (Delta A)^-1 (exp(Delta A) - I)
  Delta B of the "Method" section, per state expm1(Delta A_n) / A_n * B_n.

Pins (tests/test_oracle_pins.py): hand-worked examples in tests/golden/, the
associative-combine prefix of ``oracle.pscan``, the LTI convolution form,
Abar in (0,1), small/large-Delta limits, the gated-RNN special case.  The ZOH
variant (tests/test_oracle_zoh.py): the gated-RNN identity, the continuous-time
steady state -B u / A, numerical integration of the continuous ODE, the
small-Delta limit and A = 0; its backward (tests/test_oracle_backward.py): central
differences of the ZOH forward, A = 0 and |A| = 1e-5 included.  The causal conv1d
(tests/test_oracle_conv.py): numpy's
convolution, the impulse response, causality, chunked prefill and decode steps; its
backward: central finite differences of the forward, the linear case in closed form.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "s6_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libs6_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_lp = ctypes.POINTER(ctypes.c_long)


def build(force: bool = False) -> str:
    """Compile s6_oracle.c into libs6_oracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-fPIC", "-shared", "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.s6o_softplus.restype = ctypes.c_double
            lib.s6o_softplus.argtypes = [ctypes.c_double]
            lib.s6o_discretize.restype = ctypes.c_int
            lib.s6o_discretize.argtypes = [ctypes.c_long] * 3 + [_dp, _dp, _dp, ctypes.c_int,
                                                                 _dp, _dp]
            lib.s6o_scan.restype = ctypes.c_int
            lib.s6o_scan.argtypes = ([ctypes.c_long] * 4 + [_dp] * 8 + [_lp, ctypes.c_int,
                                                                     ctypes.c_int, _dp]
                                     + [_dp] * 3)
            lib.s6o_state_update.restype = ctypes.c_int
            lib.s6o_state_update.argtypes = ([ctypes.c_long] * 3 + [_dp] * 9 + [_lp, ctypes.c_int,
                                                                             ctypes.c_int, _dp])
            lib.s6o_scan_backward.restype = ctypes.c_int
            lib.s6o_scan_backward.argtypes = ([ctypes.c_long] * 4 + [_dp] * 8 + [_lp, ctypes.c_int,
                                               ctypes.c_int] + [_dp] * 9)
            lib.s6o_causal_conv1d.restype = ctypes.c_int
            lib.s6o_causal_conv1d.argtypes = [ctypes.c_long] * 3 + [_dp] * 4 + [ctypes.c_int,
                                                                               _dp, _dp]
            lib.s6o_causal_conv1d_update.restype = ctypes.c_int
            lib.s6o_causal_conv1d_update.argtypes = [ctypes.c_long] * 2 + [_dp] * 4 + [
                ctypes.c_int, _dp]
            lib.s6o_causal_conv1d_backward.restype = ctypes.c_int
            lib.s6o_causal_conv1d_backward.argtypes = [ctypes.c_long] * 3 + [_dp] * 4 + [
                ctypes.c_int] + [_dp] * 5
            lib.s6o_num_threads.restype = ctypes.c_int
            lib.s6o_num_threads.argtypes = []
            lib.s6o_set_num_threads.restype = ctypes.c_int
            lib.s6o_set_num_threads.argtypes = [ctypes.c_int]
            _lib = lib
    return _lib


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # a torch tensor (CPU); widen exactly through fp32
        a = a.detach().float().cpu().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(_dp)


def num_threads() -> int:
    """OpenMP threads the oracle's lane loops use."""
    return int(_load().s6o_num_threads())


def set_num_threads(n: int) -> int:
    """Use n OpenMP threads from now on; returns the previous count."""
    return int(_load().s6o_set_num_threads(int(n)))


def softplus(x: float) -> float:
    """log(1 + e^x) in double precision (the selection mechanism's tau_Delta)."""
    return float(_load().s6o_softplus(float(x)))


def discretize(delta_raw, A, delta_bias=None, softplus=True):
    """Delta (nlanes, L) and Abar = exp(Delta A) (nlanes, L, N) for lanes.

    delta_raw: (nlanes, L); A: (nlanes, N); delta_bias: (nlanes) or None.
    """
    dr, Aa, bb = _f64(delta_raw), _f64(A), _f64(delta_bias)
    nl, L = dr.shape
    N = Aa.shape[1]
    assert Aa.shape == (nl, N)
    delta = np.empty((nl, L))
    abar = np.empty((nl, L, N))
    rc = _load().s6o_discretize(nl, N, L, _ptr(dr), _ptr(Aa), _ptr(bb), int(bool(softplus)),
                                _ptr(delta), _ptr(abar))
    if rc != 0:
        raise ValueError("s6o_discretize rejected its arguments")
    return delta, abar


def scan_lanes(u, delta_raw, A, B, C, lane_batch, D=None, z=None, delta_bias=None,
               softplus=True, h0=None, return_states=False, zoh=False):
    """Sequential scan over independent lanes.

    u, delta_raw, z: (nlanes, L); A: (nlanes, N); D, delta_bias: (nlanes);
    B, C: (nbatch, N, L); lane_batch: (nlanes) int; h0: (nlanes, N) or None.
    zoh: Bbar = expm1(Delta A) / A * B (the exact zero-order hold) instead of Delta B.
    Returns y (nlanes, L), h_last (nlanes, N)[, h_all (nlanes, L, N)].
    """
    u, dr, z = _f64(u), _f64(delta_raw), _f64(z)
    Aa, Dd, bb = _f64(A), _f64(D), _f64(delta_bias)
    Bm, Cm, h0 = _f64(B), _f64(C), _f64(h0)
    nl, L = u.shape
    N = Aa.shape[1]
    nb = Bm.shape[0]
    assert dr.shape == (nl, L) and Aa.shape == (nl, N)
    assert Bm.shape == (nb, N, L) and Cm.shape == (nb, N, L)
    if z is not None:
        assert z.shape == (nl, L)
    lb = np.ascontiguousarray(np.asarray(lane_batch, dtype=np.int64).reshape(nl))
    y = np.empty((nl, L))
    h_last = np.empty((nl, N))
    h_all = np.empty((nl, L, N)) if return_states else None
    rc = _load().s6o_scan(nl, N, L, nb, _ptr(u), _ptr(dr), _ptr(z), _ptr(Aa), _ptr(Dd),
                          _ptr(bb), _ptr(Bm), _ptr(Cm), lb.ctypes.data_as(_lp),
                          int(bool(softplus)), int(bool(zoh)), _ptr(h0), _ptr(y), _ptr(h_last),
                          _ptr(h_all))
    if rc != 0:
        raise ValueError("s6o_scan rejected its arguments")
    if return_states:
        return y, h_last, h_all
    return y, h_last


def selective_scan(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                   h0=None, return_states=False, zoh=False):
    """The selective scan in the library's layouts.

    u, delta, z: (batch, dim, L); A: (dim, N); B, C: (batch, N, L);
    D, delta_bias: (dim); h0: (batch, dim, N) or None.
    Returns y (batch, dim, L) and last_state (batch, dim, N) as float64
    [and all states (batch, dim, L, N) when return_states].
    """
    u = _f64(u)
    b, d, L = u.shape
    Aa = _f64(A)
    N = Aa.shape[1]
    rep = lambda v: None if v is None else np.tile(_f64(v), b)  # noqa: E731  (per-lane copy)
    out = scan_lanes(u.reshape(b * d, L), _f64(delta).reshape(b * d, L),
                     np.tile(Aa, (b, 1)), B, C, np.repeat(np.arange(b), d),
                     D=rep(D), z=None if z is None else _f64(z).reshape(b * d, L),
                     delta_bias=rep(delta_bias), softplus=softplus,
                     h0=None if h0 is None else _f64(h0).reshape(b * d, N),
                     return_states=return_states, zoh=zoh)
    y = out[0].reshape(b, d, L)
    hl = out[1].reshape(b, d, N)
    if return_states:
        return y, hl, out[2].reshape(b, d, L, N)
    return y, hl


def state_update(state, u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                 zoh=False):
    """One decode token: returns (new_state (batch, dim, N), y (batch, dim)).

    state: (batch, dim, N); u, delta, z: (batch, dim); A: (dim, N);
    B, C: (batch, N); D, delta_bias: (dim).  The input state is not modified.
    """
    st = _f64(state).copy()
    b, d, N = st.shape
    rep = lambda v: None if v is None else np.tile(_f64(v), b)  # noqa: E731
    uu = _f64(u).reshape(b * d)
    dd = _f64(delta).reshape(b * d)
    zz = None if z is None else _f64(z).reshape(b * d)
    Aa = np.tile(_f64(A), (b, 1))
    Dd, bb = rep(D), rep(delta_bias)
    Bv, Cv = _f64(B), _f64(C)
    assert Bv.shape == (b, N) and Cv.shape == (b, N)
    lb = np.repeat(np.arange(b, dtype=np.int64), d)
    y = np.empty(b * d)
    rc = _load().s6o_state_update(
        b * d, N, b, _ptr(st), _ptr(uu), _ptr(dd), _ptr(zz), _ptr(Aa), _ptr(Dd), _ptr(bb),
        _ptr(Bv), _ptr(Cv), lb.ctypes.data_as(_lp), int(bool(softplus)), int(bool(zoh)), _ptr(y))
    if rc != 0:
        raise ValueError("s6o_state_update rejected its arguments")
    return st, y.reshape(b, d)


def state_update_lanes(state, u, delta_raw, A, B, C, lane_batch, D=None, z=None, delta_bias=None,
                       softplus=True, zoh=False, inplace=False):
    """One decode token on independent lanes: returns (new_state (nlanes, N), y (nlanes)).

    state, A: (nlanes, N); u, delta_raw, z, D, delta_bias: (nlanes);
    B, C: (nbatch, N); lane i reads row lane_batch[i].  ``state`` is not modified, unless
    ``inplace``: then it must be a C-contiguous float64 numpy array, which is updated and
    returned (long decode runs carry millions of lanes without a copy per token).
    """
    if inplace:
        if not (isinstance(state, np.ndarray) and state.dtype == np.float64
                and state.flags["C_CONTIGUOUS"]):
            raise TypeError("inplace needs a C-contiguous float64 numpy state")
        st = state
    else:
        st = _f64(state).copy()
    nl, N = st.shape
    uu, dd, zz = _f64(u).reshape(nl), _f64(delta_raw).reshape(nl), _f64(z)
    Aa, Dd, bb = _f64(A), _f64(D), _f64(delta_bias)
    Bv, Cv = _f64(B), _f64(C)
    assert Aa.shape == (nl, N) and Bv.shape[1] == N and Cv.shape == Bv.shape
    lb = np.ascontiguousarray(np.asarray(lane_batch, dtype=np.int64).reshape(nl))
    y = np.empty(nl)
    rc = _load().s6o_state_update(
        nl, N, Bv.shape[0], _ptr(st), _ptr(uu), _ptr(dd), _ptr(zz), _ptr(Aa), _ptr(Dd), _ptr(bb),
        _ptr(Bv), _ptr(Cv), lb.ctypes.data_as(_lp), int(bool(softplus)), int(bool(zoh)), _ptr(y))
    if rc != 0:
        raise ValueError("s6o_state_update rejected its arguments")
    return st, y


def scan_backward_lanes(u, delta_raw, A, B, C, lane_batch, dy, D=None, z=None, delta_bias=None,
                        softplus=True, zoh=False):
    """Gradients of sum(y * dy) for lanes: returns dict du, ddelta, dz (nlanes, L),
    dA (nlanes, N), dD, dbias (nlanes), dB, dC (nbatch, N, L)."""
    u, dr, z, dy = _f64(u), _f64(delta_raw), _f64(z), _f64(dy)
    Aa, Dd, bb = _f64(A), _f64(D), _f64(delta_bias)
    Bm, Cm = _f64(B), _f64(C)
    nl, L = u.shape
    N = Aa.shape[1]
    nb = Bm.shape[0]
    lb = np.ascontiguousarray(np.asarray(lane_batch, dtype=np.int64).reshape(nl))
    out = dict(du=np.empty((nl, L)), ddelta=np.empty((nl, L)), dz=np.empty((nl, L)),
               dA=np.empty((nl, N)), dD=np.empty(nl), dbias=np.empty(nl),
               dB=np.empty((nb, N, L)), dC=np.empty((nb, N, L)))
    rc = _load().s6o_scan_backward(
        nl, N, L, nb, _ptr(u), _ptr(dr), _ptr(z), _ptr(Aa), _ptr(Dd), _ptr(bb), _ptr(Bm),
        _ptr(Cm), lb.ctypes.data_as(_lp), int(bool(softplus)), int(bool(zoh)), _ptr(dy),
        _ptr(out["du"]),
        _ptr(out["ddelta"]), _ptr(out["dz"]), _ptr(out["dA"]), _ptr(out["dD"]),
        _ptr(out["dbias"]), _ptr(out["dB"]), _ptr(out["dC"]))
    if rc != 0:
        raise ValueError("s6o_scan_backward rejected its arguments")
    return out


def selective_scan_backward(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None,
                            softplus=True, zoh=False):
    """Backward in the library's layouts: u, delta, z, dy (b, d, L); A (d, N); B, C
    (b, N, L); D, delta_bias (d).  Returns du, ddelta, dz (b, d, L), dA (d, N), dD, dbias (d),
    dB, dC (b, N, L): the gradients of sum(y * dy)."""
    u = _f64(u)
    b, d, L = u.shape
    Aa = _f64(A)
    N = Aa.shape[1]
    rep = lambda v: None if v is None else np.tile(_f64(v), b)  # noqa: E731
    r = scan_backward_lanes(u.reshape(b * d, L), _f64(delta).reshape(b * d, L),
                            np.tile(Aa, (b, 1)), B, C, np.repeat(np.arange(b), d),
                            _f64(dy).reshape(b * d, L), D=rep(D),
                            z=None if z is None else _f64(z).reshape(b * d, L),
                            delta_bias=rep(delta_bias), softplus=softplus, zoh=zoh)
    return dict(du=r["du"].reshape(b, d, L), ddelta=r["ddelta"].reshape(b, d, L),
                dz=r["dz"].reshape(b, d, L), dA=r["dA"].reshape(b, d, N).sum(0),
                dD=r["dD"].reshape(b, d).sum(0), dbias=r["dbias"].reshape(b, d).sum(0),
                dB=r["dB"], dC=r["dC"])


def causal_conv1d(x, weight, bias=None, initial_state=None, silu=True):
    """Causal depthwise conv1d (+ SiLU) in the library's layouts.

    x: (batch, dim, L); weight: (dim, K); bias: (dim) or None; initial_state:
    (batch, dim, K-1) or None.  Returns out (batch, dim, L) and the final state
    (batch, dim, K-1): the last K-1 inputs, oldest first."""
    xx = _f64(x)
    b, d, L = xx.shape
    w = _f64(weight)
    K = w.shape[1]
    rows = b * d
    wr = np.ascontiguousarray(np.tile(w, (b, 1)))
    br = None if bias is None else np.ascontiguousarray(np.tile(_f64(bias), b))
    init = None if initial_state is None else _f64(initial_state).reshape(rows, K - 1)
    out = np.empty((rows, L))
    fin = np.empty((rows, max(K - 1, 0)))
    rc = _load().s6o_causal_conv1d(rows, L, K, _ptr(np.ascontiguousarray(xx.reshape(rows, L))),
                                   _ptr(wr), _ptr(br), _ptr(init), int(bool(silu)), _ptr(out),
                                   _ptr(fin) if K > 1 else None)
    if rc != 0:
        raise ValueError("s6o_causal_conv1d rejected its arguments")
    return out.reshape(b, d, L), fin.reshape(b, d, K - 1)


def causal_conv1d_update(state, x, weight, bias=None, silu=True):
    """One decode token: returns (new_state (batch, dim, K-1), out (batch, dim)).
    ``state`` is not modified."""
    w = _f64(weight)
    d, K = w.shape
    xx = _f64(x)
    b = xx.shape[0]
    st = _f64(state).reshape(b * d, K - 1).copy() if K > 1 else np.empty((b * d, 0))
    out = np.empty(b * d)
    rc = _load().s6o_causal_conv1d_update(
        b * d, K, _ptr(st) if K > 1 else None, _ptr(np.ascontiguousarray(xx.reshape(b * d))),
        _ptr(np.ascontiguousarray(np.tile(w, (b, 1)))),
        None if bias is None else _ptr(np.ascontiguousarray(np.tile(_f64(bias), b))),
        int(bool(silu)), _ptr(out))
    if rc != 0:
        raise ValueError("s6o_causal_conv1d_update rejected its arguments")
    return st.reshape(b, d, K - 1), out.reshape(b, d)


def causal_conv1d_backward(x, weight, dout, bias=None, initial_state=None, silu=True):
    """Gradients of sum(out * dout) for ``causal_conv1d`` (same layouts).  Returns a dict:
    dx (batch, dim, L), dweight (dim, K), dbias (dim), dinitial_state (batch, dim, K-1) or
    None when no initial state was given."""
    xx = _f64(x)
    b, d, L = xx.shape
    w = _f64(weight)
    K = w.shape[1]
    rows = b * d
    wr = np.ascontiguousarray(np.tile(w, (b, 1)))
    br = None if bias is None else np.ascontiguousarray(np.tile(_f64(bias), b))
    init = None if initial_state is None else _f64(initial_state).reshape(rows, K - 1)
    dx = np.empty((rows, L))
    dw = np.empty((rows, K))
    db = np.empty(rows)
    dinit = None if init is None else np.zeros((rows, max(K - 1, 0)))
    rc = _load().s6o_causal_conv1d_backward(
        rows, L, K, _ptr(np.ascontiguousarray(xx.reshape(rows, L))), _ptr(wr), _ptr(br),
        _ptr(init), int(bool(silu)), _ptr(np.ascontiguousarray(_f64(dout).reshape(rows, L))),
        _ptr(dx), _ptr(dw), _ptr(db), _ptr(dinit) if (dinit is not None and K > 1) else None)
    if rc != 0:
        raise ValueError("s6o_causal_conv1d_backward rejected its arguments")
    return dict(dx=dx.reshape(b, d, L), dweight=dw.reshape(b, d, K).sum(0),
                dbias=db.reshape(b, d).sum(0),
                dinitial_state=None if dinit is None else dinit.reshape(b, d, K - 1))
