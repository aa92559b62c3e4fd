"""Randomised parity sweep (needs a B200): seeded random shapes, dtypes and options for
every kernel family, each compared with the fp64 oracle under the tolerances of
s6_compare (and those of the backward and conv1d tests).  The hand-picked cases of the
other test files cover the known edges; this covers the combinations between them.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_56_b200 import inputs, ops
from tests.s6_compare import check_bf16_out, check_fp32, check_rms, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
F32, BF16 = torch.float32, torch.bfloat16


def _case(seed):
    r = np.random.default_rng(seed)
    return dict(b=int(r.integers(1, 4)), d=int(r.integers(1, 70)), N=int(r.integers(1, 17)),
                L=int(r.choice([0, 1, 2, 7, 31, 32, 33, 64, 100, 129, 257, 300])),
                in_dt=[F32, BF16][int(r.integers(0, 2))], out_dt=[F32, BF16][int(r.integers(0, 2))],
                z=bool(r.integers(0, 2)), D=bool(r.integers(0, 2)), bias=bool(r.integers(0, 2)),
                softplus=bool(r.integers(0, 4) > 0), zoh=bool(r.integers(0, 3) == 0),
                h0=bool(r.integers(0, 3) == 0))


def _check_y(y, y_ref, in_dt, out_dt, what):
    if in_dt == F32 and out_dt == F32:
        check_fp32(y, y_ref, what)
    elif out_dt == F32:
        check_rms(y, y_ref, what)
    else:
        check_bf16_out(y, y_ref, what)


@pytest.mark.parametrize("seed", range(40))
def test_random_forward(cuda_ok, seed):
    c = _case(1000 + seed)
    p = inputs.scan_inputs(c["b"], c["d"], c["N"], c["L"], c["in_dt"], seed=seed, with_z=c["z"],
                           with_d=c["D"], with_bias=c["bias"])
    if not c["softplus"]:
        p["delta"] = (0.001 + 0.2 * torch.rand(p["delta"].shape,
                                               generator=torch.Generator().manual_seed(seed))
                      ).to(c["in_dt"])
        if p["delta_bias"] is not None:
            p["delta_bias"] = torch.zeros_like(p["delta_bias"])
    h0 = (0.2 * torch.randn(c["b"], c["d"], c["N"], generator=torch.Generator().manual_seed(seed))
          if c["h0"] else None)
    g = {k: (None if v is None else v.to(DEV)) for k, v in p.items()}
    y, st = ops.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                                   delta_bias=g["delta_bias"], delta_softplus=c["softplus"],
                                   out_dtype=c["out_dt"], return_last_state=True,
                                   exact_zoh=c["zoh"],
                                   initial_state=None if h0 is None else h0.to(DEV))
    torch.cuda.synchronize()
    y_ref, st_ref = oracle.selective_scan(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"],
                                          z=p["z"], delta_bias=p["delta_bias"],
                                          softplus=c["softplus"], h0=h0, zoh=c["zoh"])
    _check_y(y, y_ref, c["in_dt"], c["out_dt"], "y %s" % c)
    if c["in_dt"] == F32:
        check_fp32(st, st_ref, "last_state %s" % c)
    else:
        check_rms(st, st_ref, "last_state %s" % c)


@pytest.mark.parametrize("seed", range(20))
def test_random_decode(cuda_ok, seed):
    c = _case(2000 + seed)
    b, d, N, dt = c["b"], c["d"], c["N"], c["in_dt"]
    gen = torch.Generator().manual_seed(seed)
    A = -torch.rand(d, N, generator=gen) * 4 - 0.05
    D = torch.randn(d, generator=gen) if c["D"] else None
    bias = torch.rand(d, generator=gen) * 2 - 4 if c["bias"] else None
    st0 = 0.1 * torch.randn(b, d, N, generator=gen)
    u, dr, z = (torch.randn(b, d, generator=gen).to(dt) for _ in range(3))
    Bm, Cm = (torch.randn(b, N, generator=gen).to(dt) for _ in range(2))
    z = z if c["z"] else None
    st = st0.to(DEV)
    y = ops.selective_state_update(st, u.to(DEV), dr.to(DEV), A.to(DEV), Bm.to(DEV), Cm.to(DEV),
                                   D=None if D is None else D.to(DEV),
                                   z=None if z is None else z.to(DEV),
                                   delta_bias=None if bias is None else bias.to(DEV),
                                   exact_zoh=c["zoh"])
    torch.cuda.synchronize()
    st_ref, y_ref = oracle.state_update(st0, u, dr, A, Bm, Cm, D=D, z=z, delta_bias=bias,
                                        zoh=c["zoh"])
    _check_y(y, y_ref, dt, dt, "decode y %s" % c)
    (check_fp32 if dt == F32 else check_rms)(st, st_ref, "decode state %s" % c)


@pytest.mark.parametrize("seed", range(12))
def test_random_backward(cuda_ok, seed):
    c = _case(3000 + seed)
    if c["L"] == 0:
        c["L"] = 17
    p = inputs.scan_inputs(c["b"], c["d"], c["N"], c["L"], F32, seed=seed, with_z=c["z"],
                           with_d=c["D"], with_bias=c["bias"])
    dy = torch.randn(c["b"], c["d"], c["L"], generator=torch.Generator().manual_seed(seed + 1))
    g = {k: (None if v is None else v.to(DEV)) for k, v in p.items()}
    grads = ops.selective_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], dy.to(DEV),
                                   D=g["D"], z=g["z"], delta_bias=g["delta_bias"])
    torch.cuda.synchronize()
    ref = oracle.selective_scan_backward(p["u"], p["delta"], p["A"], p["B"], p["C"], dy, D=p["D"],
                                         z=p["z"], delta_bias=p["delta_bias"])
    for gname, oname in (("du", "du"), ("ddelta", "ddelta"), ("dz", "dz"), ("dA", "dA"),
                         ("dB", "dB"), ("dC", "dC"), ("dD", "dD"), ("ddelta_bias", "dbias")):
        if grads[gname] is None:
            continue
        got, r = to64(grads[gname]), ref[oname]
        scale = 1e-4 * (np.abs(r) + np.sqrt(np.mean(r ** 2)))
        assert np.all(np.abs(got - r) <= scale), "%s %s" % (gname, c)


@pytest.mark.parametrize("seed", range(12))
def test_random_conv1d(cuda_ok, seed):
    r = np.random.default_rng(4000 + seed)
    b, d, L, K = int(r.integers(1, 4)), int(r.integers(1, 50)), int(r.integers(0, 90)), \
        int(r.integers(1, 5))
    p = inputs.conv_inputs(b, d, L, K, F32, seed=seed, with_bias=bool(r.integers(0, 2)),
                           with_initial_state=bool(r.integers(0, 2)) and K > 1)
    silu = bool(r.integers(0, 2))
    g = {k: (None if v is None else v.to(DEV)) for k, v in p.items()}
    out, fin = ops.causal_conv1d_fwd(g["x"], g["weight"], g["bias"], g["initial_state"], silu=silu,
                                     return_final_state=True)
    torch.cuda.synchronize()
    ref, fref = oracle.causal_conv1d(p["x"], p["weight"], p["bias"], p["initial_state"], silu=silu)
    check_fp32(out, ref, "conv out b=%d d=%d L=%d K=%d" % (b, d, L, K))
    if K > 1:
        np.testing.assert_array_equal(to64(fin), fref)
