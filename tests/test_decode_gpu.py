"""Parity of the CUDA selective_state_update (decode) with the fp64 oracle (needs a B200).

The decode workload (batch 256, dim 5120, N 16, bf16 I/O, fp32 state) runs 1000
steps with fresh seeded inputs each step, as the bench does.  The oracle carries
every (batch, channel) lane in fp64 through all 1000 steps, and y and the state
are compared on the full tensors after steps 1, 10 and 1000.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_56_b200 import inputs, ops
from tests.s6_compare import check_bf16_out, check_fp32, check_rms, rms, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_decode_workload_1000_steps(cuda_ok):
    w = inputs.DECODE_WORKLOAD
    prm = inputs.decode_params(w)
    A, D, bias = prm["A"], prm["D"], prm["delta_bias"]
    state = prm["state0"].to(DEV)
    Ag, Dg, bg = A.to(DEV), D.to(DEV), bias.to(DEV)
    nl = w.batch * w.dim
    lb = np.repeat(np.arange(w.batch, dtype=np.int64), w.dim)   # lane i = (i // dim, i % dim)
    A64 = np.ascontiguousarray(np.tile(to64(A), (w.batch, 1)))
    D64 = np.ascontiguousarray(np.tile(to64(D), w.batch))
    b64 = np.ascontiguousarray(np.tile(to64(bias), w.batch))
    ref_state = np.ascontiguousarray(to64(prm["state0"]).reshape(nl, w.dstate))  # fp64, all lanes
    checked = []
    for step in range(w.steps):
        x = inputs.decode_step_inputs(step, w)
        g = {k: v.to(DEV) for k, v in x.items()}
        y = ops.selective_state_update(state, g["u"], g["delta"], Ag, g["B"], g["C"], D=Dg,
                                       z=g["z"], delta_bias=bg)
        _, y_ref = oracle.state_update_lanes(
            ref_state, to64(x["u"]).reshape(nl), to64(x["delta"]).reshape(nl), A64, x["B"],
            x["C"], lb, D=D64, z=to64(x["z"]).reshape(nl), delta_bias=b64, inplace=True)
        if step + 1 in (1, 10, w.steps):
            torch.cuda.synchronize()
            shp = (w.batch, w.dim)
            stats = check_bf16_out(y.cpu(), y_ref.reshape(shp), "y step %d (full)" % (step + 1))
            assert stats["n"] == nl
            check_rms(state.cpu(), ref_state.reshape(shp + (w.dstate,)),
                      "state step %d (full)" % (step + 1))
            checked.append(step + 1)
    assert checked == [1, 10, w.steps]
    assert rms(ref_state) > 0


@pytest.mark.parametrize("N", [1, 4, 6, 8, 12, 16])
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_decode_shapes(cuda_ok, N, io):
    _decode_case(3, 37, N, io)


# N = 16 shapes for the two-lanes-per-thread path: one tile, many tiles, several batch
# rows, lane counts whose last warp is only partly used; each with and without z / D /
# bias.
@pytest.mark.parametrize("bd", [(1, 128), (2, 256), (3, 1024), (5, 640), (1, 136), (3, 40),
                                (4, 1000), (7, 584)])
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_decode_n16_shapes(cuda_ok, bd, io):
    _decode_case(bd[0], bd[1], 16, io)
    _decode_case(bd[0], bd[1], 16, io, with_optional=False)


def _decode_case(b, d, N, io, with_optional=True):
    g = torch.Generator().manual_seed(100 + N)
    st0 = 0.1 * torch.randn(b, d, N, generator=g)
    x = {k: torch.randn(*s, generator=g).to(io) for k, s in
         dict(u=(b, d), delta=(b, d), z=(b, d), B=(b, N), C=(b, N)).items()}
    A = -torch.arange(1, N + 1, dtype=torch.float32).expand(d, N).contiguous()
    D = torch.randn(d, generator=g)
    bias = torch.log(torch.expm1(0.001 + 0.099 * torch.rand(d, generator=g, dtype=torch.float64))).float()
    if not with_optional:
        D = bias = None
        x["z"] = None
    dev = lambda t: None if t is None else t.to(DEV)  # noqa: E731
    state = st0.to(DEV)
    y = ops.selective_state_update(state, *(x[k].to(DEV) for k in ("u", "delta")), A.to(DEV),
                                   x["B"].to(DEV), x["C"].to(DEV), D=dev(D), z=dev(x["z"]),
                                   delta_bias=dev(bias))
    s_ref, y_ref = oracle.state_update(st0, x["u"], x["delta"], A, x["B"], x["C"], D=D, z=x["z"],
                                       delta_bias=bias)
    torch.cuda.synchronize()
    if io == torch.float32:
        check_fp32(y.cpu(), y_ref, "y")
        check_fp32(state.cpu(), s_ref, "state")
    else:
        check_bf16_out(y.cpu(), y_ref, "y")
        check_rms(state.cpu(), s_ref, "state")


def test_decode_without_optional_inputs(cuda_ok):
    b, d, N = 2, 50, 16
    g = torch.Generator().manual_seed(5)
    st0 = torch.randn(b, d, N, generator=g)
    u, dl = torch.randn(b, d, generator=g), torch.rand(b, d, generator=g) * 0.5
    B, C = torch.randn(b, N, generator=g), torch.randn(b, N, generator=g)
    A = -torch.rand(d, N, generator=g) - 0.1
    state = st0.to(DEV)
    y = ops.selective_state_update(state, u.to(DEV), dl.to(DEV), A.to(DEV), B.to(DEV), C.to(DEV),
                                   delta_softplus=False)
    s_ref, y_ref = oracle.state_update(st0, u, dl, A, B, C, softplus=False)
    torch.cuda.synchronize()
    check_fp32(y.cpu(), y_ref, "y")
    check_fp32(state.cpu(), s_ref, "state")


def test_decode_steps_reproduce_the_scan(cuda_ok):
    """L decode steps from a zero state give the scan's y_t and last_state (GPU vs GPU)."""
    b, d, N, L = 2, 40, 16, 48
    p = inputs.scan_inputs(b, d, N, L, in_dtype=torch.float32, seed=77)
    g = {k: (None if v is None else v.to(DEV)) for k, v in p.items()}
    y_scan, st_scan = ops.selective_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"],
                                             z=g["z"], delta_bias=g["delta_bias"],
                                             return_last_state=True)
    state = torch.zeros(b, d, N, device=DEV)
    ys = []
    for t in range(L):
        ys.append(ops.selective_state_update(
            state, g["u"][..., t].contiguous(), g["delta"][..., t].contiguous(), g["A"],
            g["B"][..., t].contiguous(), g["C"][..., t].contiguous(), D=g["D"],
            z=g["z"][..., t].contiguous(), delta_bias=g["delta_bias"]))
    torch.cuda.synchronize()
    check_fp32(torch.stack(ys, -1).cpu(), y_scan.cpu(), "decode y vs scan y")
    check_fp32(state.cpu(), st_scan.cpu(), "decode state vs scan last_state")
