"""CUDA-graph capture of the library's calls (needs a B200): a server replays the decode
step as a graph, copying each token's inputs into static buffers first.  The captured
calls allocate nothing and synchronise nothing (the scan needs no workspace at these
sizes), so capture works; replays must equal eager calls bit for bit."""
import pytest
import torch

from selective_state_space_56_b200 import inputs, ops

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_decode_step_graph_replay_equals_eager(cuda_ok):
    b, d, N = 8, 256, 16
    w = inputs.DECODE_WORKLOAD
    prm = {k: v.to(DEV) for k, v in inputs.decode_params(w).items()}
    A, D, bias = (prm[k][:d].contiguous() for k in ("A", "D", "delta_bias"))
    state0 = prm["state0"][:b, :d].contiguous()
    toks = [inputs.decode_step_inputs(k, w, device=DEV, batch=b, dim=d) for k in range(6)]
    # eager reference
    st_e = state0.clone()
    y_eager = []
    for x in toks:
        y_eager.append(ops.selective_state_update(st_e, x["u"], x["delta"], A, x["B"], x["C"], D=D,
                                                  z=x["z"], delta_bias=bias).clone())
    # graph: static input buffers, one captured step
    static = {k: v.clone() for k, v in toks[0].items()}
    st_g = state0.clone()
    y_g = torch.empty((b, d), dtype=w.io_dtype, device=DEV)
    ops.load_library()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up on the capture stream
        tmp = state0.clone()
        ops.selective_state_update(tmp, static["u"], static["delta"], A, static["B"], static["C"],
                                   D=D, z=static["z"], delta_bias=bias, y=y_g)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        ops.selective_state_update(st_g, static["u"], static["delta"], A, static["B"], static["C"],
                                   D=D, z=static["z"], delta_bias=bias, y=y_g)
    for k, x in enumerate(toks):
        for name, v in x.items():
            static[name].copy_(v)
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(y_g, y_eager[k]), "token %d" % k
    assert torch.equal(st_g, st_e)
    del graph
    ops.check_device_error()


def test_scan_graph_replay_equals_eager(cuda_ok):
    p = inputs.scan_inputs(2, 64, 16, 512, torch.bfloat16, seed=12, device=DEV)
    assert ops.selective_scan_workspace_size(2, 64, 16, 512) == 0
    y_e, st_e = ops.selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"],
                                       z=p["z"], delta_bias=p["delta_bias"], return_last_state=True)
    y = torch.empty_like(y_e)
    st = torch.empty_like(st_e)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        ops.selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                               delta_bias=p["delta_bias"], y=y, last_state=st)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        ops.selective_scan_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                               delta_bias=p["delta_bias"], y=y, last_state=st)
    y.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, y_e) and torch.equal(st, st_e)
    del graph
    ops.check_device_error()
