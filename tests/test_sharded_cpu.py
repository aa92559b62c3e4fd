"""The L-sharded scan's exchange step on CPU: two gloo ranks all-gather their segment
summaries (selective_state_space_56_b200.sharded.gather_summaries) and must receive every
rank's (h_end, delta_sum) in rank order -- the order the fold depends on.  The kernels
themselves are covered on one GPU by tests/test_sharded_gpu.py, which emulates the ranks."""
import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    from selective_state_space_56_b200 import sharded
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    b, d, N = 2, 3, 4
    h = torch.arange(b * d * N, dtype=torch.float32).reshape(b, d, N) + 1000 * rank
    s = torch.arange(b * d, dtype=torch.float32).reshape(b, d) - 100 * rank
    H, S = sharded.gather_summaries(h, s)
    out[rank] = (H.tolist(), S.tolist())
    dist.barrier()
    dist.destroy_process_group()


def test_gather_summaries_in_rank_order():
    world = 3
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    b, d, N = 2, 3, 4
    for r in range(world):
        H, S = (torch.tensor(x) for x in res[r])
        assert H.shape == (world, b, d, N) and S.shape == (world, b, d)
        for q in range(world):
            assert torch.equal(H[q], torch.arange(b * d * N, dtype=torch.float32).reshape(b, d, N)
                               + 1000 * q)
            assert torch.equal(S[q], torch.arange(b * d, dtype=torch.float32).reshape(b, d)
                               - 100 * q)
