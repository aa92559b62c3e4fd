"""The bench's multi-process host logic on CPU: two ranks over gloo.

bench.py runs one process per GPU; every rank scans its own batch (weak scaling, no
data-path collective) and the ranks only agree on timing through a max-reduction of
one scalar.  Here two CPU processes run that plumbing over gloo on 127.0.0.1.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    r, w, local = bench.dist_setup()
    assert (r, w, local) == (rank, world, rank)
    bench.barrier(w)
    timed = 10.0 + rank          # each rank "measured" a different time
    out[rank] = (bench.max_over_ranks(timed, w), bench.rank_seed(56003, r))
    bench.barrier(w)
    bench.dist_teardown(w)


def test_two_ranks_agree_on_max_time_and_use_distinct_seeds():
    world = 2
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
    assert [res[r][0] for r in range(world)] == [11.0, 11.0]
    assert len({res[r][1] for r in range(world)}) == world


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)
    bench.dist_teardown(1)


@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_weak_scaling_value_counts_every_rank(n):
    # value = units all ranks processed / max time over ranks
    elems = 4 * 5120 * 4096
    ms_total, steps = 637.0, 1000
    assert n * elems * steps / (ms_total * 1e-3) == pytest.approx(n * 1.3168e11, rel=1e-3)


def test_committed_profile_traffic_is_found_for_unchanged_kernels(tmp_path, monkeypatch):
    """bench.py reads a kernel's DRAM bytes from its committed ncu summary only while the
    kernel source still has the digest recorded there."""
    import bench
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    prof = tmp_path / "profiles"
    prof.mkdir()
    digest = bench.source_digest(str(src))
    (prof / "k.txt").write_text("source_sha256_16: %s   (k.cu)\ndram_bytes_per_launch: 1234\n" % digest)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profile_traffic("k.txt", "k.cu") == 1234.0
    src.write_text("kernel v1 // a comment\n/* another */")
    assert bench.profile_traffic("k.txt", "k.cu") == 1234.0
    src.write_text("kernel v2")
    assert bench.profile_traffic("k.txt", "k.cu") is None
    # a summary can depend on several sources ('+'-joined): a change in any of them counts
    hdr = tmp_path / "k.cuh"
    hdr.write_text("helper v1")
    both = bench.source_digest(str(src) + "+" + str(hdr))
    assert both != bench.source_digest(str(src))
    (prof / "kk.txt").write_text("source_sha256_16: %s   (k.cu+k.cuh)\ndram_bytes_per_launch: 99\n" % both)
    assert bench.profile_traffic("kk.txt", "k.cu+k.cuh") == 99.0
    hdr.write_text("helper v2")
    assert bench.profile_traffic("kk.txt", "k.cu+k.cuh") is None


def test_cpu_baseline_reports_all_cores_and_one_thread():
    import bench
    import oracle
    from selective_state_space_56_b200 import inputs
    before = oracle.num_threads()
    r = bench.cpu_baseline(inputs.SCAN_WORKLOADS["tiny_fp32"], budget_s=0.05)
    assert r["kind"] == "oracle" and r["value"] > 0 and r["single_thread_value"] > 0
    assert r["cores"] == before and oracle.num_threads() == before  # setting restored
    assert r["cpu_model"]
