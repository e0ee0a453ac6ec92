"""The bench's multi-process path on CPU: two gloo ranks (world size 2).

Each rank times its own replica; the reported time is the slowest rank's
and the rate counts every rank's units.  Ranks run independent replicas
(their own sequences), with no data-path collective.
"""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from cross_layer_top_full_b200 import synth
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        got = bench.max_over_ranks(ms, dist, "cpu")
        wl = bench.replica_workload(synth.WORKLOADS["prefill_512_fp32"], rank)
        inp = synth.layer_inputs(wl, 0, "cpu")
        q.put((rank, got, wl.seed, float(inp["q"].double().sum())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [r[1] for r in res] == [15.0, 15.0]          # both ranks report the slowest time
    assert res[0][2] != res[1][2]                        # distinct seeds ...
    assert res[0][3] != res[1][3]                        # ... hence distinct sequences


def test_whole_job_rate_counts_all_ranks():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.whole_job_rate(8192, 1, 1000.0) == pytest.approx(8192.0)
    assert bench.whole_job_rate(8192, 4, 500.0) == pytest.approx(4 * 8192 * 2.0)
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
