"""The N > 1 path of the benchmark on CPU: world-size-2 gloo process groups.

Each rank runs its own batch (no data-path collective); only the timing is combined:
the slowest rank's time is every rank's time, the whole-job throughput counts the units
of all ranks, and only rank 0 reports.  The reference arm under torchrun runs on rank 0
alone and the other ranks leave without work.
"""

import datetime
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from gated_delta_rule_70_b200 import dist as kdist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r "took" 10 + r ms for its steps and 5 - r ms for its end-to-end step
        got = kdist.max_over_ranks([10.0 + rank, 5.0 - rank])
        rate = kdist.whole_job_rate(32768, world, got[0] / 4)
        import bench
        ns = type("A", (), {"ref_tokens": 64, "warmup": 3, "steps": 1, "gpus": world})()
        ref = bench.run_reference(ns, rank) if rank != 0 else "skipped"
        q.put((rank, got, rate, kdist.report_rank(rank), ref))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_gloo():
    import multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        results = sorted(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    for rank, got, rate, reports, ref in results:
        assert got == [11.0, 5.0]                      # the slowest rank's times, on every rank
        assert rate == pytest.approx(32768 * 2 / (11.0 / 4 * 1e-3))   # all ranks' units
        assert reports == (rank == 0)
        if rank != 0:
            assert ref is None                         # the reference arm: rank 0 only


def test_single_process_defaults():
    from gated_delta_rule_70_b200 import dist as kdist

    assert kdist.world_info({}) == (0, 1, 0)
    assert kdist.world_info({"RANK": "3", "WORLD_SIZE": "8", "LOCAL_RANK": "3"}) == (3, 8, 3)
    assert kdist.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]   # no process group: unchanged
    assert kdist.whole_job_rate(100, 1, 10.0) == pytest.approx(1e4)
