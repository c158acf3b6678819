"""bench.py's replica mode on CPU: with more than one rank every replica runs its own bank
and query stream, the ranks agree on the slowest rank's device times (max over ranks)
and the reported value is all ranks' units over that time.  Two gloo ranks, no GPU."""
import os
import socket

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    import sys

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench
    try:
        w, r, _ = bench.init_ranks("gloo", timeout_s=60)
        # rank r took (10 + r) ms for its steps and (5 - 5 r) ms end to end
        times = bench.max_over_ranks([10.0 + r, 5.0 * (1 - r)], "cpu")
        value = bench.replica_throughput(1000.0, w, times[0])
        dist.barrier()
        out.put((r, w, times, value))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_rank():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, w, times, value in results:
        assert w == 2
        assert times == [11.0, 5.0]                          # the max of each entry over the ranks
        assert value == pytest.approx(2 * 1000.0 / 11e-3)    # both ranks' units over the slowest time


def test_single_process_keeps_its_own_times():
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        assert k not in os.environ or os.environ[k] in ("1", "0")
    assert bench.max_over_ranks([3.0, 4.0], "cpu") == [3.0, 4.0]
    assert bench.replica_throughput(1e8, 1, 10.0) == pytest.approx(1e10)
