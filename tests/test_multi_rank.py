"""The N > 1 bench plumbing on the CPU: two gloo ranks on 127.0.0.1.

The path shards by sequence (batch rows), so ranks exchange nothing on the
data path; only the barrier and the job-level timing reduce across ranks:
the step time is the slowest rank's, the throughput sums every rank's rows."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import bench
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    # rank r "took" (r + 1) * 100 ms for 10 steps of 64 rows
    value, ms_step = bench.weak_scaling(d, 64, (rank + 1) * 100.0, 10)
    d.barrier()
    d.close()
    q.put((rank, value, ms_step))


@pytest.mark.timeout(120)
def test_weak_scaling_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=90) for _ in procs]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, value, ms_step in res:
        assert ms_step == pytest.approx(20.0)  # slowest rank: 200 ms / 10 steps
        assert value == pytest.approx(2 * 64 / 0.020)  # both ranks' rows per step / step time


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    assert d.world == 1 or os.environ.get("WORLD_SIZE") not in (None, "1")
    value, ms_step = bench.weak_scaling(d, 32, 50.0, 5)
    assert ms_step == pytest.approx(10.0) and value == pytest.approx(32 / 0.010)
