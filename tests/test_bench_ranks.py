"""The benchmark's multi-process plumbing on CPU: two gloo ranks take the barrier and the max over ranks of their
device-timed durations, and the whole-job value divides the work of both ranks by the slowest rank's time (weak
scaling: every rank runs its own independent layer). Runs without a GPU."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    g = bench.RankGroup("gloo", timeout_s=60)
    g.barrier()
    seconds = 1.5 * (rank + 1)  # rank r "took" 1.5 (r + 1) seconds
    t_max = g.max(seconds)
    out.put((rank, g.world, t_max, bench.whole_job_value(g.world, 3, 1e12, t_max)))
    g.close()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_max_and_value():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    for _, world, t_max, value in res:
        assert world == 2
        assert t_max == 3.0  # the slowest rank's time, on every rank
        assert value == pytest.approx(2 * 3 * 1e12 / 3.0 / 1e12)


def test_single_process_group_is_a_no_op():
    sys.path.insert(0, ROOT)
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    g = bench.RankGroup("gloo")
    assert g.world == 1 and g.dist is None
    g.barrier()
    assert g.max(2.5) == 2.5
    g.close()
    assert bench.whole_job_value(1, 4, 2e12, 2.0) == pytest.approx(4.0)
