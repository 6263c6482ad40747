"""World-size-2 checks of the multi-rank benchmark plumbing on CPU (gloo).

The path shards without any exchange (independent projections / heads), so the
multi-GPU benchmark runs one replica per rank; the only collectives are the
barrier around the timed region and the max over ranks of the times.  These
tests run that plumbing as two gloo processes on the host.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out_q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import bench
    ranks = bench.Ranks(world, rank, device=None, backend="gloo")
    ranks.barrier()
    m = ranks.max(times[rank])
    v = bench.weak_scaled_value(world, 1e12, m)
    ranks.close()
    out_q.put((rank, m, v))


@pytest.mark.parametrize("times", [(1.5, 2.5), (3.0, 0.5)])
def test_two_ranks_take_the_max_time_and_scale_the_work(times):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, v in res:
        assert m == max(times)
        assert v == pytest.approx(world * 1e12 / (max(times) * 1e-3) / 1e12)


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    r = bench.Ranks(1, 0, device=None)
    r.barrier()
    assert r.max(4.25) == 4.25
    assert bench.weak_scaled_value(1, 2e12, 2.0) == pytest.approx(1000.0)
    r.close()
