"""Host logic of the multi-rank benchmark on CPU with two gloo ranks:
per-rank workloads differ (weak scaling, no data exchange) and the timing is
the max over ranks."""

import datetime
import multiprocessing as mp
import os
import socket


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        m = bench.max_over_ranks(10.0 * (rank + 1))
        w = bench.rank_workload(rank)
        dist.barrier()
        out.put((rank, m, w.seed, w.batch, w.context))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_batches():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    os.environ["PYTHONPATH"] = root + os.pathsep + os.environ.get("PYTHONPATH", "")
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = sorted(out.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [20.0, 20.0]               # max over ranks
    assert res[0][2] != res[1][2]                             # each rank its own seeded batch
    assert res[0][3:] == res[1][3:]                           # same shape per rank (weak scaling)


def test_query_ring_walks_back_and_forth():
    import bench
    seq = [bench.ring_index(t, 4) for t in range(10)]
    assert seq == [0, 1, 2, 3, 2, 1, 0, 1, 2, 3]
    assert all(abs(a - b) == 1 for a, b in zip(seq, seq[1:]))
