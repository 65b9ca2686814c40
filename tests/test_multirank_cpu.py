"""The multi-rank path of bench.py on CPU: two gloo ranks (one process
each, as torchrun starts them) agree on the slowest rank's time, pass a
barrier, draw different replica inputs and aggregate the throughput of the
whole job."""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    from lightning_indexer_cross_b200 import workloads as W
    w, r, _ = bench.dist_setup(world, backend="gloo")
    ms = 10.0 + 5.0 * r  # this rank's device time
    m = bench.max_over_ranks(ms, w)
    bench.barrier(w)
    wl = W.stack("cpu", seed=bench.replica_seed(r), L=4, n_full=2, B=2, N=256, topk=16, H=8, schedule="FSFS")
    first = float(wl.layers[0].q[0, 0, 0])
    value = bench.replica_value(w, 32, 10, m)
    dist.destroy_process_group()
    q.put((r, m, first, value))


def test_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=180) for _ in ps)
    for p in ps:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in ps)
    assert [m for _, m, _, _ in res] == [15.0, 15.0]   # max over ranks
    assert res[0][2] != res[1][2]                        # independent replicas
    assert res[0][3] == pytest.approx(2 * 32 * 10 / 0.015)  # both ranks' queries over the slowest time


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.replica_value(1, 32, 10, 20.0) == pytest.approx(16000.0)
