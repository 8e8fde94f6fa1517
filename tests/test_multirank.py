"""The multi-rank path of bench.py (one process per GPU, token-parallel, no
collective on the data path) on two CPU processes with the gloo backend:
rank seeds, the slowest-rank timing and the whole-job aggregate."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import synth
    try:
        w, r, local = bench.dist_setup(None, backend="gloo")
        assert (w, r, local) == (world, rank, rank)
        # every rank draws its own tokens; the weights are the same everywhere
        x = synth.make_x(4, 256, seed=bench.x_seed(r, 0))
        wt = synth.make_w(8, 256, seed=7)
        xs = [torch.zeros_like(x) for _ in range(world)]
        torch.distributed.all_gather(xs, x)
        ws = [torch.zeros_like(wt) for _ in range(world)]
        torch.distributed.all_gather(ws, wt)
        distinct_x = all(not torch.equal(xs[0], xs[i]) for i in range(1, world))
        same_w = all(torch.equal(ws[0], ws[i]) for i in range(1, world))
        # rank r did (r + 1) * 10 units in (r + 1) seconds
        units, secs = bench.aggregate(10.0 * (r + 1), float(r + 1), w)
        bench.barrier(w)
        q.put((r, distinct_x, same_w, units, secs))
    finally:
        if torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_token_parallel_aggregation_on_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    for r, distinct_x, same_w, units, secs in res:
        assert distinct_x and same_w
        assert units == pytest.approx(10.0 * sum(range(1, world + 1)))
        assert secs == pytest.approx(float(world))     # the slowest rank's time


def test_single_rank_aggregate_is_identity():
    import bench
    assert bench.aggregate(5.0, 2.0, 1) == (5.0, 2.0)
    assert bench.x_seed(0, 3) == 3 and bench.x_seed(1, 3) != bench.x_seed(0, 3)
