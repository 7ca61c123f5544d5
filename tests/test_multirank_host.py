"""The N > 1 host path of bench.py on CPU: world-size-2 gloo process groups.

bench.py runs one replica per GPU under torchrun; the ranks meet only at barriers and
in the max-over-ranks reduction of the timed region (the path has no data exchange).
These tests run that logic as two host processes on a gloo group.
"""
import datetime
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


def _rank_main(rank, world, port, values, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench._barrier(world)
        out.put((rank, bench._max_over_ranks(world, values[rank])))
        bench._barrier(world)
    finally:
        dist.destroy_process_group()


def _run(world, values):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, values, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    codes = [p.exitcode for p in procs]
    results = sorted(out.get(timeout=10) for _ in range(world))
    return codes, results


def test_max_over_ranks_two_gloo_ranks():
    # each rank's timed region (ms); the job's time is the slowest rank's
    codes, results = _run(2, [3.25, 7.5])
    assert codes == [0, 0]
    assert results == [(0, 7.5), (1, 7.5)]


def test_max_over_ranks_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench._max_over_ranks(1, 4.0) == 4.0
