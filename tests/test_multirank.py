"""The replica timing of bench.py across ranks, on CPU with gloo (world size 2).

The DiT step does not shard: N GPUs run N independent replicas, and the only
collectives are a barrier and the max over ranks of the timed region.  This
runs those exact helpers in two processes and checks the whole-job value."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import bench
    r = bench.Ranks(world, backend="gloo")
    ms = [120.0, 150.0][rank]          # rank 1 is the slower replica
    r.barrier()
    mx = r.max(ms)
    value = bench.aggregate_throughput(world, 10, mx)
    r.barrier()
    r.close()
    q.put((rank, mx, value))


def test_replica_timing_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, value in out:
        assert mx == 150.0                     # the slowest replica sets the time
        assert value == pytest.approx(2 * 10 / 0.150)   # both replicas' steps count


def test_single_rank_needs_no_process_group():
    import bench
    r = bench.Ranks(1)
    assert r.dist is None and r.max(3.0) == 3.0
    assert bench.aggregate_throughput(1, 5, 500.0) == pytest.approx(10.0)
