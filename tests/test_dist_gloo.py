"""Host logic of the multi-GPU bench path with two gloo ranks on the CPU.

With N GPUs every rank runs independent canvases (no data-path collective); the
only cross-rank steps are the barriers around the timed region and the
max-over-ranks of the elapsed time.  Both are exercised here without a GPU.
"""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, n_canvas, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    r, w, lr = bench.dist_env()
    dist.init_process_group("gloo", rank=r, world_size=w)
    try:
        lo, hi = bench.shard_canvases(n_canvas, r, w)
        elapsed = 10.0 + 3.0 * r                 # a rank-dependent "timed region"
        dist.barrier()
        mx = bench.max_over_ranks(elapsed)
        q.put((r, w, lr, lo, hi, mx))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,n_canvas", [(2, 2), (2, 16), (2, 5)])
def test_replica_sharding_and_max_over_ranks(world, n_canvas):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n_canvas, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    covered = []
    for r, w, lr, lo, hi, mx in res:
        assert w == world and lr == r
        assert mx == 10.0 + 3.0 * (world - 1)     # every rank sees the slowest rank's time
        covered.extend(range(lo, hi))
    assert covered == list(range(n_canvas))       # disjoint shards covering every canvas


def test_single_process_defaults(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import bench
    assert bench.dist_env() == (0, 1, 0)
    assert bench.shard_canvases(7, 0, 1) == (0, 7)
    assert bench.max_over_ranks(3.5) == 3.5
