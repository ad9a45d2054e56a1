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


# ------------------------------------------------------------------ vocabulary-parallel exchange
def _split_worker(rank, world, port, q):
    """Each rank packs the oracle's statistics of its vocabulary shard into the partial layout,
    the ranks exchange partials with the package's all-gather, and rank 0 merges what it received."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import math

    import numpy as np
    import torch
    from discrete_diffusion_decoding_b200 import vocab_parallel as vp
    from oracle import stage
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        V, d, N, T = 1280, 16, 256, 0.8
        rng = np.random.default_rng(0)                 # the same problem on every rank
        h = rng.standard_normal((N, d))
        W = rng.standard_normal((V, d)) * 0.5
        E = rng.standard_normal((V, d))
        v0, v1 = vp.shard_bounds(V, world, rank)
        z = stage.logits(h, W[v0:v1], T)
        st = stage.partial_stats(z)
        L = vp.partial_layout(N, d)
        buf = np.zeros(L["total"], np.uint8)
        log2e = 1.0 / math.log(2.0)
        stats = np.stack([st["m"] * log2e, st["l"], st["u"] * log2e, st["m"] * T], axis=1).astype(np.float32)
        buf[L["stats"]:L["stats"] + stats.nbytes] = stats.reshape(-1).view(np.uint8)
        idx = (st["a"] + v0).astype(np.int32)
        buf[L["idx"]:L["idx"] + idx.nbytes] = idx.view(np.uint8)
        o = (np.exp(z - st["m"][:, None]) @ E[v0:v1]).astype(np.float32)
        buf[L["o"]:L["o"] + o.nbytes] = o.reshape(-1).view(np.uint8)
        gathered = torch.empty(world * L["total"], dtype=torch.uint8)
        vp.exchange_partials(torch.from_numpy(buf), gathered)
        if rank == 0:
            g = gathered.numpy()
            merged, num, shards = None, None, []
            for r in range(world):
                base = r * L["total"]
                s4 = g[base + L["stats"]:base + L["stats"] + 16 * N].view(np.float32).reshape(N, 4).astype(np.float64)
                ix = g[base + L["idx"]:base + L["idx"] + 4 * N].view(np.int32).astype(np.int64)
                orr = g[base + L["o"]:base + L["o"] + 4 * N * d].view(np.float32).reshape(N, d).astype(np.float64)
                part = {"m": s4[:, 0] / log2e, "l": s4[:, 1], "u": s4[:, 2] / log2e, "a": ix}
                shards.append(vp.shard_bounds(V, world, r))
                if merged is None:
                    merged, num = part, orr
                else:
                    M = np.maximum(merged["m"], part["m"])
                    num = num * np.exp(merged["m"] - M)[:, None] + orr * np.exp(part["m"] - M)[:, None]
                    merged = stage.merge_stats(merged, part, 0)
            fin = stage.finish_stats(merged)
            full = stage.distribution_stats(stage.logits(h, W, T))
            sc = stage.self_conditioning(full["p"], E)
            q.put({"shards": shards,
                   "dH": float(np.abs(fin["H"] - full["H"]).max()),
                   "dlse": float(np.abs(fin["lse"] - full["lse"]).max()),
                   "argmax_eq": bool(np.array_equal(fin["argmax"], full["argmax"])),
                   "dsc": float(np.abs(num / merged["l"][:, None] - sc).max())})
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_vocab_split_exchange_and_merge(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    lo = [a for a, _ in res["shards"]]
    hi = [b for _, b in res["shards"]]
    assert lo[0] == 0 and hi[-1] == 1280 and lo[1:] == hi[:-1]          # contiguous, in rank order
    assert all(b % 256 == 0 for b in lo + hi)
    assert res["argmax_eq"]
    assert res["dH"] < 1e-5 and res["dlse"] < 1e-5 and res["dsc"] < 1e-4     # float32 transport of the partials


def test_partial_layout_matches_the_library():
    """The Python view of a partial and the library's dg_partial_bytes agree (host-only call)."""
    import ctypes
    from discrete_diffusion_decoding_b200 import _abi, build
    from discrete_diffusion_decoding_b200 import vocab_parallel as vp
    L = ctypes.CDLL(build.build())
    L.dg_params_default.argtypes = [ctypes.POINTER(_abi.DgParams), ctypes.c_int, ctypes.c_int, ctypes.c_int]
    L.dg_partial_bytes.argtypes = [ctypes.POINTER(_abi.DgParams)]
    L.dg_partial_bytes.restype = ctypes.c_size_t
    for C, V, d in [(1, 262144, 2816), (3, 4096, 128), (16, 8960, 512)]:
        p = _abi.DgParams()
        L.dg_params_default(ctypes.byref(p), C, V, d)
        assert L.dg_partial_bytes(ctypes.byref(p)) == vp.partial_layout(C * 256, d)["total"]
    with pytest.raises(ValueError):
        vp.shard_bounds(1000, 2, 0)
    assert vp.shard_bounds(262144, 8, 7) == (229376, 262144)
