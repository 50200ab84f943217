"""Multi-process plumbing on CPU: two gloo ranks, no GPU.

Each rank runs an independent problem (weak scaling): seeds differ per rank,
(batch, head) slices partition exactly, and the reported time is the max
over ranks."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from efficient_transformer_lsh_b200 import dist


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    r, local, w = dist.init("gloo", timeout_s=60)
    t = dist.max_over_ranks(1.5 + rank)          # rank 1 is the slower one
    lo, hi = dist.shard(13, r, w)
    import numpy as np
    from efficient_transformer_lsh_b200.workloads import WORKLOADS, generate
    wl = WORKLOADS["toy-f32-L1024"].with_sizes(L=128)
    x = generate(wl, seed=dist.rank_seed(100, r))["qk"]
    gathered = [None] * w
    torch.distributed.all_gather_object(gathered, (lo, hi, float(np.asarray(x).sum())))
    dist.barrier()
    dist.finish()
    q.put((r, t, gathered))


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, t, gathered in res:
        assert t == 2.5                      # max over ranks
        (lo0, hi0, s0), (lo1, hi1, s1) = gathered
        assert (lo0, hi0, lo1, hi1) == (0, 7, 7, 13)
        assert s0 != s1                      # independent problems per rank


def test_shard_covers_everything():
    for n in (1, 7, 8, 64, 65):
        for world in (1, 2, 3, 8):
            parts = [dist.shard(n, r, world) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            for a, b in zip(parts, parts[1:]):
                assert a[1] == b[0]
            sizes = [h - l for l, h in parts]
            assert max(sizes) - min(sizes) <= 1
