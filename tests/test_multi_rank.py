"""Multi-process plumbing on CPU: two gloo ranks, no GPU.

A problem is split across ranks by contiguous ranges of its (batch, head)
slices; each rank draws and runs only its shard, and the reported time is
the max over ranks. Running the oracle shard by shard on the ranks gives
exactly the whole problem's result (the slices are independent)."""
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
    from efficient_transformer_lsh_b200.workloads import WORKLOADS, generate_slices
    from oracle import lsh_oracle as orc
    # one global problem of 2 x 3 slices; this rank's shard through the oracle
    gw = WORKLOADS["batch-bf16-8x8x4096"].with_sizes(B=2, H=3, L=256, n_rounds=2)
    s0, s1 = dist.shard(gw.B * gw.H, r, w)
    inp = generate_slices(gw, s0, s1)
    qk = inp["qk"].astype(np.float64)[None]
    v = inp["v"].astype(np.float64)[None]
    res = orc.lsh_attention(qk, v, inp["R"].astype(np.float64), gw.chunk, gw.causal, gw.scale)
    gathered = [None] * w
    torch.distributed.all_gather_object(gathered, (lo, hi, s0, s1, res["O"][0], res["LSE"][0]))
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
    import numpy as np
    from efficient_transformer_lsh_b200.workloads import WORKLOADS, generate
    from oracle import lsh_oracle as orc
    gw = WORKLOADS["batch-bf16-8x8x4096"].with_sizes(B=2, H=3, L=256, n_rounds=2)
    whole = generate(gw)
    full = orc.lsh_attention(whole["qk"].astype(np.float64), whole["v"].astype(np.float64),
                             whole["R"].astype(np.float64), gw.chunk, gw.causal, gw.scale)
    for r, t, gathered in res:
        assert t == 2.5                      # max over ranks
        (lo0, hi0, a0, b0, O0, L0), (lo1, hi1, a1, b1, O1, L1) = gathered
        assert (lo0, hi0, lo1, hi1) == (0, 7, 7, 13)
        assert (a0, b0, a1, b1) == (0, 3, 3, 6)
        # the shards' results, put together, are the whole problem's
        O = np.concatenate([O0, O1]).reshape(full["O"].shape)
        LSE = np.concatenate([L0, L1]).reshape(full["LSE"].shape)
        np.testing.assert_array_equal(O, full["O"])
        np.testing.assert_array_equal(LSE, full["LSE"])


def test_shard_covers_everything():
    for n in (1, 7, 8, 64, 65):
        for world in (1, 2, 3, 8):
            parts = [dist.shard(n, r, world) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            for a, b in zip(parts, parts[1:]):
                assert a[1] == b[0]
            sizes = [h - l for l, h in parts]
            assert max(sizes) - min(sizes) <= 1
