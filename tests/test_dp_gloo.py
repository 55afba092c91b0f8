"""Multi-rank host logic on the CPU: two gloo ranks on 127.0.0.1.

The data-parallel exchange of the block (partial-amax MAX, dW sum/mean) and
the max-over-ranks timing that bench.py uses are exercised with CPU tensors;
the oracle's scale update run on the reduced amax must give every rank the
same scale.  No GPU is touched.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from fp8_relu_mlp_b200 import dp
        from oracle import ref
        g = np.random.default_rng(rank)
        # each rank's partial amax over its own tokens
        pa = torch.from_numpy((np.abs(g.standard_normal((16, 6))) * (rank + 1)).astype(np.float32))
        local_max = float(pa.max())
        dp.allreduce_amax(pa)
        st = ref.scale_update(ref.scale_state_init(2.0, 1.0), ref.reduce_partials(pa.numpy()))
        dW1 = torch.full((4, 3), float(rank + 1))
        dW2 = torch.full((4, 3), float(10 * (rank + 1)))
        dp.allreduce_grads(dW1, dW2, average=True)
        t = dp.max_over_ranks(0.25 * (rank + 1))
        # reduce-scatter: rank r keeps rows [2r, 2r+2) of the mean over ranks
        G1 = torch.arange(12, dtype=torch.float32).reshape(4, 3) * (rank + 1)
        G2 = -G1
        s1, s2 = torch.empty(2, 3), torch.empty(2, 3)
        dp.reduce_scatter_grads(G1, G2, s1, s2, average=True)
        out_q.put((rank, local_max, float(pa.max()), float(st["scale"]), dW1.numpy().copy(), dW2.numpy().copy(), t,
                   s1.numpy().copy(), s2.numpy().copy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_exchange():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=100) for _ in range(world)]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    res.sort()
    global_max = max(r[1] for r in res)
    full = np.arange(12, dtype=np.float32).reshape(4, 3) * 1.5   # mean of x1 and x2
    for rank, local_max, reduced_max, scale, dW1, dW2, t, s1, s2 in res:
        assert reduced_max == global_max           # every rank sees the global amax
        assert np.all(dW1 == 1.5) and np.all(dW2 == 15.0)   # mean over ranks
        assert t == 0.5                             # max over ranks
        assert np.array_equal(s1, full[2 * rank:2 * rank + 2]) and np.array_equal(s2, -full[2 * rank:2 * rank + 2])
    assert res[0][3] == res[1][3]                   # identical delayed scale on both ranks
