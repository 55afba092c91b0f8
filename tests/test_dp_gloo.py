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


# ---------------------------------------------------------------------------
# The partitioning itself: two ranks each run the oracle's block on their half
# of the tokens, then exchange through the dp helpers.  Sharding by tokens
# must reproduce the whole-batch step: the MAX-reduced partial amax gives the
# whole batch's delayed scale bit for bit; under that scale every rank's
# forward and dX rows equal the whole batch's rows (the block is row-wise
# independent); the mean of the ranks' dW equals the whole-batch dW / N up to
# the fp32 roundings of the two partial sums and of their sum.
# ---------------------------------------------------------------------------

SHARD_PROBLEM = dict(M=256, d=64, h=256, seed=3)


def _whole_batch_reference():
    from fp8_relu_mlp_b200 import synth
    from oracle import ref
    p = SHARD_PROBLEM
    P = synth.make_problem(p["M"], p["d"], p["h"], seed=p["seed"])
    post = ref.relu2_post(ref.up_proj(P["x"], P["W1"]))
    st1 = ref.scale_update(ref.scale_state_init(2.0, 1.0), ref.amax(post))
    W2q, _, s_wi = ref.w2_cache(P["W2"])
    f = ref.forward(P["x"], P["W1"], W2q, s_wi, st1["scale"], st1["scale_inv"])
    b = ref.backward(P["x"], P["W1"], P["W2"], f["post"], P["dOut"])
    return P, st1, f, b


def _shard_worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from fp8_relu_mlp_b200 import dp, synth
        from oracle import ref
        p = SHARD_PROBLEM
        P = synth.make_problem(p["M"], p["d"], p["h"], seed=p["seed"])
        m = p["M"] // world
        rows = slice(rank * m, (rank + 1) * m)
        x, dOut = P["x"][rows], P["dOut"][rows]
        # step 0 on this rank's tokens: partial amax in the kernel's 32 x 64 blocks
        post0 = ref.relu2_post(ref.up_proj(x, P["W1"]))
        pa = torch.from_numpy(ref.partial_amax(post0, 32, 64))
        dp.allreduce_amax(pa)
        st1 = ref.scale_update(ref.scale_state_init(2.0, 1.0), ref.reduce_partials(pa.numpy()))
        # step 1 under the shared scale
        W2q, _, s_wi = ref.w2_cache(P["W2"])
        f = ref.forward(x, P["W1"], W2q, s_wi, st1["scale"], st1["scale_inv"])
        b = ref.backward(x, P["W1"], P["W2"], f["post"], dOut)
        local = (b["dW1"].copy(), b["dW2"].copy())
        dW1, dW2 = torch.from_numpy(b["dW1"].copy()), torch.from_numpy(b["dW2"].copy())
        dp.allreduce_grads(dW1, dW2, average=True)
        h = p["h"]
        s1 = torch.empty(h // world, p["d"])
        s2 = torch.empty(h // world, p["d"])
        dp.reduce_scatter_grads(torch.from_numpy(b["dW1"].copy()), torch.from_numpy(b["dW2"].copy()), s1, s2,
                                average=True)
        out_q.put((rank, float(st1["scale"]), float(st1["scale_inv"]), f["post"], f["q"], f["out"], b["dX"],
                   local, dW1.numpy().copy(), dW2.numpy().copy(), s1.numpy().copy(), s2.numpy().copy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_token_sharding_reproduces_the_whole_batch_step():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=150) for _ in range(world)], key=lambda r: r[0])
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    P, st1, f, b = _whole_batch_reference()
    m = SHARD_PROBLEM["M"] // world
    h = SHARD_PROBLEM["h"]
    for rank, scale, scale_inv, post, qc, out, dX, local, dW1, dW2, s1, s2 in res:
        rows = slice(rank * m, (rank + 1) * m)
        assert np.float32(scale) == st1["scale"] and np.float32(scale_inv) == st1["scale_inv"]
        assert np.array_equal(post, f["post"][rows])
        assert np.array_equal(qc, f["q"][rows])
        assert np.array_equal(out, f["out"][rows])
        assert np.array_equal(dX, b["dX"][rows])
    # mean over ranks vs the whole-batch gradient / N: each rank's dW is an
    # fp32 rounding of its exact partial sum, and the mean adds one rounding
    # of their sum and an exact halving
    a1, a2 = res[0][7], res[1][7]
    for k, full in ((0, b["dW1"]), (1, b["dW2"])):
        pa, pb = np.abs(a1[k].astype(np.float64)), np.abs(a2[k].astype(np.float64))
        bound = 2.0 ** -24 * (pa + pb) * 2 + 2.0 ** -24 * np.abs(full) + 1e-30
        want = full.astype(np.float64) / world
        for r in res:
            got = r[8 + k].astype(np.float64)
            assert np.all(np.abs(got - want) <= bound / world), k
            # both ranks hold the same reduced tensor
            assert np.array_equal(r[8 + k], res[0][8 + k])
        # reduce-scatter: rank r keeps rows [r h/N, (r+1) h/N) of the same mean
        for r in res:
            sl = slice(r[0] * (h // world), (r[0] + 1) * (h // world))
            assert np.array_equal(r[10 + k], res[0][8 + k][sl])
