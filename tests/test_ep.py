"""Expert parallelism on CPU: the exchange plan (host logic) and the two row exchanges over
gloo ranks, with the oracle standing in for the kernels.

Each rank routes its own tokens, sends the rows of its real slots to the ranks that hold
their experts (null slots are never sent: MoE++ page, 局限性与开放问题 / 分布式部署复杂度),
computes its expert shard on the rows it received, and gets its rows' outputs back (MoE
tutorial page, 五、通信: a dispatch and a combine all-to-all). y must equal the
single-process layer output of the rank's tokens.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from token_choice_routing_b200 import ep


def test_plan_layout_by_hand():
    # 2 ranks, 4 experts (2 each). This rank (1) has rows per global expert [3, 0, 2, 5];
    # it receives, for its experts 2 and 3, [1, 4] rows from rank 0 and [2, 5] from itself.
    p = ep.make_plan(np.array([3, 0, 2, 5]), np.array([[1, 4], [2, 5]]), world=2, rank=1)
    assert p.n_local == 2
    assert p.send.tolist() == [[3, 0], [2, 5]]
    assert p.send_start.tolist() == [[0, 3], [3, 5]]
    # expert-major: expert 2 from rank 0 (1 row), then from rank 1 (2); expert 3 from rank 0 (4),
    # then from rank 1 (5)
    assert p.recv_start.tolist() == [[0, 3], [1, 7]]
    assert p.offsets_local.tolist() == [0, 3, 12]
    assert p.rows_recv == 12


def test_plan_rejects_uneven_split():
    with pytest.raises(ValueError):
        ep.make_plan(np.ones(6), np.ones((4, 1)), world=4, rank=0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _case():
    rng = np.random.default_rng(91)
    T, d, N, M, K, F, Fs = 96, 16, 8, 8, 4, 12, 10
    x = rng.standard_normal((T, d))
    w_r = rng.standard_normal((N + 1, d)) / np.sqrt(d)
    s = x @ w_r.T
    s[:, N] += rng.choice([-3.0, 0.0, 3.0], size=T)   # tokens with 0 .. K real experts
    experts = (rng.standard_normal((N, F, d)), rng.standard_normal((N, F, d)), rng.standard_normal((N, d, F)))
    shared = (rng.standard_normal((Fs, d)), rng.standard_normal((Fs, d)), rng.standard_normal((d, Fs)))
    return x, s, experts, shared, N, M, K


def _rank_step(rank, world, q):
    x, s, experts, shared, N, M, K = _case()
    tok = np.array_split(np.arange(x.shape[0]), world)[rank]
    xr, sr = x[tok], s[tok]
    r = O.route(sr, M, K)
    counts, offsets, perm, slot_row = O.dispatch(r["idx"], N)
    xs = torch.from_numpy(xr[perm].copy())
    tr = ep.DistTransport()
    recv = tr.exchange_counts(torch.from_numpy(counts.astype(np.int32)))
    plan = ep.make_plan(counts, recv, world, rank)
    xs_recv = torch.zeros((max(plan.rows_recv, 1), x.shape[1]), dtype=torch.float64)
    tr.exchange(*ep.dispatch_ops(plan, xs, xs_recv))
    # this rank's expert shard on the rows it received (oracle SwiGLU per expert segment)
    ys_recv = torch.zeros_like(xs_recv)
    for j in range(plan.n_local):
        e = rank * plan.n_local + j
        a, b = int(plan.offsets_local[j]), int(plan.offsets_local[j + 1])
        if b > a:
            ys_recv[a:b] = torch.from_numpy(O.swiglu(xs_recv[a:b].numpy(), experts[0][e], experts[1][e],
                                                     experts[2][e]))
    ys = torch.zeros_like(xs)
    tr.exchange(*ep.combine_ops(plan, ys_recv, ys))
    # combine in rank order
    y = O.swiglu(xr, *shared)
    for t in range(len(tok)):
        for k in range(K):
            if slot_row[t, k] >= 0:
                y[t] += r["gates"][t, k] * ys[slot_row[t, k]].numpy()
    q.put((rank, tok, y, int(plan.send.sum()), int(counts.sum()), int(plan.rows_recv), plan.recv.tolist()))


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        _rank_step(rank, world, q)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_exchanges_reproduce_the_layer_output(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, s, experts, shared, N, M, K = _case()
    r_all = O.route(s, M, K)
    real_per_rank = {}
    for rank, tok, y, sent, real, got, recv in res:
        y_ref = O.layer_output(x[tok], r_all["idx"][tok], r_all["gates"][tok], N, experts, shared)
        np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-12)
        assert sent == real            # exactly the real slots leave (null slots never do)
        real_per_rank[rank] = (got, recv)
    # every row sent is received once: the ranks' received totals add up to all real slots
    assert sum(g for g, _ in real_per_rank.values()) == int((r_all["idx"] < N).sum())
