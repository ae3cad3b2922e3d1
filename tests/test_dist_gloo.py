"""Data-parallel aux statistics on CPU ranks (gloo, world size 2).

Each rank takes half of the tokens, builds its additive statistics in the
library's float64 layout (from the oracle, on CPU), and all-reduces them with
the package's host logic. The reduced vector must equal the single-process
statistics (integers exactly, float64 sums to 1e-13), and L_bal / L_z formed
from it must equal the oracle's on all tokens.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def packed_sums(idx, p, lse, N, M, K):
    from token_choice_routing_b200.dist import aux_sums_slices
    sl = aux_sums_slices(N, K)
    v = np.zeros(sl["T"].stop)
    counts_ext, psum, lsq, T = O.aux_partial_sums(idx, p, lse, N, M)
    v[sl["counts_real"]] = counts_ext[:N]
    nulls = (np.asarray(idx) >= N).sum(axis=1)
    v[sl["null_hist"]] = np.bincount(nulls, minlength=K + 1)[:K + 1]
    v[sl["psum"]] = np.concatenate([psum[:N], [psum[N] if M else 0.0]])
    v[sl["lse2"]] = lsq
    v[sl["T"]] = T
    return v


def finalize(v, N, M, K):
    from token_choice_routing_b200.dist import aux_sums_slices
    sl = aux_sums_slices(N, K)
    hist = v[sl["null_hist"]]
    counts_ext = np.concatenate([v[sl["counts_real"]], [hist[j + 1:].sum() for j in range(M)]])
    psum = v[sl["psum"]]
    psum_ext = np.concatenate([psum[:N], np.full(M, psum[N])])
    T = v[sl["T"]][0]
    return O.aux_finalize(counts_ext, psum_ext, v[sl["lse2"]][0], T, N)


def _case():
    rng = np.random.default_rng(77)
    T, N, M, K = 400, 8, 24, 6
    s = rng.standard_normal((T, N + 1))
    s[:, N] += 0.8
    return s, N, M, K


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from token_choice_routing_b200.dist import allreduce_aux_sums
        s, N, M, K = _case()
        shard = np.array_split(np.arange(s.shape[0]), world)[rank]
        r = O.route(s[shard], M, K)
        v = torch.from_numpy(packed_sums(r["idx"], r["p"], r["lse"], N, M, K))
        allreduce_aux_sums(v)
        q.put((rank, v.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_rank_aux_allreduce_matches_single_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    s, N, M, K = _case()
    r = O.route(s, M, K)
    whole = packed_sums(r["idx"], r["p"], r["lse"], N, M, K)
    from token_choice_routing_b200.dist import aux_sums_slices
    sl = aux_sums_slices(N, K)
    for rank in (0, 1):
        v = res[rank]
        for key in ("counts_real", "null_hist", "T"):
            assert np.array_equal(v[sl[key]], whole[sl[key]]), key
        np.testing.assert_allclose(v, whole, rtol=1e-13, atol=1e-12)
        f, P, L_bal, L_z = finalize(v, N, M, K)
        _, f0, P0, L_bal0, L_z0 = O.aux_stats(r["idx"], r["p"], r["lse"], N, M)
        assert L_bal == pytest.approx(L_bal0, rel=1e-13)
        assert L_z == pytest.approx(L_z0, rel=1e-13)
        np.testing.assert_allclose(P, P0, rtol=1e-13)
    # both ranks agree bit for bit
    assert np.array_equal(res[0], res[1])


def test_sums_layout_matches_library_count():
    from token_choice_routing_b200.dist import aux_sums_slices
    from token_choice_routing_b200 import binding as B
    for N, M, K in ((8, 4, 4), (64, 8, 8), (5, 16, 16)):
        assert aux_sums_slices(N, K)["T"].stop == B.aux_sums_count(B.dims(10, 128, N, M, K, 64, 64))
    for N, M, K, Cc, V in ((8, 4, 4, 2, 3), (60, 0, 8, 10, 5)):
        assert aux_sums_slices(N, K, Cc + V)["T"].stop == B.aux_sums_count(B.dims(10, 128, N, M, K, 64, 64,
                                                                                C=Cc, V=V))


def _bwd_case():
    rng = np.random.default_rng(78)
    T, d, N, M, K, F, Fs = 40, 8, 4, 3, 2, 6, 5
    x = rng.standard_normal((T, d))
    w_r = rng.standard_normal((N + 1, d)) / np.sqrt(d)
    s = x @ w_r.T
    s[:, N] += rng.choice([-4.0, 0.0, 4.0], size=T)
    experts = (rng.standard_normal((N, F, d)), rng.standard_normal((N, F, d)), rng.standard_normal((N, d, F)))
    shared = (rng.standard_normal((Fs, d)), rng.standard_normal((Fs, d)), rng.standard_normal((d, Fs)))
    dy = rng.standard_normal((T, d))
    return x, w_r, s, experts, shared, dy, N, M, K


def _bwd_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from token_choice_routing_b200.dist import allreduce_grads, allreduce_token_total
        x, w_r, s, experts, shared, dy, N, M, K = _bwd_case()
        shard = np.array_split(np.arange(x.shape[0]), world)[rank]
        # whole-batch statistics from the ranks: slot counts (the forward's all-reduce) and T
        idx = O.route(s[shard], M, K)["idx"]
        counts = torch.from_numpy(np.bincount(idx.reshape(-1), minlength=N + M).astype(np.int64))
        dist.all_reduce(counts)
        t_total = allreduce_token_total(len(shard))
        g = O.layer_backward(x[shard], s[shard], w_r, N, M, K, experts, shared, dy[shard], 0.5, 0.25,
                             counts=counts.numpy(), t_total=t_total)
        grads = {"dw_router": torch.from_numpy(g["dW_r"]), "dbias": torch.from_numpy(g["dbias"]),
                 "dw_gate": torch.from_numpy(g["dW_gate"]), "dws_down": torch.from_numpy(g["dWs_down"]),
                 "dx": torch.from_numpy(g["dx"].copy())}
        dx_before = grads["dx"].clone()
        allreduce_grads(grads)
        q.put((rank, t_total, {k: v.numpy() for k, v in grads.items()}, torch.equal(dx_before, grads["dx"])))
    finally:
        dist.destroy_process_group()


def test_two_rank_backward_statistics_and_gradient_sum():
    """Data-parallel backward plumbing on two CPU ranks: the token total and slot counts are
    all-reduced, each rank differentiates its own tokens with them, and allreduce_grads sums the
    weight gradients (not dx) into the whole batch's gradient."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bwd_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, w_r, s, experts, shared, dy, N, M, K = _bwd_case()
    whole = O.layer_backward(x, s, w_r, N, M, K, experts, shared, dy, 0.5, 0.25)
    for rank, t_total, grads, dx_kept in res:
        assert t_total == x.shape[0] and dx_kept
        np.testing.assert_allclose(grads["dw_router"], whole["dW_r"], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(grads["dbias"], whole["dbias"], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(grads["dw_gate"], whole["dW_gate"], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(grads["dws_down"], whole["dWs_down"], rtol=1e-12, atol=1e-12)


def _bf16_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from token_choice_routing_b200.dist import allreduce_grads
        g = torch.from_numpy(_bf16_grads(rank)).to(torch.bfloat16)
        grads = {"dw_down": g, "dw_router": torch.from_numpy(_bf16_grads(rank).astype(np.float32))}
        allreduce_grads(grads)
        q.put((rank, grads["dw_down"].float().numpy(), grads["dw_router"].numpy()))
    finally:
        dist.destroy_process_group()


def _bf16_grads(rank):
    """A rank's bf16-valued gradient: values spread over several binades, so that rounding
    after each partial sum would differ from one rounding of the exact sum."""
    rng = np.random.default_rng(500 + rank)
    mant = rng.integers(128, 256, size=4096)          # 8 significant bits: exactly a bf16 value
    sign = rng.choice([-1.0, 1.0], size=4096)
    return (sign * mant * np.exp2(rng.integers(-3, 4, size=4096) - 7.0)).astype(np.float32)


def test_bf16_gradients_are_summed_in_fp32_and_rounded_once():
    """allreduce_grads over four ranks gives each bf16 weight gradient as bf16(the exact sum of
    the ranks' values): at most one rounding, whatever the number of ranks. (Four bf16 values
    within seven binades of each other add exactly in float32.)"""
    world = 4
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bf16_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    exact = sum(_bf16_grads(r).astype(np.float64) for r in range(world))
    once = torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(exact.astype(np.float32).astype(np.float64), exact)  # the fp32 sum is exact
    # a bf16 running sum (what an all-reduce in bf16 does) would not be: the case can tell them apart
    run = torch.from_numpy(_bf16_grads(0)).to(torch.bfloat16)
    for r in range(1, world):
        run = (run + torch.from_numpy(_bf16_grads(r)).to(torch.bfloat16))
    assert not np.array_equal(run.float().numpy(), once)
    for rank, g, gr in res:
        assert np.array_equal(g, once), rank
        np.testing.assert_allclose(gr, exact, rtol=1e-6, atol=1e-6)
