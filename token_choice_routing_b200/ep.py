"""Expert-parallel execution of the null-expert MoE layer.

The routed experts are split over the ranks: rank r holds experts
[r N/W, (r+1) N/W). Every rank keeps the router and the shared expert and routes
its own tokens. Two exchanges move the routed rows (MoE tutorial page, 五、通信：
All-to-All 为什么是成本中心: a dispatch all-to-all sends each token's rows to the
ranks that hold its experts, a combine all-to-all brings the expert outputs
back). Null slots never leave the rank: zero-computation experts live on every
GPU (MoE++ page, 局限性与开放问题 / 分布式部署复杂度), and dispatch has already cut
them from the expert-contiguous row list, so only real slots are sent.

One step on rank r:
 1. route, and the aux statistics all-reduced over the ranks as in data
    parallelism (f_i and P_i are means over the whole batch);
 2. dispatch: this rank's real slots, expert-contiguous (moe_dispatch). The rows
    for rank p's experts are then one contiguous range of xs;
 3. counts exchange (an all-to-all of N int32 per rank): how many rows each rank
    sends to each other rank for each of its experts. The sizes of the row
    exchange are host-side arguments of NCCL's point-to-point calls, so the
    received counts come back to the host here (one small synchronisation);
 4. row exchange: for every (rank, expert) pair with rows, one send of that
    range of xs, received straight into its place in an expert-major buffer
    (experts in order, source ranks in order inside an expert). No permutation
    pass is needed before the grouped GEMMs;
 5. the shard's grouped gate/up and down GEMMs over the received rows
    (moe_expert_gate_up_rows / moe_expert_down_rows), the shared expert over this
    rank's own tokens;
 6. the reverse exchange returns each output row into this rank's ys, at the
    row dispatch gave its slot;
 7. combine (moe_combine), exactly as on one GPU.

A row's expert output does not depend on which rank or tile computes it, so y is
bit-identical to the single-GPU forward of the same tokens.

Transports: DistTransport (torch.distributed: all_to_all_single for the counts,
batch_isend_irecv for the rows; NCCL between GPUs, gloo between CPU processes)
and LocalFabric (W ranks as threads of one process sharing one device, rows
copied in stream order; for tests on one GPU).
"""
from __future__ import annotations

import dataclasses
import threading
from typing import Callable, Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch
import torch.distributed as dist


@dataclasses.dataclass
class EpPlan:
    """Host-side sizes of one step's row exchanges on one rank."""
    world: int
    rank: int
    n_local: int               # experts per rank
    send: np.ndarray           # [world, n_local] rows for rank p's j-th expert
    send_start: np.ndarray     # [world, n_local] first such row in this rank's xs / ys
    recv: np.ndarray           # [world, n_local] rows from rank s for this rank's j-th expert
    recv_start: np.ndarray     # [world, n_local] first such row in the received buffers
    offsets_local: np.ndarray  # [n_local + 1] expert segments of the received buffers
    rows_recv: int


def make_plan(counts: np.ndarray, recv: np.ndarray, world: int, rank: int) -> EpPlan:
    """Exchange plan from this rank's rows per global expert (``counts`` [N], the dispatch
    counts) and the rows every rank sends it for its own experts (``recv`` [world, n_local],
    from the counts exchange). Sends follow this rank's expert-contiguous layout; the
    received rows are laid out expert-major, source ranks in order inside an expert."""
    counts = np.asarray(counts, dtype=np.int64).reshape(-1)
    N = counts.size
    if N % world != 0:
        raise ValueError(f"{N} experts do not split evenly over {world} ranks")
    n_local = N // world
    recv = np.asarray(recv, dtype=np.int64).reshape(world, n_local)
    send = counts.reshape(world, n_local)
    off = np.concatenate([[0], np.cumsum(counts)])
    send_start = off[:-1].reshape(world, n_local)
    order = recv.T.reshape(-1)                              # (expert j, source s), j major
    starts = np.concatenate([[0], np.cumsum(order)])[:-1]
    recv_start = starts.reshape(n_local, world).T.copy()    # back to [s, j]
    per_expert = recv.sum(axis=0)
    offsets_local = np.concatenate([[0], np.cumsum(per_expert)])
    return EpPlan(world, rank, n_local, send, send_start, recv, recv_start, offsets_local,
                  int(offsets_local[-1]))


def dispatch_ops(plan: EpPlan, xs: torch.Tensor, xs_recv: torch.Tensor):
    """(sends, recvs) of the dispatch exchange: (peer, row block) lists, in (peer, expert)
    order on both sides, so the k-th send from a to b meets b's k-th receive from a."""
    sends, recvs = [], []
    for p in range(plan.world):
        for j in range(plan.n_local):
            n = int(plan.send[p, j])
            if n:
                a = int(plan.send_start[p, j])
                sends.append((p, xs[a:a + n]))
    for s in range(plan.world):
        for j in range(plan.n_local):
            n = int(plan.recv[s, j])
            if n:
                a = int(plan.recv_start[s, j])
                recvs.append((s, xs_recv[a:a + n]))
    return sends, recvs


def combine_ops(plan: EpPlan, ys_recv: torch.Tensor, ys: torch.Tensor):
    """(sends, recvs) of the combine exchange: the dispatch exchange reversed."""
    sends, recvs = dispatch_ops(plan, ys, ys_recv)
    return ([(p, t) for p, t in recvs], [(p, t) for p, t in sends])


class DistTransport:
    """Exchanges over torch.distributed (NCCL for CUDA tensors, gloo for CPU ones)."""

    def __init__(self, group=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def exchange_counts(self, send: torch.Tensor) -> np.ndarray:
        """All-to-all of the per-expert row counts: send [N] (N/world per destination)."""
        send = send.contiguous()
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send, group=self.group)
        return recv.cpu().numpy().reshape(self.world, -1)

    def exchange(self, sends, recvs):
        """Row blocks: self-addressed pairs are copied locally, the rest go out as one batch
        of point-to-point operations."""
        own_s = [t for p, t in sends if p == self.rank]
        own_r = [t for p, t in recvs if p == self.rank]
        for dst, src in zip(own_r, own_s):
            dst.copy_(src)
        ops = []
        for p, t in sends:
            if p != self.rank:
                ops.append(dist.P2POp(dist.isend, t.contiguous(), p, self.group))
        for p, t in recvs:
            if p != self.rank:
                ops.append(dist.P2POp(dist.irecv, t, p, self.group))
        if ops:
            for req in dist.batch_isend_irecv(ops):
                req.wait()

    def all_reduce_sum(self, t: torch.Tensor):
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)


class LocalFabric:
    """W ranks in one process, each a thread with its own endpoint (``endpoint(rank)``).
    Exchanges meet at a barrier; row blocks are copied on the device in stream order (the
    sender's buffers were written by work enqueued before the barrier)."""

    def __init__(self, world: int):
        self.world = world
        self.barrier = threading.Barrier(world)
        self.box: Dict[Tuple[str, int], object] = {}

    def endpoint(self, rank: int) -> "_LocalTransport":
        return _LocalTransport(self, rank)

    def run(self, fn: Callable[[int, "_LocalTransport"], object]) -> List[object]:
        """Runs fn(rank, transport) for every rank on its own thread; returns the results."""
        res: List[object] = [None] * self.world
        err: List[BaseException] = []

        def body(r):
            try:
                res[r] = fn(r, self.endpoint(r))
            except BaseException as e:  # noqa: BLE001  (re-raised below)
                err.append(e)
                self.barrier.abort()

        th = [threading.Thread(target=body, args=(r,)) for r in range(self.world)]
        for t in th:
            t.start()
        for t in th:
            t.join()
        if err:
            raise err[0]
        return res


class _LocalTransport:
    def __init__(self, fabric: LocalFabric, rank: int):
        self.f = fabric
        self.world = fabric.world
        self.rank = rank

    def exchange_counts(self, send: torch.Tensor) -> np.ndarray:
        f = self.f
        f.box[("c", self.rank)] = send.cpu().numpy().reshape(self.world, -1)
        f.barrier.wait()
        recv = np.stack([f.box[("c", s)][self.rank] for s in range(self.world)])
        f.barrier.wait()
        return recv

    def exchange(self, sends, recvs):
        f = self.f
        f.box[("s", self.rank)] = sends
        f.barrier.wait()
        taken = {s: 0 for s in range(self.world)}
        for s, dst in recvs:
            mine = [t for p, t in f.box[("s", s)] if p == self.rank]
            dst.copy_(mine[taken[s]])
            taken[s] += 1
        f.barrier.wait()

    def all_reduce_sum(self, t: torch.Tensor):
        f = self.f
        f.box[("r", self.rank)] = t.clone()
        f.barrier.wait()
        acc = f.box[("r", 0)].clone()
        for s in range(1, self.world):
            acc += f.box[("r", s)]
        f.barrier.wait()
        t.copy_(acc)


class ExpertShard:
    """The part of a layer one expert-parallel rank computes with: the router and the
    shared expert in full, and the routed experts [rank n_local, (rank+1) n_local). It reads
    the routed weights of its own experts only (views into ``layer``'s packed weights)."""

    def __init__(self, layer, rank: int, world: int):
        if layer.N % world != 0:
            raise ValueError(f"{layer.N} experts do not split evenly over {world} ranks")
        self.layer, self.rank, self.world = layer, rank, world
        n = layer.N // world
        self.n_local = n
        F, d = layer.F, layer.d
        self.gate_up = layer.gate_up[rank * n * 2 * F * d:(rank + 1) * n * 2 * F * d]
        self.w_down = layer.w_down[rank * n:(rank + 1) * n]

    def local_dims(self, T: int):
        from . import binding as B
        L = self.layer
        return B.dims(T, L.d, self.n_local, 0, 1, L.F, L.F_shared, 0)


def ep_forward(shard: ExpertShard, x: torch.Tensor, tok_null_bias: Optional[torch.Tensor], out: Dict,
               transport, sums: torch.Tensor) -> Dict:
    """One expert-parallel layer step on this rank's tokens (see the module docstring).
    ``out`` comes from ``shard.layer.alloc(T)`` with the combine "inplace" or "separate" (it
    runs after the return exchange, not inside the down GEMM); ``sums`` is a
    float64 device tensor of ``aux_sums_count`` elements. Adds ``out["ep_plan"]``."""
    from . import binding as B
    layer = shard.layer
    T = x.shape[0]
    dm = layer.dims(T)
    ws = out["workspace"]
    if out.get("shared_out") is None or out.get("xs") is None:
        raise ValueError("expert parallelism needs xs and a shared-expert output buffer (or y)")
    if layer.router_split is not None:
        B.route_prepared(dm, x, layer.router_split, layer.router_bias, tok_null_bias, out.get("logits"),
                         out["topk_idx"], out["topk_gate"], out["n_real"], ws)
    else:
        B.route(dm, x, layer.w_router, layer.router_bias, tok_null_bias, out.get("logits"), out["topk_idx"],
                out["topk_gate"], out["n_real"], ws)
    B.aux_sums(dm, ws, sums)
    transport.all_reduce_sum(sums)
    B.aux_finalize(dm, sums, out["counts_ext"], out["P"], out["losses"])
    B.dispatch(dm, x, out["topk_idx"], ws, out["counts"], out["offsets"], out["perm_tok"], out["slot_row"],
               out["xs"])
    recv = transport.exchange_counts(out["counts"])
    plan = make_plan(out["counts"].cpu().numpy(), recv, transport.world, transport.rank)
    dev = x.device
    rows = max(plan.rows_recv, 1)
    xs_recv = torch.empty((rows, layer.d), dtype=torch.bfloat16, device=dev)
    transport.exchange(*dispatch_ops(plan, out["xs"], xs_recv))
    offsets_local = torch.from_numpy(plan.offsets_local.astype(np.int32)).to(dev)
    h_recv = torch.empty((rows, layer.F), dtype=torch.bfloat16, device=dev)
    ys_recv = torch.empty((rows, layer.d), dtype=torch.bfloat16, device=dev)
    dl = shard.local_dims(T)
    B.expert_gate_up_rows(dl, rows, xs_recv, x, offsets_local, shard.gate_up, layer.shared_gate_up, h_recv,
                          out["h_shared"], ws)
    B.expert_down_rows(dl, rows, offsets_local, h_recv, out["h_shared"], shard.w_down, layer.shared_down, ys_recv,
                       out["shared_out"], ws)
    transport.exchange(*combine_ops(plan, ys_recv, out["ys"]))
    B.combine(dm, out["ys"], out["shared_out"], out["topk_gate"], out["slot_row"], out["y"],
              topk_idx=out["topk_idx"], x=x, const_vectors=layer.const_vectors)
    out["ep_plan"] = plan
    return out
