"""Data-parallel execution of the null-expert MoE layer.

Every rank holds the full router and expert weights and runs the layer on its
own tokens; y needs no exchange. The load-balance loss is a product of global
means (f_i and P_i are averages over all tokens: Kilian et al., "Improving MoE
Compute Efficiency by Composing Weight and Data Sparsity", review page,
section 三 / 负载均衡损失), so ranks all-reduce the additive statistics, not the
per-rank losses: one SUM all-reduce of a float64 vector laid out as

    [counts_real (N) | null-slot histogram (K+1) | sum_t p (N+1) | sum_t lse^2 | T]

(moe_aux_sums writes it, moe_aux_finalize reads it). Counts are integers held
exactly in float64, so the reduced statistics equal a single-rank run's up to
the order of the float64 sums.
"""
from __future__ import annotations

from typing import Dict

import torch
import torch.distributed as dist


def aux_sums_slices(N: int, K: int, PP: int = 0) -> Dict[str, slice]:
    """Layout of moe_aux_sums' vector; PP = MoE++ copy + constant experts (their slot
    counts follow the null histogram, their probability sums follow the null logit's)."""
    o = 0
    out = {}
    for name, n in (("counts_real", N), ("null_hist", K + 1 + PP), ("psum", N + 1 + PP), ("lse2", 1), ("T", 1)):
        out[name] = slice(o, o + n)
        o += n
    return out


def allreduce_aux_sums(sums: torch.Tensor, group=None) -> torch.Tensor:
    """In-place SUM all-reduce of one rank's aux statistics vector."""
    if sums.dtype != torch.float64:
        raise TypeError("aux statistics are float64")
    dist.all_reduce(sums, op=dist.ReduceOp.SUM, group=group)
    return sums


def dp_forward(layer, x, tok_null_bias, out, sums, group=None):
    """One data-parallel layer step on this rank's tokens (stream-ordered).

    route -> local aux sums -> all-reduce -> global L_bal/L_z -> dispatch ->
    expert GEMMs -> combine. ``out`` comes from ``layer.alloc``; ``sums`` is a
    float64 CUDA tensor of ``aux_sums_count`` elements.
    """
    from . import binding as B
    dm = layer.dims(x.shape[0])
    ws = out["workspace"]
    if getattr(layer, "router_split", None) is not None:
        B.route_prepared(dm, x, layer.router_split, layer.router_bias, tok_null_bias, out.get("logits"),
                         out["topk_idx"], out["topk_gate"], out["n_real"], ws)
    else:
        B.route(dm, x, layer.w_router, layer.router_bias, tok_null_bias, out.get("logits"), out["topk_idx"],
                out["topk_gate"], out["n_real"], ws)
    B.aux_sums(dm, ws, sums)
    allreduce_aux_sums(sums, group)
    B.aux_finalize(dm, sums, out["counts_ext"], out["P"], out["losses"])
    xs = out.get("xs")
    B.dispatch(dm, x, out["topk_idx"], ws, out["counts"], out["offsets"], out["perm_tok"], out["slot_row"], xs)
    if xs is None:  # gate/up gathers the routed rows of x itself
        B.expert_gate_up_gather(dm, x, out["perm_tok"], out["offsets"], layer.gate_up, layer.shared_gate_up,
                                out["h"], out["h_shared"], ws)
    else:
        B.expert_gate_up(dm, xs, x, out["offsets"], layer.gate_up, layer.shared_gate_up, out["h"], out["h_shared"],
                         ws)
    if out.get("shared_out") is None:  # the combine inside the down GEMM's shared-expert tiles
        B.expert_down_combine(dm, out["offsets"], out["h"], out["h_shared"], layer.w_down, layer.shared_down,
                              out["ys"], out["topk_gate"], out["slot_row"], out["y"], ws, topk_idx=out["topk_idx"],
                              x=x, const_vectors=layer.const_vectors)
    else:
        B.expert_down(dm, out["offsets"], out["h"], out["h_shared"], layer.w_down, layer.shared_down, out["ys"],
                      out["shared_out"], ws)
        B.combine(dm, out["ys"], out["shared_out"], out["topk_gate"], out["slot_row"], out["y"],
                  topk_idx=out["topk_idx"], x=x, const_vectors=layer.const_vectors)
    return out


# Weight gradients summed over the ranks in data-parallel training. dx and the per-token
# null-offset gradient belong to each rank's own tokens and are not reduced.
GRAD_SUM_KEYS = ("dw_router", "dbias", "dw_gate", "dw_up", "dw_down", "dws_gate", "dws_up", "dws_down", "dconst")


def allreduce_token_total(T_local: int, device="cpu", group=None) -> int:
    """Tokens over all ranks (the denominator of f_i and of both losses' means)."""
    t = torch.tensor([int(T_local)], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return int(t.item())


def allreduce_grads(grads: Dict[str, torch.Tensor], keys=GRAD_SUM_KEYS, group=None) -> Dict[str, torch.Tensor]:
    """In-place SUM all-reduce of the weight gradients. Each rank's backward differentiates
    its own tokens' terms of <y, dy> + alpha L_bal + beta L_z with the whole-batch f_i and
    token total, so the sum over ranks is the whole batch's gradient.

    bf16 gradients (the expert weights') are summed in float32 and rounded to bf16 once:
    each is widened into a float32 staging tensor, all-reduced, and written back. A bf16
    all-reduce would round after every partial sum, so its error would grow with the
    number of ranks; here it is one rounding of the float32 sum."""
    for k in keys:
        t = grads.get(k)
        if t is None or t.numel() == 0:
            continue
        if t.dtype in (torch.bfloat16, torch.float16):
            acc = t.to(torch.float32)
            dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)
            t.copy_(acc)
        else:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return grads


def dp_backward(layer, x, out, dy, t_total: int, alpha: float = 2e-2, beta: float = 1e-3, grads=None, group=None,
                reduce_grads: bool = True):
    """Data-parallel backward after ``dp_forward``: ``out["counts_ext"]`` already holds the
    all-reduced slot counts and ``t_total`` is ``allreduce_token_total`` of the ranks' T. The
    weight gradients are then summed over the ranks (``reduce_grads``)."""
    g = layer.backward(x, out, dy, alpha, beta, grads=grads, t_total=t_total)
    if reduce_grads:
        allreduce_grads(g, group=group)
    return g
