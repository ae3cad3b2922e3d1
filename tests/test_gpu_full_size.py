"""GPU parity at the benchmark's full sizes, element by element, and of the data-parallel
statistics path.

* The data-parallel statistics (Kilian et al., review page, 三 / 负载均衡损失: f_i and P_i
  are means over every token of the batch): a 0.6B-shaped batch split in two halves, each
  routed on its own with moe_aux_sums, the two float64 vectors added on the device and
  moe_aux_finalize called once, must give the whole batch's counts (bit-exact), P, L_bal
  and L_z (1e-5) of the oracle; and dp_forward in a one-rank process group must give
  exactly what moe_forward gives.
* The expert GEMMs (三 / 核心公式) at the 0.6B, 1.7B and skewed workloads' full sizes: every
  row of h and ys of four experts (the most and the least loaded, two more at random) and
  >= 2048 rows of the shared expert, each against float64 products.
* The backward at the 0.6B and 1.7B shapes and on the skewed 131072-token batch (the
  benchmark's workload; 四 / 训练配置 trains the layer with both losses): every gradient in
  full against the oracle's layer_backward, in training mode (pre-activations saved by the
  forward) and with the pre-activations recomputed.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle as O
from token_choice_routing_b200 import inputs as I
from tests import gpu_helpers as H
from tests.test_gpu_backward import ALPHA, BETA, check_all

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_dp_statistics_of_a_split_batch_match_the_whole_batch():
    from token_choice_routing_b200 import binding as B
    cfg = I.CONFIGS["qwen3_0p6b"]
    inp = I.make_inputs(cfg)
    layer, x, tnb, out = H.run_forward(inp)
    halves = [(0, cfg.T // 2 + 37), (cfg.T // 2 + 37, cfg.T)]  # unequal halves: ragged route tiles
    dm_all = layer.dims(cfg.T)
    total = torch.zeros(B.aux_sums_count(dm_all), dtype=torch.float64, device="cuda")
    logits = []
    for a, b in halves:
        T = b - a
        o = layer.alloc(T)
        dm = layer.dims(T)
        B.route(dm, x[a:b], layer.w_router, layer.router_bias, None if tnb is None else tnb[a:b], o["logits"],
                o["topk_idx"], o["topk_gate"], o["n_real"], o["workspace"])
        sums = torch.empty(B.aux_sums_count(dm), dtype=torch.float64, device="cuda")
        B.aux_sums(dm, o["workspace"], sums)
        total += sums
        st = B.get_device_status(o["workspace"])
        assert st == B.OK, B.status_string(st)
        logits.append(o["logits"][:T].cpu())
    counts_ext = torch.empty_like(out["counts_ext"])
    P = torch.empty_like(out["P"])
    losses = torch.empty_like(out["losses"])
    B.aux_finalize(dm_all, total, counts_ext, P, losses)
    torch.cuda.synchronize()
    # the halves' logits are the whole batch's (a token's logits do not depend on its tile)
    assert torch.equal(torch.cat(logits), out["logits"][:cfg.T].cpu())
    r = O.route(torch.cat(logits).numpy().astype(np.float64), cfg.M, cfg.K)
    ce, f, Pref, L_bal, L_z = O.aux_stats(r["idx"], r["p"], r["lse"], cfg.N, cfg.M)
    assert np.array_equal(counts_ext.cpu().numpy(), ce)
    np.testing.assert_allclose(P.cpu().numpy(), Pref, rtol=H.P_REL, atol=1e-9)
    lb, lz = losses.cpu().numpy().astype(np.float64)
    assert abs(lb - L_bal) <= H.LOSS_REL * abs(L_bal) and abs(lz - L_z) <= H.LOSS_REL * abs(L_z)
    # and the single call's statistics over the whole batch
    assert torch.equal(counts_ext, out["counts_ext"])
    np.testing.assert_allclose(P.cpu().numpy(), out["P"].cpu().numpy(), rtol=1e-6, atol=1e-12)
    np.testing.assert_allclose(losses.cpu().numpy(), out["losses"].cpu().numpy(), rtol=1e-6)


@pytest.mark.parametrize("combine", ["inplace", "separate", "fused"])
def test_dp_forward_in_a_one_rank_group_equals_forward_bitwise(combine):
    """dp_forward's sequence (route, aux sums, NCCL all-reduce, finalize, dispatch, expert GEMMs,
    combine in the down GEMM or on its own) with one rank is moe_forward, bit for bit."""
    import torch.distributed as dist
    from token_choice_routing_b200 import binding as B
    from token_choice_routing_b200.dist import dp_forward
    cfg = I.CONFIGS["qwen3_0p6b"]
    inp = I.make_inputs(cfg)
    layer, x, tnb, ref = H.run_forward(inp, combine=combine)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        out = layer.alloc(cfg.T, combine=combine)
        sums = torch.zeros(B.aux_sums_count(layer.dims(cfg.T)), dtype=torch.float64, device="cuda")
        dp_forward(layer, x, tnb, out, sums)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    st = B.get_device_status(out["workspace"])
    assert st == B.OK, B.status_string(st)
    R = int(ref["offsets"][-1])
    keys = ["logits", "topk_idx", "topk_gate", "n_real", "counts", "offsets", "slot_row", "h_shared", "y",
            "counts_ext", "P", "losses"] + (["shared_out"] if combine == "separate" else [])
    for k in keys:
        assert torch.equal(out[k], ref[k]), k
    for k in ("perm_tok", "xs", "h", "ys"):
        assert torch.equal(out[k][:R], ref[k][:R]), k
    assert int(sums[-1].item()) == cfg.T


def _pick_experts(counts, rng):
    nz = [e for e in range(len(counts)) if counts[e] > 0]
    big = max(nz, key=lambda e: (counts[e], -e))
    small = min(nz, key=lambda e: (counts[e], e))
    rest = [e for e in nz if e not in (big, small)]
    return [big, small] + [int(e) for e in rng.choice(rest, size=min(2, len(rest)), replace=False)]


@pytest.mark.parametrize("name", ["qwen3_0p6b", "qwen3_1p7b", "skew"])
def test_full_size_expert_gemms_row_by_row(name):
    cfg = I.CONFIGS[name]
    inp = I.make_inputs(cfg)
    layer, x, tnb, out = H.run_forward(inp)
    r = H.check_routing(inp, out)
    counts, offsets, perm, slot_row = H.check_dispatch(inp, out, r)
    ex, sh = H.expert_weights(inp)
    rng = np.random.default_rng(5)
    experts = _pick_experts(counts, rng)
    for e in experts:
        a, b = int(offsets[e]), int(offsets[e + 1])
        z = H.f64(inp.x[perm[a:b]])
        g = z @ ex[0][e].T
        u = z @ ex[1][e].T
        h_gpu = H.bf16_f64(out["h"][a:b])
        H.check_y(h_gpu, g / (1 + np.exp(-g)) * u)
        H.check_y(H.bf16_f64(out["ys"][a:b]), h_gpu @ ex[2][e].T)
    rows = np.unique(np.concatenate([np.arange(128), rng.choice(cfg.T, size=2048, replace=False),
                                     np.arange(cfg.T - 130, cfg.T)]))
    xf = H.f64(inp.x[rows])
    g = xf @ sh[0].T
    u = xf @ sh[1].T
    hs = H.bf16_f64(out["h_shared"][rows])
    H.check_y(hs, g / (1 + np.exp(-g)) * u)
    H.check_y(H.bf16_f64(out["shared_out"][rows]), hs @ sh[2].T)


@pytest.mark.parametrize("name", ["qwen3_0p6b", "qwen3_1p7b", "skew"])
def test_full_size_backward_against_the_oracle(name):
    """Every gradient in full, both ways of getting the gate/up pre-activations."""
    from token_choice_routing_b200 import binding as B
    from token_choice_routing_b200.layer import bf16_tensor
    cfg = I.CONFIGS[name]
    inp = I.make_inputs(cfg)
    layer, x, tnb = H.make_layer(inp)
    out = layer.forward(x, tnb, layer.alloc(cfg.T, save_preact=True))
    dy_bits = I.upstream_grad(cfg)
    dy = bf16_tensor(dy_bits, "cuda")
    g_train = layer.backward(x, out, dy, ALPHA, BETA)
    torch.cuda.synchronize()
    assert B.get_device_status(g_train["workspace"]) == B.OK
    s = out["logits"].cpu().numpy().astype(np.float64)
    ex, sh = H.expert_weights(inp)
    ref = O.layer_backward(H.f64(inp.x), s, inp.w_router.astype(np.float64), cfg.N, cfg.M, cfg.K, ex, sh,
                           H.f64(dy_bits), ALPHA, BETA)
    counts = out["counts"].cpu().numpy()
    check_all(inp, out, g_train, ref, counts)
    g_train = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in g_train.items()}
    # the same forward's outputs without the saved pre-activations: recomputed on the tensor cores
    rec = dict(out)
    rec["z"] = rec["z_shared"] = None
    g_rec = layer.backward(x, rec, dy, ALPHA, BETA)
    torch.cuda.synchronize()
    assert B.get_device_status(g_rec["workspace"]) == B.OK
    check_all(inp, out, g_rec, ref, counts)
