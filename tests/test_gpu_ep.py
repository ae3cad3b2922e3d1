"""Expert parallelism with the CUDA kernels on one GPU: W ranks run as threads of one
process (ep.LocalFabric), each with its own tokens and its shard of the routed experts; the
exchanges are device copies in stream order. A row's expert output does not depend on
which rank or tile computes it, so every rank's y must be bit-identical to the one-GPU
forward's rows for its tokens, and the all-reduced losses must match the whole batch's.
The row-capacity GEMM entry points are also checked against the oracle directly.
"""
import numpy as np
import pytest
import torch

import oracle as O
from token_choice_routing_b200 import ep
from token_choice_routing_b200 import inputs as I
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,world", [("qwen3_0p6b", 2), ("qwen3_0p6b", 4), ("skew_small", 4), ("m0", 2)])
def test_expert_parallel_forward_matches_one_gpu(name, world):
    from token_choice_routing_b200 import binding as B
    cfgs = {"skew_small": I.small_config("ep_skew", T=1024, d=256, N=64, F=128, F_shared=128, K=8, M=64,
                                         config_id=950, skew=True, seqs=2),
            "m0": I.small_config("ep_m0", T=600, d=256, N=16, F=128, F_shared=128, K=2, M=0, config_id=951)}
    cfg = I.CONFIGS[name] if name in I.CONFIGS else cfgs[name]
    inp = I.make_inputs(cfg)
    layer, x, tnb = H.make_layer(inp)
    ref = layer.forward(x, tnb, layer.alloc(cfg.T))
    torch.cuda.synchronize()
    bounds = np.linspace(0, cfg.T, world + 1).astype(int)
    fabric = ep.LocalFabric(world)
    nsum = B.aux_sums_count(layer.dims(1))

    def rank_fn(rank, tr):
        a, b = int(bounds[rank]), int(bounds[rank + 1])
        shard = ep.ExpertShard(layer, rank, world)
        out = layer.alloc(b - a)
        sums = torch.zeros(nsum, dtype=torch.float64, device="cuda")
        ep.ep_forward(shard, x[a:b], None if tnb is None else tnb[a:b], out, tr, sums)
        torch.cuda.synchronize()
        return out

    outs = fabric.run(rank_fn)
    sent = 0
    for rank, out in enumerate(outs):
        a, b = int(bounds[rank]), int(bounds[rank + 1])
        assert B.get_device_status(out["workspace"]) == B.OK
        assert torch.equal(out["y"][:b - a], ref["y"][a:b]), rank
        assert torch.equal(out["topk_idx"], ref["topk_idx"][a:b])
        assert torch.equal(out["counts_ext"], ref["counts_ext"])     # whole-batch statistics
        np.testing.assert_allclose(out["losses"].cpu().numpy(), ref["losses"].cpu().numpy(), rtol=1e-6)
        plan = out["ep_plan"]
        assert int(plan.send.sum()) == int(out["n_real"].sum())      # null slots are never sent
        sent += int(plan.rows_recv)
    assert sent == int(ref["offsets"][-1])


def test_row_capacity_gemms_against_the_oracle():
    """moe_expert_gate_up_rows / moe_expert_down_rows on an expert shard (experts 3..5 of 8)
    with a row capacity unrelated to T*K, ragged segments and an empty expert."""
    from token_choice_routing_b200 import binding as B
    cfg = I.small_config("rows", T=200, d=256, N=8, F=192, F_shared=128, K=2, M=2, config_id=952)
    inp = I.make_inputs(cfg)
    layer, x, tnb = H.make_layer(inp)
    rng = np.random.default_rng(952)
    seg = [300, 0, 129]                      # rows received per shard expert
    rows_cap = sum(seg) + 77                 # more than T*K = 400 would allow, with slack
    xs = torch.from_numpy(rng.standard_normal((rows_cap, cfg.d)).astype(np.float32)).to(torch.bfloat16).cuda()
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(seg)]), dtype=torch.int32, device="cuda")
    e0, n = 3, 3
    F, d = cfg.F, cfg.d
    gate_up = layer.gate_up[e0 * 2 * F * d:(e0 + n) * 2 * F * d]
    w_down = layer.w_down[e0:e0 + n]
    dm = B.dims(cfg.T, d, n, 0, 1, F, cfg.F_shared)
    h = torch.empty((rows_cap, F), dtype=torch.bfloat16, device="cuda")
    ys = torch.empty((rows_cap, d), dtype=torch.bfloat16, device="cuda")
    hs = torch.empty((cfg.T, cfg.F_shared), dtype=torch.bfloat16, device="cuda")
    so = torch.empty((cfg.T, d), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    B.expert_gate_up_rows(dm, rows_cap, xs, x, offsets, gate_up, layer.shared_gate_up, h, hs, ws)
    B.expert_down_rows(dm, rows_cap, offsets, h, hs, w_down, layer.shared_down, ys, so, ws)
    torch.cuda.synchronize()
    assert B.get_device_status(ws) == B.OK
    ex, sh = H.expert_weights(inp)
    xf = xs.float().cpu().numpy().astype(np.float64)
    off = offsets.cpu().numpy()
    for j in range(n):
        a, b = off[j], off[j + 1]
        if a == b:
            continue
        g = xf[a:b] @ ex[0][e0 + j].T
        u = xf[a:b] @ ex[1][e0 + j].T
        hg = H.bf16_f64(h[a:b])
        H.check_y(hg, g / (1 + np.exp(-g)) * u)
        H.check_y(H.bf16_f64(ys[a:b]), hg @ ex[2][e0 + j].T)
    xr = H.f64(inp.x)
    H.check_y(H.bf16_f64(so), O.swiglu(xr, *sh))
