"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Routing outputs (top-K indices, counts, offsets, permutation, slot rows, the
gathered rows) must be bit-exact with the oracle run on the GPU's fp32 logits;
logits within a rigorous fp32 dot-product bound of the oracle's fp64 logits;
gates to 1e-6; y to rel. Frobenius 1e-2 and max|dy| <= 5e-2 max|y|; L_bal and
L_z to 1e-5 relative.
"""
import numpy as np
import pytest
import torch

import oracle as O
from token_choice_routing_b200 import inputs as I
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": I.CONFIGS["tiny"],
    # several route tiles with a ragged tail, N not a multiple of 8, M < K
    "ragged_a": I.small_config("ragged_a", T=200, d=256, N=5, F=128, F_shared=192, K=3, M=1, config_id=901),
    "ragged_b": I.small_config("ragged_b", T=333, d=384, N=13, F=192, F_shared=64, K=5, M=9, config_id=902),
    "m0": I.small_config("m0", T=130, d=256, N=16, F=128, F_shared=128, K=2, M=0, config_id=903),
    "k1": I.small_config("k1", T=257, d=128, N=32, F=64, F_shared=64, K=1, M=32, config_id=904),
    "n64_k16": I.small_config("n64_k16", T=190, d=512, N=64, F=256, F_shared=256, K=16, M=48, config_id=905),
    "t1": I.small_config("t1", T=1, d=128, N=8, F=64, F_shared=64, K=4, M=8, config_id=906),
    "skew_small": I.small_config("skew_small", T=512, d=256, N=64, F=128, F_shared=128, K=8, M=64,
                                 config_id=907, skew=True, seqs=2),
    # T K > 128 N: the expert GEMMs take their 256-wide column tiles (ragged expert tails)
    "bn256": I.small_config("bn256", T=600, d=256, N=4, F=256, F_shared=128, K=2, M=2, config_id=908),
}


# (router, expert GEMM kernel, routed rows copied into xs or gathered inside gate/up)
VARIANTS = [("tensor", "single", False), ("tensor", "single", True), ("fp32_cores", "single", True),
            ("tensor", "pair", True), ("fp32_cores", "pair", False)]


@pytest.mark.parametrize("router,ffn,xs", VARIANTS)
@pytest.mark.parametrize("name", list(SMALL))
def test_small_layer_full_parity(name, router, ffn, xs):
    cfg = SMALL[name]
    inp = I.make_inputs(cfg)
    if cfg.name.startswith("ragged") or cfg.name in ("k1", "n64_k16", "t1"):
        inp.bias[cfg.N] = np.float32(0.3)
    layer, x, tnb, out = H.run_forward(inp, router=router, ffn=ffn, xs=xs)
    r = H.check_routing(inp, out)
    H.check_dispatch(inp, out, r)
    H.check_aux(inp, out, r)
    # each GEMM against the oracle's definition on the GPU's own inputs
    counts, offsets, perm, slot_row = O.dispatch(r["idx"], cfg.N)
    R = int(offsets[-1])
    ex, sh = H.expert_weights(inp)
    xs = H.f64(inp.x)[perm]
    h_gpu = H.bf16_f64(out["h"][:R])
    for e in range(cfg.N):
        a, b = offsets[e], offsets[e + 1]
        if a == b:
            continue
        g = xs[a:b] @ ex[0][e].T
        u = xs[a:b] @ ex[1][e].T
        h_ref = g / (1 + np.exp(-g)) * u
        H.check_y(h_gpu[a:b], h_ref)
        ys_ref = h_gpu[a:b] @ ex[2][e].T
        H.check_y(H.bf16_f64(out["ys"][a:b]), ys_ref)
    xf = H.f64(inp.x)
    g = xf @ sh[0].T
    u = xf @ sh[1].T
    H.check_y(H.bf16_f64(out["h_shared"][:cfg.T]), g / (1 + np.exp(-g)) * u)
    H.check_y(H.bf16_f64(out["shared_out"][:cfg.T]), H.bf16_f64(out["h_shared"][:cfg.T]) @ sh[2].T)
    H.check_layer_output(inp, out, r)


@pytest.mark.parametrize("name,router,ffn,xs", [("qwen3_0p6b", "tensor", "single", False),
                                                ("qwen3_1p7b", "tensor", "single", False),
                                                ("qwen3_0p6b", "tensor", "single", True),
                                                ("qwen3_0p6b", "fp32_cores", "single", True),
                                                ("qwen3_0p6b", "tensor", "pair", True)])
def test_full_size_layer_parity_sampled(name, router, ffn, xs):
    cfg = I.CONFIGS[name]
    inp = I.make_inputs(cfg)
    layer, x, tnb, out = H.run_forward(inp, router=router, ffn=ffn, xs=xs)
    r = H.check_routing(inp, out)
    H.check_dispatch(inp, out, r)
    H.check_aux(inp, out, r)
    rng = np.random.default_rng(0)
    tokens = np.sort(rng.choice(cfg.T, size=384, replace=False))
    tokens = np.concatenate([tokens, [0, cfg.T - 1]])
    H.check_layer_output(inp, out, r, tokens=tokens)
    # mean real count near rho*K (the calibrated null bias)
    assert abs(out["n_real"].float().mean().item() - cfg.rho * cfg.K) < 0.02


@pytest.mark.parametrize("name,ffn", [("sweep_k2_m0", "single"), ("sweep_k3_m32", "single"),
                                      ("sweep_k4_m64", "single"), ("sweep_k8_m192", "auto"), ("skew", "single"),
                                      ("skew", "auto")])
def test_large_configs_routing_and_sampled_output(name, ffn):
    """The forward as the benchmark runs it (the shared expert written into y, the combine in
    place; with ffn="auto" these sizes take the CTA-pair GEMMs), against the oracle."""
    cfg = I.CONFIGS[name]
    inp = I.make_inputs(cfg)
    layer, x, tnb, out = H.run_forward(inp, ffn=ffn, combine="inplace")
    r = H.check_routing(inp, out)
    H.check_dispatch(inp, out, r)
    H.check_aux(inp, out, r)
    rng = np.random.default_rng(1)
    tokens = np.sort(rng.choice(cfg.T, size=192, replace=False))
    H.check_layer_output(inp, out, r, tokens=tokens)


def test_route_on_cta_pairs_with_an_odd_tile_count():
    """Above 148 route tiles the route runs on CTA pairs; with an odd tile count the last
    pair's second CTA has no tokens (loaded as zeros, never written). T = 19250: 151 tiles,
    the last one holding 50 tokens. Routing, dispatch and statistics against the oracle, and
    the prepared-weight route bit-identical to the one that splits the weight per call."""
    from token_choice_routing_b200 import binding as B
    cfg = I.small_config("odd_pairs", T=19250, d=256, N=16, F=128, F_shared=128, K=4, M=8, config_id=914)
    assert (cfg.T + 127) // 128 == 151
    inp = I.make_inputs(cfg)
    inp.bias[cfg.N] = np.float32(0.3)
    layer, x, tnb, out = H.run_forward(inp)
    r = H.check_routing(inp, out)
    H.check_dispatch(inp, out, r)
    H.check_aux(inp, out, r)
    dm = layer.dims(cfg.T)
    o = [torch.empty_like(out[k]) for k in ("topk_idx", "topk_gate", "n_real")]
    ws = torch.empty(B.workspace_bytes(dm), dtype=torch.uint8, device="cuda")
    B.route(dm, x, layer.w_router, layer.router_bias, tnb, None, o[0], o[1], o[2], ws)
    torch.cuda.synchronize()
    assert B.get_device_status(ws) == B.OK
    for a, k in zip(o, ("topk_idx", "topk_gate", "n_real")):
        assert torch.equal(a, out[k]), k


@pytest.mark.parametrize("name", ["qwen3_0p6b", "ragged_b", "skew_small", "t1"])
def test_row_gather_matches_row_copy_bitwise(name):
    """Gate/up reading the routed rows of x through TMA row gathers feeds the
    tensor cores exactly the rows dispatch would have copied, so h, ys and y
    are bit-identical to the copy path."""
    cfg = I.CONFIGS[name] if name in I.CONFIGS else SMALL[name]
    inp = I.make_inputs(cfg)
    layer, x, tnb = H.make_layer(inp)
    outs = []
    for xs in (True, False):
        out = layer.forward(x, tnb, layer.alloc(cfg.T, xs=xs, combine="separate"))
        torch.cuda.synchronize()
        outs.append(out)
    R = int(outs[0]["offsets"][-1])
    for k in ("perm_tok", "h", "ys"):
        assert torch.equal(outs[0][k][:R], outs[1][k][:R]), k
    for k in ("h_shared", "shared_out", "y", "losses", "counts_ext"):
        assert torch.equal(outs[0][k], outs[1][k]), k


@pytest.mark.parametrize("name,T", [("decode_0p6b", 1), ("decode_0p6b", 8), ("decode_0p6b", 64),
                                    ("decode_0p6b", 256), ("decode_1p7b", 64)])
def test_decode_sized_forward_parity(name, T):
    """Small-batch forwards with a full-size layer's weights (a few rows per expert; the
    expert GEMMs only read the weights of experts that some token chose)."""
    import dataclasses
    cfg = dataclasses.replace(I.CONFIGS[name], T=T)
    inp = I.make_inputs(cfg)
    layer, x, tnb, out = H.run_forward(inp)
    r = H.check_routing(inp, out)
    counts, offsets, perm, slot_row = H.check_dispatch(inp, out, r)
    H.check_aux(inp, out, r)
    H.check_layer_output(inp, out, r)
    assert int(offsets[-1]) == int(r["n_real"].sum())
    assert (counts == 0).sum() >= cfg.N - int(r["n_real"].sum())  # unchosen experts have empty segments


# MoE++ copy and constant experts next to the null expert
PP = {
    "pp_a": I.small_config("pp_a", T=300, d=256, N=8, F=128, F_shared=128, K=4, M=4, C=2, V=2, config_id=920),
    "pp_b": I.small_config("pp_b", T=200, d=384, N=13, F=64, F_shared=192, K=5, M=0, C=3, V=1, config_id=921),
    "pp_80rows": I.small_config("pp_80rows", T=256, d=256, N=64, F=128, F_shared=128, K=8, M=8, C=10, V=5,
                                config_id=922),
    "pp_copy_only": I.small_config("pp_copy_only", T=130, d=128, N=4, F=64, F_shared=64, K=3, M=2, C=3, V=0,
                                   config_id=923),
    # 65 router rows with a constant expert in logit column 64
    "pp_65rows": I.small_config("pp_65rows", T=200, d=128, N=60, F=64, F_shared=64, K=6, M=4, C=2, V=2,
                                config_id=925),
}


@pytest.mark.parametrize("name", list(PP))
def test_moepp_copy_and_constant_experts_parity(name):
    cfg = PP[name]
    inp = I.make_inputs(cfg)
    inp.bias[cfg.N] = np.float32(0.4)
    inp.bias[cfg.N + 1:] = np.float32(0.6)  # copy/constant experts chosen often enough
    layer, x, tnb, out = H.run_forward(inp)
    r = H.check_routing(inp, out)
    H.check_dispatch(inp, out, r)
    H.check_aux(inp, out, r)
    idx = out["topk_idx"].cpu().numpy()
    assert np.any(idx >= cfg.N + cfg.M)  # some copy/constant slots were taken
    H.check_layer_output(inp, out, r)


def test_moepp_null_copies_precede_copy_and_constant_experts_on_ties():
    """Integer-valued x and 1/8-multiple weights give exact logits: the null row
    equals copy expert 0's and constant expert 0's rows, so on equal logits the
    null copies (pool indices N..N+M-1) must come first."""
    cfg = I.small_config("pp_ties", T=150, d=256, N=6, F=64, F_shared=64, K=5, M=2, C=2, V=2, config_id=924)
    inp = I.make_inputs(cfg)
    rng = np.random.default_rng(924)
    inp.x = I.bf16_round(rng.integers(-3, 4, size=(cfg.T, cfg.d)).astype(np.float32))
    w = (rng.integers(-4, 5, size=(cfg.router_rows, cfg.d)) / 8.0).astype(np.float32)
    w[cfg.N + 1] = w[cfg.N]  # copy expert 0 ties the null logit
    w[cfg.N + 3] = w[cfg.N]  # constant expert 0 ties it too
    inp.w_router = w
    inp.bias[:] = 0
    layer, x, tnb, out = H.run_forward(inp)
    lg = out["logits"].cpu().numpy()
    assert np.array_equal(lg, H.oracle_logits(inp).astype(np.float32))
    r = H.check_routing(inp, out)
    H.check_aux(inp, out, r)
    idx = out["topk_idx"].cpu().numpy()
    n_tie = 0
    for t in range(cfg.T):
        row = idx[t].tolist()
        for sp in (cfg.N + cfg.M, cfg.N + cfg.M + cfg.C):  # copy 0, constant 0
            if sp in row:
                assert all(cfg.N + j in row[:row.index(sp)] for j in range(cfg.M)), row
                n_tie += 1
    assert n_tie > 0
    H.check_layer_output(inp, out, r)


def test_all_null_tokens_get_only_the_shared_expert():
    cfg = I.small_config("allnull", T=100, d=256, N=8, F=64, F_shared=128, K=4, M=8, config_id=910)
    inp = I.make_inputs(cfg, null_bias=1000.0)
    layer, x, tnb, out = H.run_forward(inp)
    assert int(out["n_real"].sum()) == 0
    assert int(out["offsets"][-1]) == 0
    assert torch.equal(out["y"][:cfg.T], out["shared_out"][:cfg.T])
    assert torch.all(out["topk_gate"] == 0)
    r = H.check_routing(inp, out)
    H.check_aux(inp, out, r)
    H.check_layer_output(inp, out, r)


@pytest.mark.parametrize("router", H.ROUTERS)
@pytest.mark.parametrize("N", [8, 15, 64])
def test_one_hot_tokens_read_back_router_weights_exactly(N, router):
    """x_t = 2^k e_{c_t} gives s_tj = 2^k W_r[j, c_t] exactly: a single exact
    product per logit. On the tensor-core path this holds only if the three
    bf16 terms of every fp32 weight add back to it exactly and each term's
    product lands in the right output column (hi, mid and lo side by side)."""
    T, d = 300, 256
    cfg = I.small_config("onehot", T=T, d=d, N=N, F=64, F_shared=64, K=2, M=4, config_id=913)
    inp = I.make_inputs(cfg)
    rng = np.random.default_rng(913)
    c = rng.integers(0, d, size=T)
    k = rng.integers(-3, 4, size=T)
    x = np.zeros((T, d), dtype=np.float32)
    x[np.arange(T), c] = np.ldexp(1.0, k)
    inp.x = I.bf16_round(x)
    # weights spanning many binades, with all 24 significant bits in use
    w = (rng.standard_normal((N + 1, d)) * np.exp2(rng.integers(-20, 4, size=(N + 1, d)))).astype(np.float32)
    inp.w_router = w
    inp.bias[:] = 0
    layer, xt, tnb, out = H.run_forward(inp, router=router)
    lg = out["logits"].cpu().numpy()
    want = (w[:, c].T * np.ldexp(1.0, k)[:, None]).astype(np.float32)
    assert np.array_equal(lg, want), np.argwhere(lg != want)[:5]
    H.check_routing(inp, out)


def test_router_paths_agree_within_twice_the_bound():
    """Tensor-core and fp32 CUDA-core logits on the same full-size inputs: each
    is within the fp32 dot-product bound of the exact value, so they differ by
    at most twice that bound; both route exactly as the oracle does on them."""
    inp = I.make_inputs(I.CONFIGS["qwen3_0p6b"])
    outs = {}
    for router in H.ROUTERS:
        layer, x, tnb, out = H.run_forward(inp, router=router)
        H.check_routing(inp, out)
        outs[router] = out["logits"].cpu().numpy().astype(np.float64)
        del layer, out
        torch.cuda.empty_cache()
    diff = np.abs(outs["tensor"] - outs["fp32_cores"])
    assert np.all(diff <= 2 * H.logit_bound(inp))


@pytest.mark.parametrize("router", H.ROUTERS)
def test_exact_ties_break_by_index(router):
    # Integer-valued x and multiples of 1/8 in W_r make every router logit an
    # exact fp32 value whatever the summation order, so equal rows give equal
    # logits: many real-real ties, and the null row is a copy of real row 2, so
    # real 2 ties the null logit and must precede every copy.
    cfg = I.small_config("ties", T=150, d=256, N=8, F=64, F_shared=64, K=6, M=4, config_id=911)
    inp = I.make_inputs(cfg)
    rng = np.random.default_rng(911)
    inp.x = I.bf16_round(rng.integers(-3, 4, size=(cfg.T, cfg.d)).astype(np.float32))
    w = (rng.integers(-4, 5, size=(cfg.N + 1, cfg.d)) / 8.0).astype(np.float32)
    w[3] = w[1]
    w[5] = w[1]
    w[cfg.N] = w[2]
    inp.w_router = w
    inp.bias[:] = 0
    layer, x, tnb, out = H.run_forward(inp, router=router)
    lg = out["logits"].cpu().numpy()
    assert np.array_equal(lg, H.oracle_logits(inp).astype(np.float32))
    assert np.array_equal(lg[:, 3], lg[:, 1]) and np.array_equal(lg[:, cfg.N], lg[:, 2])
    r = H.check_routing(inp, out)
    H.check_dispatch(inp, out, r)
    H.check_aux(inp, out, r)
    idx = out["topk_idx"].cpu().numpy()
    n_tie = 0
    for t in range(cfg.T):
        row = idx[t].tolist()
        if 2 in row and cfg.N in row:
            assert row.index(2) < row.index(cfg.N)
            n_tie += 1
        if 1 in row and 3 in row:
            assert row.index(1) < row.index(3)
    assert n_tie > 0
    H.check_layer_output(inp, out, r)


def _subset(inp, cfg, rows):
    import dataclasses
    return dataclasses.replace(inp, cfg=cfg, x=np.ascontiguousarray(inp.x[rows]),
                               tok_null_bias=None if inp.tok_null_bias is None else inp.tok_null_bias[rows])


@pytest.mark.parametrize("router", H.ROUTERS)
def test_k4_half_reproduces_k2_dense_bitwise(router):
    """Solution-space preservation (review page, section 三 / 解决方案空间保持):
    with each token's null logit strictly between its 2nd and 3rd real logit,
    K=4/M=64 selects the same two reals as K=2/M=0 and gives the same y."""
    T, d, N, F = 1000, 512, 64, 256
    draw = I.small_config("k4k2_draw", T=1400, d=d, N=N, F=F, F_shared=F, K=4, M=64, config_id=912)
    inp = I.make_inputs(draw)
    inp.bias[:] = 0
    s = O.router_logits(H.f64(inp.x), inp.w_router, inp.bias)
    srt = -np.sort(-s[:, :N], axis=1)
    gap = srt[:, 1] - srt[:, 2]
    rows = np.nonzero(gap > 1e-2)[0][:T]  # a margin the fp32 logits cannot cross
    assert rows.size == T
    cfg4 = I.small_config("k4k2", T=T, d=d, N=N, F=F, F_shared=F, K=4, M=64, config_id=912)
    cfg2 = I.small_config("k4k2_dense", T=T, d=d, N=N, F=F, F_shared=F, K=2, M=0, config_id=912)
    inp4 = _subset(inp, cfg4, rows)
    inp4.tok_null_bias = (0.5 * (srt[rows, 1] + srt[rows, 2]) - s[rows, N]).astype(np.float32)
    inp2 = _subset(inp, cfg2, rows)
    layer4, _, _, out4 = H.run_forward(inp4, router=router)
    layer2, _, _, out2 = H.run_forward(inp2, router=router)
    assert np.all(out4["n_real"].cpu().numpy() == 2)
    H.check_routing(inp4, out4)
    H.check_routing(inp2, out2)
    assert torch.equal(out4["topk_idx"][:, :2], out2["topk_idx"])
    assert torch.all(out4["topk_idx"][:, 2:] >= N)
    assert torch.equal(out4["topk_gate"][:, :2], out2["topk_gate"])
    assert torch.equal(out4["counts"], out2["counts"])
    assert torch.equal(out4["offsets"], out2["offsets"])
    R = int(out2["offsets"][-1])
    assert torch.equal(out4["perm_tok"][:R], out2["perm_tok"][:R])
    assert torch.equal(out4["y"], out2["y"])


def test_zero_tokens_is_a_noop():
    from token_choice_routing_b200 import binding as B
    cfg = I.CONFIGS["tiny"]
    inp = I.make_inputs(cfg)
    layer, x, tnb = H.make_layer(inp)
    out = layer.alloc(0)
    layer.forward(x[:0], None, out)
    torch.cuda.synchronize()


def test_bounded_wait_reports_timeout_and_context_survives():
    from token_choice_routing_b200 import binding as B
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    B.selftest_bounded_wait(ws, 2_000_000)  # 2 ms on a barrier nothing arrives at
    assert B.get_device_status(ws) == B.ERR_TIMEOUT
    B.clear_device_status(ws)
    assert B.get_device_status(ws) == B.OK
    # the context is still usable: a full small forward afterwards
    inp = I.make_inputs(I.CONFIGS["tiny"])
    layer, x, tnb, out = H.run_forward(inp)
    r = H.check_routing(inp, out)
    H.check_layer_output(inp, out, r)


def test_repeated_calls_same_workspace_deterministic():
    inp = I.make_inputs(I.CONFIGS["tiny"])
    layer, x, tnb = H.make_layer(inp)
    out = layer.alloc(inp.cfg.T)
    layer.forward(x, tnb, out)
    y1 = out["y"].clone()
    l1 = out["losses"].clone()
    for _ in range(3):
        layer.forward(x, tnb, out)
    torch.cuda.synchronize()
    assert torch.equal(out["y"], y1) and torch.equal(out["losses"], l1)


# The combine folded into the down GEMM's shared-expert tiles (moe_expert_down_combine, what
# the forward runs when no shared_out buffer is given) against the separate down GEMM and
# combine launches: same arithmetic, so y must be bit-identical; every other output too.
FUSED = [("tiny", "tensor", "single", True), ("ragged_b", "tensor", "single", True),
         ("bn256", "tensor", "single", True), ("m0", "fp32_cores", "single", True),
         ("n64_k16", "tensor", "single", False), ("skew_small", "tensor", "pair", True),
         ("t1", "tensor", "single", True), ("pp_a", "tensor", "single", True), ("pp_b", "tensor", "single", True),
         ("pp_80rows", "tensor", "single", True), ("qwen3_0p6b", "tensor", "single", True),
         ("qwen3_1p7b", "tensor", "single", True), ("skew", "tensor", "single", True),
         ("decode_0p6b", "tensor", "single", True)]


@pytest.mark.parametrize("name,router,ffn,xs", FUSED)
def test_combine_in_down_gemm_is_bitwise_the_separate_combine(name, router, ffn, xs):
    cfg = I.CONFIGS.get(name) or SMALL.get(name) or PP[name]
    inp = I.make_inputs(cfg)
    if cfg.C + cfg.V:
        inp.bias[cfg.N] = np.float32(0.4)
        inp.bias[cfg.N + 1:] = np.float32(0.6)
    layer, x, tnb = H.make_layer(inp, router=router, ffn=ffn)
    ref = layer.forward(x, tnb, layer.alloc(cfg.T, xs=xs, combine="separate"))
    outs = [layer.forward(x, tnb, layer.alloc(cfg.T, xs=xs, combine=c)) for c in ("fused", "fused", "inplace")]
    torch.cuda.synchronize()
    from token_choice_routing_b200 import binding as B
    R = int(ref["offsets"][-1])
    for out in outs:
        assert B.get_device_status(out["workspace"]) == B.OK
        for k in ("y", "topk_idx", "topk_gate", "counts", "offsets", "slot_row", "h_shared", "counts_ext", "P",
                  "losses"):
            assert torch.equal(out[k], ref[k]), k
        for k in ("perm_tok", "h", "ys"):
            assert torch.equal(out[k][:R], ref[k][:R]), k


def test_down_combine_entry_point_called_alone_twice():
    """moe_expert_down_combine on its own, twice in a row after one forward (its counters are
    reset by the last CTA of each launch), gives the forward's y both times."""
    from token_choice_routing_b200 import binding as B
    cfg = I.CONFIGS["qwen3_0p6b"]
    inp = I.make_inputs(cfg)
    layer, x, tnb = H.make_layer(inp)
    out = layer.forward(x, tnb, layer.alloc(cfg.T, combine="fused"))
    torch.cuda.synchronize()
    y0 = out["y"].clone()
    dm = layer.dims(cfg.T)
    for _ in range(2):
        out["y"].zero_()
        B.expert_down_combine(dm, out["offsets"], out["h"], out["h_shared"], layer.w_down, layer.shared_down,
                              out["ys"], out["topk_gate"], out["slot_row"], out["y"], out["workspace"])
        torch.cuda.synchronize()
        assert B.get_device_status(out["workspace"]) == B.OK
        assert torch.equal(out["y"], y0)


# a ragged batch above the persistent grid's threshold (16 tokens per resident warp), routed on
# CTA pairs (more tiles than SMs), with a ragged last tile
LIST_CASES = {"ragged_60k": I.small_config("ragged_60k", T=60001, d=128, N=16, F=64, F_shared=64, K=4, M=16,
                                           config_id=931)}


@pytest.mark.parametrize("name,router", [("skew_small", "tensor"), ("pp_a", "tensor"), ("pp_b", "tensor"),
                                         ("m0", "fp32_cores"), ("t1", "tensor"), ("ragged_b", "tensor"),
                                         ("qwen3_1p7b", "tensor"), ("sweep_k8_m192", "tensor"),
                                         ("ragged_60k", "tensor"), ("ragged_60k", "fp32_cores")])
def test_inplace_combine_over_the_route_token_list(name, router):
    """moe_combine_inplace visits only the tokens the route listed as having a source (a real,
    copy or constant expert): called alone after a forward, with y reset to the shared expert's
    output, it gives the forward's y and moe_combine's in-place y bit for bit. The small grid
    (one token per warp) and the persistent one (sweep_k8_m192, 65536 tokens) both run; every
    token with no source keeps bf16(shared) untouched."""
    from token_choice_routing_b200 import binding as B
    cfg = I.CONFIGS.get(name) or SMALL.get(name) or PP.get(name) or LIST_CASES[name]
    inp = I.make_inputs(cfg)
    if cfg.C + cfg.V:
        inp.bias[cfg.N] = np.float32(0.4)
        inp.bias[cfg.N + 1:] = np.float32(0.6)
    layer, x, tnb = H.make_layer(inp, router=router)
    out = layer.forward(x, tnb, layer.alloc(cfg.T, combine="inplace"))
    torch.cuda.synchronize()
    assert B.get_device_status(out["workspace"]) == B.OK
    y_fwd = out["y"].clone()
    dm = layer.dims(cfg.T)

    def reset_to_shared():
        B.expert_down(dm, out["offsets"], out["h"], out["h_shared"], layer.w_down, layer.shared_down, out["ys"],
                      out["y"], out["workspace"])

    reset_to_shared()
    torch.cuda.synchronize()
    shared = out["y"].clone()
    extra = dict(topk_idx=out["topk_idx"], x=x, const_vectors=layer.const_vectors)
    B.combine(dm, out["ys"], out["y"], out["topk_gate"], out["slot_row"], out["y"], **extra)
    torch.cuda.synchronize()
    y_scan = out["y"].clone()
    for _ in range(2):
        reset_to_shared()
        B.combine_inplace(dm, out["ys"], out["topk_gate"], out["slot_row"], out["y"], out["workspace"], **extra)
        torch.cuda.synchronize()
        assert B.get_device_status(out["workspace"]) == B.OK
        assert torch.equal(out["y"], y_fwd) and torch.equal(out["y"], y_scan)
    # a token has a source iff one of its slots is a real, copy or constant expert
    idx = out["topk_idx"].cpu().numpy()
    has = ((idx < cfg.N) | (idx >= cfg.N + cfg.M)).any(axis=1)
    assert 0 < has.sum() <= cfg.T
    none = torch.from_numpy(~has).to(out["y"].device)
    assert torch.equal(y_fwd[none], shared[none])


@pytest.mark.parametrize("name,chunk,nsets", [("qwen3_0p6b", 4096, 2), ("qwen3_0p6b", 5000, 3),
                                              ("skew_small", 200, 2), ("tiny", 256, 2), ("pp_a", 128, 3)])
def test_forward_from_host_memory_in_chunks(name, chunk, nsets):
    """MoENullLayer.forward_host: the batch in token chunks (short ones at both ends) from and
    to pinned host memory, copies overlapping the chunks' compute, two or three buffer sets.
    y is bit-identical to one forward over the whole batch; the batch's statistics (summed
    over the chunks) give its counts exactly and P and the losses to fp64 summation order."""
    cfg = I.CONFIGS.get(name) or SMALL.get(name) or PP[name]
    inp = I.make_inputs(cfg)
    layer, x, tnb = H.make_layer(inp)
    ref = layer.forward(x, tnb, layer.alloc(cfg.T))
    torch.cuda.synchronize()
    x_pin = x.cpu().pin_memory()
    y_pin = torch.empty_like(x_pin).pin_memory()
    tnb_pin = None if tnb is None else tnb.cpu().pin_memory()
    pipe = layer.alloc_host_pipeline(chunk, nsets)
    for _ in range(2):  # twice: the pipeline's buffers are reused
        y_pin.zero_()
        st = layer.forward_host(x_pin, y_pin, pipe, tnb_pin)
        torch.cuda.synchronize()
        assert torch.equal(y_pin, ref["y"][:cfg.T].cpu())
        assert torch.equal(st["counts_ext"], ref["counts_ext"])
        np.testing.assert_allclose(st["P"].cpu().numpy(), ref["P"].cpu().numpy(), rtol=1e-6, atol=1e-12)
        np.testing.assert_allclose(st["losses"].cpu().numpy(), ref["losses"].cpu().numpy(), rtol=1e-6)


@pytest.mark.parametrize("name", ["decode_0p6b", "skew_small", "pp_a", "t1"])
def test_captured_forward_graph_replays_the_eager_forward(name):
    """MoENullLayer.capture_forward: replaying the CUDA graph of one forward gives the eager
    forward's outputs bit for bit, and after new tokens are copied into x in place it gives
    the eager forward of those tokens; replays are deterministic and leave the status OK."""
    from token_choice_routing_b200 import binding as B
    cfg = I.CONFIGS.get(name) or SMALL.get(name) or PP[name]
    inp = I.make_inputs(cfg)
    if cfg.C + cfg.V:
        inp.bias[cfg.N] = np.float32(0.4)
        inp.bias[cfg.N + 1:] = np.float32(0.6)
    layer, x, tnb = H.make_layer(inp)
    x_static = x.clone()
    out = layer.alloc(cfg.T)
    g = layer.capture_forward(x_static, tnb, out)
    ref1 = layer.forward(x, tnb, layer.alloc(cfg.T))
    x2 = torch.flip(x, dims=[0]).contiguous()  # other tokens: the batch reversed
    ref2 = layer.forward(x2, tnb, layer.alloc(cfg.T))
    torch.cuda.synchronize()
    keys = ("y", "topk_idx", "topk_gate", "n_real", "counts", "offsets", "slot_row", "counts_ext", "P", "losses")
    for xin, ref in ((x, ref1), (x2, ref2), (x, ref1)):
        x_static.copy_(xin)
        for k in ("y", "topk_idx", "counts"):
            out[k].zero_()
        g.replay()
        torch.cuda.synchronize()
        assert B.get_device_status(out["workspace"]) == B.OK
        for k in keys:
            assert torch.equal(out[k], ref[k]), k
    del g


def test_forward_host_batches_of_growing_size_reuse_the_pipeline():
    """One pipeline, host-buffer forwards of 1000 tokens, then 2600, then 1000 again, with
    per-token null offsets (copied in once per call into a device buffer the pipeline keeps
    and grows): each y is bit-identical to the device forward of the same tokens."""
    cfg = I.small_config("skew_3k", T=3072, d=256, N=64, F=128, F_shared=128, K=8, M=64, config_id=930,
                         skew=True, seqs=3)
    inp = I.make_inputs(cfg)
    layer, x, tnb = H.make_layer(inp)
    assert tnb is not None
    pipe = layer.alloc_host_pipeline(512, 3)
    for n in (1000, 2600, 1000):
        ref = layer.forward(x[:n], tnb[:n], layer.alloc(n))
        torch.cuda.synchronize()
        x_pin = x[:n].cpu().pin_memory()
        y_pin = torch.zeros_like(x_pin).pin_memory()
        layer.forward_host(x_pin, y_pin, pipe, tnb[:n].cpu().pin_memory())
        torch.cuda.synchronize()
        assert torch.equal(y_pin, ref["y"][:n].cpu())


@pytest.mark.parametrize("name", ["tiny", "ragged_b", "pp_80rows", "skew"])
def test_route_from_the_prepared_router_weight_is_bitwise_moe_route(name):
    """moe_route_prepared (the weight split once by moe_prepare_router, as the layer's forward
    uses it) gives exactly what moe_route (splitting per call) gives; the fp32 CUDA-core
    router has no prepared form and is refused."""
    from token_choice_routing_b200 import binding as B
    cfg = I.CONFIGS.get(name) or SMALL.get(name) or PP[name]
    inp = I.make_inputs(cfg, weights=False)
    from token_choice_routing_b200.layer import bf16_tensor
    x = bf16_tensor(inp.x, "cuda")
    w = torch.from_numpy(inp.w_router).cuda()
    b = torch.from_numpy(inp.bias).cuda()
    tnb = None if inp.tok_null_bias is None else torch.from_numpy(inp.tok_null_bias).cuda()
    dm = B.dims(cfg.T, cfg.d, cfg.N, cfg.M, cfg.K, cfg.F, cfg.F_shared, 0, cfg.C, cfg.V)
    split = torch.empty(B.router_split_elems(dm), dtype=torch.bfloat16, device="cuda")
    B.prepare_router(dm, w, split)
    outs = []
    for prepared in (False, True):
        ws = torch.empty(B.workspace_bytes(dm), dtype=torch.uint8, device="cuda")
        o = [torch.empty((cfg.T, cfg.router_rows), dtype=torch.float32, device="cuda"),
             torch.empty((cfg.T, cfg.K), dtype=torch.int32, device="cuda"),
             torch.empty((cfg.T, cfg.K), dtype=torch.float32, device="cuda"),
             torch.empty((cfg.T,), dtype=torch.int32, device="cuda")]
        if prepared:
            B.route_prepared(dm, x, split, b, tnb, *o, ws)
        else:
            B.route(dm, x, w, b, tnb, *o, ws)
        torch.cuda.synchronize()
        assert B.get_device_status(ws) == B.OK
        outs.append(o)
    for a, c in zip(*outs):
        assert torch.equal(a, c)
    dm32 = B.dims(cfg.T, cfg.d, cfg.N, cfg.M, cfg.K, cfg.F, cfg.F_shared, B.FLAG_ROUTER_FP32_CORES, cfg.C, cfg.V)
    if cfg.C + cfg.V == 0:
        ws = torch.empty(B.workspace_bytes(dm32), dtype=torch.uint8, device="cuda")
        with pytest.raises(B.MoEError):
            B.route_prepared(dm32, x, split, b, tnb, *outs[0], ws)
