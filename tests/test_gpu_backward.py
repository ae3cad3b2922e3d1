"""GPU parity of the backward pass: the CUDA path (through the C ABI) against the
oracle's layer_backward, run on the GPU's own fp32 logits so both sides take the
same routing.

Tolerances: every gradient to relative Frobenius error 1e-2 (bf16 activations and
bf16 weight gradients, fp32 accumulation; the oracle is fp64 without rounding), each
routed expert's weight gradients to 2e-2, and experts that received no rows exactly
zero. With dy = 0 only the load-balance and Z-loss terms act: the logit, router-weight
and bias gradients then follow from fp32 softmax arithmetic alone and are held to 1e-4,
and every expert gradient is exactly zero.
"""
import numpy as np
import pytest
import torch

import oracle as O
from token_choice_routing_b200 import inputs as I
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

ALPHA, BETA = 2e-2, 1e-3   # the paper's loss weights (review page, 四 / 训练配置)
REL = 1e-2
REL_EXPERT = 2e-2

CASES = {
    "tiny": I.CONFIGS["tiny"],
    # ragged: several 128-row tiles per expert with tails, N not a power of two
    "ragged": I.small_config("bwd_ragged", T=300, d=256, N=12, F=192, F_shared=128, K=3, M=4, config_id=930),
    # F and F_shared multiples of 128 and d a multiple of 256: the wide tiles of every GEMM
    "wide": I.small_config("bwd_wide", T=700, d=512, N=6, F=256, F_shared=384, K=2, M=2, config_id=931),
    # T > 2048: the shared expert's weight gradients are split into K chunks and reduced
    "split": I.small_config("bwd_split", T=4500, d=256, N=8, F=128, F_shared=128, K=4, M=8, config_id=932),
    # d not a multiple of 256 and F not a multiple of 128: the 128- and 64-wide tiles
    "odd": I.small_config("bwd_odd", T=333, d=384, N=13, F=192, F_shared=64, K=5, M=9, config_id=940),
    # M = 0 (plain top-K) and K = 1
    "m0": I.small_config("bwd_m0", T=130, d=128, N=16, F=64, F_shared=64, K=2, M=0, config_id=933),
    "k1": I.small_config("bwd_k1", T=257, d=128, N=32, F=64, F_shared=64, K=1, M=32, config_id=934),
    "t1": I.small_config("bwd_t1", T=1, d=128, N=8, F=64, F_shared=64, K=4, M=8, config_id=935),
    # skewed routing: experts with many rows next to experts with none
    "skew": I.small_config("bwd_skew", T=512, d=256, N=64, F=128, F_shared=128, K=8, M=64, config_id=936,
                           skew=True, seqs=2),
}

PP_CASES = {
    "pp": I.small_config("bwd_pp", T=300, d=256, N=8, F=128, F_shared=128, K=4, M=4, C=2, V=2, config_id=937),
    "pp_copy": I.small_config("bwd_pp_copy", T=160, d=128, N=4, F=64, F_shared=64, K=3, M=2, C=3, V=0,
                              config_id=938),
}


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def run(cfg, dy_scale=1.0, alpha=ALPHA, beta=BETA, router="tensor", ffn="single"):
    inp = I.make_inputs(cfg)
    layer, x, tnb, out = H.run_forward(inp, router=router, ffn=ffn)
    dy_bits = I.upstream_grad(cfg, scale=dy_scale) if dy_scale else np.zeros((cfg.T, cfg.d), np.uint16)
    from token_choice_routing_b200.layer import bf16_tensor
    from token_choice_routing_b200 import binding as B
    dy = bf16_tensor(dy_bits, "cuda")
    g = layer.backward(x, out, dy, alpha, beta)
    torch.cuda.synchronize()
    st = B.get_device_status(g["workspace"])
    assert st == B.OK, B.status_string(st)
    return inp, layer, x, out, dy, dy_bits, g


def oracle_backward(inp, out, dy_bits, alpha, beta):
    c = inp.cfg
    s = out["logits"].cpu().numpy().astype(np.float64)
    experts = (H.f64(inp.w_gate), H.f64(inp.w_up), H.f64(inp.w_down))
    shared = (H.f64(inp.ws_gate), H.f64(inp.ws_up), H.f64(inp.ws_down))
    cv = H.f64(inp.const_vectors) if c.V else None
    return O.layer_backward(H.f64(inp.x), s, inp.w_router.astype(np.float64), c.N, c.M, c.K, experts, shared,
                            H.f64(dy_bits), alpha, beta, C=c.C, V=c.V, const_vectors=cv)


def check_all(inp, out, g, ref, counts):
    c = inp.cfg
    assert np.array_equal(out["topk_idx"].cpu().numpy(), ref["idx"])
    assert rel(f64(g["dx"]), ref["dx"]) < REL
    assert rel(f64(g["dw_router"]), ref["dW_r"]) < REL
    assert rel(f64(g["dbias"]), ref["dbias"]) < REL
    if c.M > 0:
        assert rel(f64(g["dtok_null_bias"]), ref["dtnb"]) < REL
    for k_gpu, k_ref in (("dws_gate", "dWs_gate"), ("dws_up", "dWs_up"), ("dws_down", "dWs_down")):
        assert rel(f64(g[k_gpu]), ref[k_ref]) < REL, k_gpu
    for k_gpu, k_ref in (("dw_gate", "dW_gate"), ("dw_up", "dW_up"), ("dw_down", "dW_down")):
        G, R = f64(g[k_gpu]), ref[k_ref]
        assert rel(G, R) < REL, k_gpu
        for e in range(c.N):
            if counts[e] == 0:
                assert not np.any(G[e]), f"{k_gpu}[{e}] must be zero (expert without rows)"
            else:
                assert rel(G[e], R[e]) < REL_EXPERT, (k_gpu, e, counts[e])
    if c.V:
        assert rel(f64(g["dconst"]), ref["dconst"]) < REL


@pytest.mark.parametrize("name", list(CASES))
def test_backward_parity(name):
    inp, layer, x, out, dy, dy_bits, g = run(CASES[name])
    ref = oracle_backward(inp, out, dy_bits, ALPHA, BETA)
    counts = out["counts"].cpu().numpy()
    check_all(inp, out, g, ref, counts)


@pytest.mark.parametrize("router,ffn", [("fp32_cores", "single"), ("tensor", "pair")])
def test_backward_after_each_forward_path(router, ffn):
    """The backward reads only the forward's outputs: after the fp32 CUDA-core router or the
    CTA-pair expert GEMMs it matches the oracle the same way."""
    inp, layer, x, out, dy, dy_bits, g = run(CASES["wide"], router=router, ffn=ffn)
    ref = oracle_backward(inp, out, dy_bits, ALPHA, BETA)
    check_all(inp, out, g, ref, out["counts"].cpu().numpy())


@pytest.mark.parametrize("name", list(PP_CASES))
def test_backward_parity_moepp(name):
    inp, layer, x, out, dy, dy_bits, g = run(PP_CASES[name])
    ref = oracle_backward(inp, out, dy_bits, ALPHA, BETA)
    idx = out["topk_idx"].cpu().numpy()
    c = inp.cfg
    assert (idx >= c.N + c.M).any(), "the case must select copy or constant experts"
    check_all(inp, out, g, ref, out["counts"].cpu().numpy())


@pytest.mark.parametrize("name", ["tiny", "ragged", "skew"])
def test_backward_loss_terms_only(name):
    """dy = 0: only alpha L_bal + beta L_z act (weights 1 and 0.5 to make them large)."""
    inp, layer, x, out, dy, dy_bits, g = run(CASES[name], dy_scale=0.0, alpha=1.0, beta=0.5)
    ref = oracle_backward(inp, out, dy_bits, 1.0, 0.5)
    for k in ("dw_gate", "dw_up", "dw_down", "dws_gate", "dws_up", "dws_down"):
        assert not torch.any(g[k].float() != 0), k
    assert rel(f64(g["dw_router"]), ref["dW_r"]) < 1e-4
    assert rel(f64(g["dbias"]), ref["dbias"]) < 1e-4
    assert rel(f64(g["dx"]), ref["dx"]) < REL  # router part only, rounded to bf16


def test_backward_step_entry_points_match_the_whole_call():
    """combine, router, router weight, expert FFN and input-gradient entry points called one
    by one give bit-identical gradients to moe_backward: with the shared expert's input
    gradient in a buffer of its own, and in place (written into dx, then the gather over the
    tokens with a real or copy slot, as moe_backward runs it)."""
    from token_choice_routing_b200 import binding as B
    cfg = CASES["ragged"]
    inp, layer, x, out, dy, dy_bits, g = run(cfg)
    T, c = cfg.T, cfg
    dm = layer.dims(T)
    g2 = layer.alloc_grads(T)
    bws = g2["workspace"]
    dev = "cuda"
    R = T * c.K
    dys = torch.empty((R, c.d), dtype=torch.bfloat16, device=dev)
    dg = torch.empty((T, c.K), dtype=torch.float32, device=dev)
    ds = torch.empty((T, c.N + 1), dtype=torch.float32, device=dev)
    dxs = torch.empty((R, c.d), dtype=torch.bfloat16, device=dev)
    dxsh = torch.empty((T, c.d), dtype=torch.bfloat16, device=dev)
    B.clear_device_status(bws)
    B.combine_backward(dm, dy, out["ys"], out["topk_gate"], out["slot_row"], dys, dg, bws)
    B.router_backward(dm, out["logits"], out["topk_idx"], out["topk_gate"], dg, out["counts_ext"], T, ALPHA, BETA,
                      ds, bws, g2["dtok_null_bias"])
    B.router_weight_grad(dm, x, g2["dw_router"], g2["dbias"], bws)
    sv = layer.saved(x, out)
    gr = B.Grads(*[None if g2.get(n) is None else g2[n].data_ptr() for n in B.GRAD_FIELDS])
    B.expert_ffn_backward(dm, layer._weights, sv, dys, dy, dxs, dxsh, gr, bws)
    B.input_grad(dm, dxsh, dxs, out["slot_row"], out["topk_idx"], out["topk_gate"], dy, g2["dx"], bws)
    torch.cuda.synchronize()
    assert B.get_device_status(bws) == B.OK
    for k in ("dx", "dw_router", "dbias", "dtok_null_bias", "dw_gate", "dw_up", "dw_down", "dws_gate", "dws_up",
              "dws_down"):
        assert torch.equal(g[k], g2[k]), k
    # and the five GEMM stages one by one give the same expert gradients and dx, in place
    g3 = layer.alloc_grads(T)
    bws3 = g3["workspace"]
    B.clear_device_status(bws3)
    B.combine_backward(dm, dy, out["ys"], out["topk_gate"], out["slot_row"], dys, dg, bws3)
    B.router_backward(dm, out["logits"], out["topk_idx"], out["topk_gate"], dg, out["counts_ext"], T, ALPHA, BETA,
                      ds, bws3, g3["dtok_null_bias"])
    B.expert_dgrad_down(dm, out["offsets"], dys, dy, layer.w_down, layer.shared_down, bws3)
    B.expert_swiglu_backward(dm, out["xs"], x, out["offsets"], layer.gate_up, layer.shared_gate_up, bws3)
    B.expert_wgrad_down(dm, out["offsets"], dys, dy, out["h"], out["h_shared"], g3["dw_down"], g3["dws_down"], bws3)
    g3["dx"].fill_(7.0)  # every row is overwritten by the shared expert's input gradient
    B.expert_dgrad_gate_up(dm, out["offsets"], layer.gate_up, layer.shared_gate_up, layer.w_router, dxs, g3["dx"],
                           bws3)
    B.expert_wgrad_gate_up(dm, out["offsets"], out["xs"], x, g3["dw_gate"], g3["dw_up"], g3["dws_gate"],
                           g3["dws_up"], bws3)
    B.input_grad(dm, g3["dx"], dxs, out["slot_row"], out["topk_idx"], out["topk_gate"], dy, g3["dx"], bws3)
    torch.cuda.synchronize()
    assert B.get_device_status(bws3) == B.OK
    for k in ("dx", "dw_gate", "dw_up", "dw_down", "dws_gate", "dws_up", "dws_down"):
        assert torch.equal(g[k], g3[k]), k


# shapes where the weight gradients can run on CTA pairs: output rows per expert (d for
# W_down, 2 F and 2 F_shared for gate/up) and columns (F, F_shared, d) multiples of 256
PAIR_CASES = {
    "plain": I.small_config("wgp_plain", T=700, d=512, N=6, F=256, F_shared=256, K=2, M=2, config_id=941),
    # T > 2048: the shared expert's K chunks (fp32 partials, then the reduce)
    "split": I.small_config("wgp_split", T=4500, d=256, N=8, F=256, F_shared=512, K=4, M=8, config_id=942),
    # experts without rows, ragged tails of every length
    "skew": I.small_config("wgp_skew", T=1500, d=512, N=64, F=256, F_shared=256, K=8, M=64, config_id=943,
                           skew=True, seqs=2),
    # F = 384: gate/up on pairs (2F = 768 output rows), down on single CTAs (384 columns)
    "mixed": I.small_config("wgp_mixed", T=900, d=256, N=8, F=384, F_shared=384, K=2, M=2, config_id=944),
}


@pytest.mark.parametrize("name", list(PAIR_CASES))
def test_wgrad_on_cta_pairs_is_bitwise_the_single_cta_wgrad(name):
    """moe_expert_wgrad_down / moe_expert_wgrad_gate_up with MOE_FLAG_WGRAD_CTA_PAIR (256 x 256
    tiles, one MMA shared by two CTAs) give exactly the single-CTA weight gradients: the same
    fp32 sums over the same 16-row steps, in the same order. The layer's backward (pairs by
    default) is checked against the oracle here too."""
    from token_choice_routing_b200 import binding as B
    cfg = PAIR_CASES[name]
    inp, layer, x, out, dy, dy_bits, g = run(cfg)
    T, c = cfg.T, cfg
    flags = layer.dims(T).flags & ~B.FLAG_WGRAD_CTA_PAIR
    dm = B.dims(T, c.d, c.N, c.M, c.K, c.F, c.F_shared, flags, c.C, c.V)
    dmp = B.dims(T, c.d, c.N, c.M, c.K, c.F, c.F_shared, flags | B.FLAG_WGRAD_CTA_PAIR, c.C, c.V)
    g2 = layer.alloc_grads(T)
    bws = g2["workspace"]
    R = T * c.K
    dys = torch.empty((R, c.d), dtype=torch.bfloat16, device="cuda")
    dg = torch.empty((T, c.K), dtype=torch.float32, device="cuda")
    ds = torch.empty((T, c.N + 1), dtype=torch.float32, device="cuda")
    B.clear_device_status(bws)
    B.combine_backward(dm, dy, out["ys"], out["topk_gate"], out["slot_row"], dys, dg, bws)
    B.router_backward(dm, out["logits"], out["topk_idx"], out["topk_gate"], dg, out["counts_ext"], T, ALPHA, BETA,
                      ds, bws, g2["dtok_null_bias"])
    B.expert_dgrad_down(dm, out["offsets"], dys, dy, layer.w_down, layer.shared_down, bws)
    B.expert_swiglu_backward(dm, out["xs"], x, out["offsets"], layer.gate_up, layer.shared_gate_up, bws)
    res = {}
    for tag, d_ in (("single", dm), ("pair", dmp)):
        o = {k: torch.full_like(g[k], float("nan")) for k in ("dw_down", "dws_down", "dw_gate", "dw_up", "dws_gate",
                                                             "dws_up")}
        B.expert_wgrad_down(d_, out["offsets"], dys, dy, out["h"], out["h_shared"], o["dw_down"], o["dws_down"], bws)
        B.expert_wgrad_gate_up(d_, out["offsets"], out["xs"], x, o["dw_gate"], o["dw_up"], o["dws_gate"],
                               o["dws_up"], bws)
        torch.cuda.synchronize()
        assert B.get_device_status(bws) == B.OK
        res[tag] = o
    for k in res["single"]:
        assert torch.equal(res["single"][k].view(torch.int16), res["pair"][k].view(torch.int16)), k
        assert torch.equal(res["single"][k], g[k]), k
    # the layer's backward (weight gradients on pairs by default) against the oracle
    assert layer.dims(T).flags & B.FLAG_WGRAD_CTA_PAIR
    ref = oracle_backward(inp, out, dy_bits, ALPHA, BETA)
    check_all(inp, out, g, ref, out["counts"].cpu().numpy())


def test_backward_is_deterministic():
    cfg = CASES["split"]
    inp, layer, x, out, dy, dy_bits, g = run(cfg)
    g2 = layer.backward(x, out, dy, ALPHA, BETA)
    torch.cuda.synchronize()
    for k in ("dx", "dw_router", "dbias", "dw_gate", "dw_down", "dws_gate", "dws_up", "dws_down"):
        assert torch.equal(g[k], g2[k]), k


def test_backward_data_parallel_statistics():
    """With counts and a token total from several ranks (here a made-up global total), the
    load-balance gradient uses the global f_i and 1/T_total: compare with the oracle's
    aux_backward evaluated on those statistics."""
    from token_choice_routing_b200 import binding as B
    cfg = CASES["tiny"]
    inp, layer, x, out, dy, dy_bits, g = run(cfg, dy_scale=0.0, alpha=1.0, beta=0.5)
    T, c = cfg.T, cfg
    ce = (out["counts_ext"] * 3).contiguous()  # as if three ranks had routed alike
    g3 = layer.backward(x, out, dy, 1.0, 0.5, counts_ext=ce, t_total=3 * T)
    torch.cuda.synchronize()
    s = out["logits"].cpu().numpy().astype(np.float64)
    r = O.route(s, c.M, c.K)
    dv = O.aux_backward(r["idx"], r["p"], r["lse"], c.N, 1.0, 0.5, counts=ce.cpu().numpy(), t_total=3 * T)
    ds = O.pool_grad_to_logits(dv, c.N, c.M)
    assert rel(f64(g3["dbias"]), ds.sum(axis=0)) < 1e-4
    assert rel(f64(g3["dw_router"]), ds.T @ H.f64(inp.x)) < 1e-4


@pytest.mark.parametrize("T", [1, 8, 64])
def test_backward_decode_sized_with_full_weights(T):
    """Small batches with the 0.6B-shaped layer's weights: most experts receive no rows
    (their weight gradients must be exactly zero) and the shared expert's K is a few rows."""
    base = I.CONFIGS["decode_0p6b"]
    cfg = I.small_config("bwd_decode", T=T, d=base.d, N=base.N, F=base.F, F_shared=base.F_shared, K=base.K,
                         M=base.M, config_id=939)
    inp = I.make_inputs(cfg, null_bias=I.NULL_BIAS.get("qwen3_0p6b", 0.0))
    layer, x, tnb, out = H.run_forward(inp)
    from token_choice_routing_b200.layer import bf16_tensor
    from token_choice_routing_b200 import binding as B
    dy_bits = I.upstream_grad(cfg)
    g = layer.backward(x, out, bf16_tensor(dy_bits, "cuda"), ALPHA, BETA)
    torch.cuda.synchronize()
    assert B.get_device_status(g["workspace"]) == B.OK
    ref = oracle_backward(inp, out, dy_bits, ALPHA, BETA)
    check_all(inp, out, g, ref, out["counts"].cpu().numpy())


def test_backward_empty_batch_is_a_no_op():
    """T = 0: the forward and the backward return without touching any buffer."""
    cfg = I.CONFIGS["tiny"]
    inp = I.make_inputs(cfg)
    layer = H.make_layer(inp)[0]
    x0 = torch.empty((0, cfg.d), dtype=torch.bfloat16, device="cuda")
    out = layer.forward(x0, None, layer.alloc(0))
    g = layer.alloc_grads(0)
    sentinel = g["dw_gate"].clone()
    layer.backward(x0, out, torch.empty((0, cfg.d), dtype=torch.bfloat16, device="cuda"), ALPHA, BETA, grads=g)
    torch.cuda.synchronize()
    assert torch.equal(g["dw_gate"], sentinel)


@pytest.mark.parametrize("name", ["tiny", "ragged", "wide", "split", "odd", "skew"])
def test_backward_with_saved_preactivations(name):
    """Training mode: the forward also writes the gate/up pre-activations z (bf16, packed
    order) and the backward takes the SwiGLU derivative from them instead of recomputing
    them. y is bit-identical to the forward without z; z matches x W_g^T and x W_u^T of the
    oracle's fp64 products to bf16 rounding; the gradients match the oracle like the
    recomputing backward does."""
    from token_choice_routing_b200.layer import bf16_tensor
    from token_choice_routing_b200 import binding as B
    cfg = CASES[name]
    inp = I.make_inputs(cfg)
    layer, x, tnb = H.make_layer(inp)
    plain = layer.forward(x, tnb, layer.alloc(cfg.T))
    out = layer.forward(x, tnb, layer.alloc(cfg.T, save_preact=True))
    torch.cuda.synchronize()
    assert B.get_device_status(out["workspace"]) == B.OK
    assert torch.equal(plain["y"], out["y"]) and torch.equal(plain["h"][: int(out["offsets"][-1])],
                                                            out["h"][: int(out["offsets"][-1])])
    # z of the routed rows against the oracle's products, in the packed column order
    R = int(out["offsets"][-1])
    perm = out["perm_tok"][:R].cpu().numpy()
    offs = out["offsets"].cpu().numpy()
    xf = H.f64(inp.x)
    wg, wu = H.f64(inp.w_gate), H.f64(inp.w_up)
    z = f64(out["z"][:R])
    F = cfg.F
    zref = np.zeros((R, 2 * F))
    for e in range(cfg.N):
        rows = np.arange(offs[e], offs[e + 1])
        if rows.size == 0:
            continue
        a = xf[perm[rows]] @ wg[e].T
        b = xf[perm[rows]] @ wu[e].T
        for p in range(F // 64):
            zref[rows, p * 128:p * 128 + 64] = a[:, p * 64:(p + 1) * 64]
            zref[rows, p * 128 + 64:p * 128 + 128] = b[:, p * 64:(p + 1) * 64]
    assert rel(z, zref) < 5e-3
    dy_bits = I.upstream_grad(cfg)
    g = layer.backward(x, out, bf16_tensor(dy_bits, "cuda"), ALPHA, BETA)
    torch.cuda.synchronize()
    assert B.get_device_status(g["workspace"]) == B.OK
    ref = oracle_backward(inp, out, dy_bits, ALPHA, BETA)
    check_all(inp, out, g, ref, out["counts"].cpu().numpy())
    # and close to the recomputing backward (z there is fp32 in TMEM, here bf16)
    g2 = layer.backward(x, plain, bf16_tensor(dy_bits, "cuda"), ALPHA, BETA)
    torch.cuda.synchronize()
    for k in ("dx", "dw_gate", "dw_up", "dws_gate"):
        assert rel(f64(g[k]), f64(g2[k])) < 5e-3, k
