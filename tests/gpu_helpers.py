"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare with the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from token_choice_routing_b200 import inputs as I

# Tolerances for floating-point outputs of the layer.
Y_REL_FRO = 1e-2        # ||y - y_ref||_F / ||y_ref||_F
Y_MAX_REL = 5e-2        # max|y - y_ref| / max|y_ref|
LOSS_REL = 1e-5         # L_bal, L_z
GATE_REL = 1e-6         # gates from identical fp32 logits
P_REL = 1e-5


def f64(bits):
    return I.bf16_to_f32(bits).astype(np.float64)


def t2bits(t: torch.Tensor) -> np.ndarray:
    """torch bf16 tensor -> host uint16 bits."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().float().numpy().astype(np.float64)


# Both router paths of the library: tensor cores (default) and fp32 CUDA cores.
ROUTERS = ("tensor", "fp32_cores")


# Both expert GEMM variants: single-CTA tiles (default) and CTA pairs.
FFNS = ("single", "pair")


def make_layer(inp, device="cuda", router="tensor", ffn="single"):
    from token_choice_routing_b200.layer import MoENullLayer, bf16_tensor
    layer = MoENullLayer.from_inputs(inp, device, router=router, ffn=ffn)
    x = bf16_tensor(inp.x, device)
    tnb = None if inp.tok_null_bias is None else torch.from_numpy(inp.tok_null_bias).to(device)
    return layer, x, tnb


def run_forward(inp, device="cuda", router="tensor", ffn="single", xs=True, combine="separate"):
    """xs=False: no gathered copy of the routed rows; gate/up gathers rows of x.
    combine="separate" (the default here): the shared expert's output gets a buffer of its
    own (checked by the GEMM tests) and the combine reads it; "inplace": the down GEMM
    writes it into y and the combine adds the routed rows there; "fused": the combine runs
    in the down GEMM's shared-expert tiles."""
    from token_choice_routing_b200 import binding as B
    layer, x, tnb = make_layer(inp, device, router, ffn)
    out = layer.forward(x, tnb, layer.alloc(inp.cfg.T, xs=xs, combine=combine))
    torch.cuda.synchronize()
    st = B.get_device_status(out["workspace"])
    assert st == B.OK, B.status_string(st)
    return layer, x, tnb, out


def logit_bound(inp):
    """Rigorous bound on |fp32 router logit - exact| for a length-d fp32 dot
    product evaluated by sequential FMAs plus bias additions:
    (d + 3) * 2^-24 * (sum_c |x_c w_jc| + |bias_j| + |offset|) per element."""
    x = np.abs(f64(inp.x))
    w = np.abs(inp.w_router.astype(np.float64))
    mag = x @ w.T + np.abs(inp.bias.astype(np.float64))[None, :]
    if inp.tok_null_bias is not None:
        mag[:, inp.cfg.N] += np.abs(inp.tok_null_bias.astype(np.float64))
    return (inp.cfg.d + 3) * 2.0 ** -24 * mag + 1e-30


def oracle_logits(inp):
    return O.router_logits(f64(inp.x), inp.w_router, inp.bias, inp.tok_null_bias, null_col=inp.cfg.N)


def check_routing(inp, out, full_gates=True):
    """Logits within the fp32 bound; top-K, n_real, gates from the GPU logits."""
    cfg = inp.cfg
    N, M, K = cfg.N, cfg.M, cfg.K
    s_gpu = out["logits"].cpu().numpy().astype(np.float64)
    s_ref = oracle_logits(inp)
    err = np.abs(s_gpu - s_ref)
    assert np.all(err <= logit_bound(inp)), float((err / logit_bound(inp)).max())
    r = O.route_pp(s_gpu, N, M, cfg.C, cfg.V, K)  # = O.route when C = V = 0
    idx = out["topk_idx"].cpu().numpy()
    assert np.array_equal(idx, r["idx"]), np.argwhere(idx != r["idx"])[:5]
    assert np.array_equal(out["n_real"].cpu().numpy(), r["n_real"])
    g = out["topk_gate"].cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(g, r["gates"], rtol=GATE_REL, atol=1e-7)
    return r


def check_dispatch(inp, out, r):
    N = inp.cfg.N
    counts, offsets, perm, slot_row = O.dispatch(r["idx"], N)
    assert np.array_equal(out["counts"].cpu().numpy(), counts)
    assert np.array_equal(out["offsets"].cpu().numpy(), offsets)
    R = int(offsets[-1])
    assert np.array_equal(out["perm_tok"][:R].cpu().numpy(), perm)
    assert np.array_equal(out["slot_row"].cpu().numpy(), slot_row)
    if out.get("xs") is not None:  # None: the forward gathered rows of x instead of copying them
        xs = t2bits(out["xs"][:R])
        assert np.array_equal(xs, inp.x[perm])
    return counts, offsets, perm, slot_row


def check_aux(inp, out, r):
    cfg = inp.cfg
    counts_ext, f, P, L_bal, L_z = O.aux_stats(r["idx"], r["p"], r["lse"], cfg.N, cfg.M)
    assert np.array_equal(out["counts_ext"].cpu().numpy(), counts_ext)
    np.testing.assert_allclose(out["P"].cpu().numpy(), P, rtol=P_REL, atol=1e-9)
    lb, lz = out["losses"].cpu().numpy().astype(np.float64)
    assert abs(lb - L_bal) <= LOSS_REL * abs(L_bal), (lb, L_bal)
    assert abs(lz - L_z) <= LOSS_REL * abs(L_z), (lz, L_z)


def expert_weights(inp):
    return ((f64(inp.w_gate), f64(inp.w_up), f64(inp.w_down)),
            (f64(inp.ws_gate), f64(inp.ws_up), f64(inp.ws_down)))


def check_y(y_gpu, y_ref):
    num = np.linalg.norm(y_gpu - y_ref)
    den = np.linalg.norm(y_ref)
    assert num <= Y_REL_FRO * den, (num / den)
    assert np.abs(y_gpu - y_ref).max() <= Y_MAX_REL * np.abs(y_ref).max()


def check_layer_output(inp, out, r, tokens=None):
    ex, sh = expert_weights(inp)
    x = f64(inp.x)
    c = inp.cfg
    if c.C + c.V > 0:
        cv = f64(inp.const_vectors) if c.V else None
        y_ref = O.layer_output_pp(x, r["idx"], r["gates"], c.N, c.M, c.C, c.V, ex, sh, cv, tokens=tokens)
    else:
        y_ref = O.layer_output(x, r["idx"], r["gates"], c.N, ex, sh, tokens=tokens)
    y_gpu = bf16_f64(out["y"][:inp.cfg.T])
    if tokens is not None:
        y_gpu = y_gpu[tokens]
    check_y(y_gpu, y_ref)
    return y_ref
