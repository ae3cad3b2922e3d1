"""moe_route_noalloc: the routing entry point that takes no workspace.

It exists for callers that cannot allocate device memory (plugin-style
interfaces that receive only input and output buffers, hot paths that must
not call cudaMalloc). It must return exactly what moe_route returns for the
same inputs. Two calls in a row on different inputs check that the shared,
persistent scratch array does not leak one call's state into the next.
This file is collected last so that a failure here stops a -x run only after
every other test has run.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from token_choice_routing_b200 import inputs as I

pytestmark = pytest.mark.gpu

GATE_REL = 1e-6  # the gate tolerance of the other routing tests


def _fn():
    from token_choice_routing_b200 import binding as B
    f = B.LIB.moe_route_noalloc
    vp = C.c_void_p
    f.restype = C.c_int
    f.argtypes = [C.POINTER(B.Dims), vp, vp, vp, vp, vp, vp, vp, vp, vp]
    return B, f


def _inputs(cfg, null_bias=None):
    from token_choice_routing_b200.layer import bf16_tensor
    inp = I.make_inputs(cfg, weights=False, null_bias=null_bias)
    dev = "cuda"
    x = bf16_tensor(inp.x, dev)
    w = torch.from_numpy(inp.w_router).to(dev)
    b = torch.from_numpy(inp.bias).to(dev)
    tnb = None if inp.tok_null_bias is None else torch.from_numpy(inp.tok_null_bias).to(dev)
    return x, w, b, tnb


def _outputs(cfg):
    T, K, N = cfg.T, cfg.K, cfg.N
    return dict(logits=torch.empty((T, N + 1), dtype=torch.float32, device="cuda"),
                idx=torch.empty((T, K), dtype=torch.int32, device="cuda"),
                gate=torch.empty((T, K), dtype=torch.float32, device="cuda"),
                n_real=torch.empty((T,), dtype=torch.int32, device="cuda"))


def _ref(B, cfg, x, w, b, tnb):
    dm = B.dims(cfg.T, cfg.d, cfg.N, cfg.M, cfg.K, cfg.F, cfg.F_shared)
    ws = torch.empty(B.workspace_bytes(dm), dtype=torch.uint8, device="cuda")
    o = _outputs(cfg)
    B.route(dm, x, w, b, tnb, o["logits"], o["idx"], o["gate"], o["n_real"], ws)
    return o


def _noalloc(B, f, cfg, x, w, b, tnb):
    dm = B.dims(cfg.T, cfg.d, cfg.N, cfg.M, cfg.K, cfg.F, cfg.F_shared)
    o = _outputs(cfg)
    p = lambda t: None if t is None else C.c_void_p(t.data_ptr())
    s = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = f(C.byref(dm), p(x), p(w), p(b), p(tnb), p(o["logits"]), p(o["idx"]), p(o["gate"]), p(o["n_real"]), s)
    assert rc == B.OK, B.status_string(rc)
    return o


def _same(o, r):
    torch.cuda.synchronize()
    assert torch.equal(o["idx"], r["idx"])
    assert torch.equal(o["n_real"], r["n_real"])
    assert torch.equal(o["logits"], r["logits"])
    np.testing.assert_allclose(o["gate"].cpu().numpy(), r["gate"].cpu().numpy(), rtol=GATE_REL, atol=1e-7)


@pytest.mark.parametrize("first,second", [("tiny", "qwen3_0p6b"), ("qwen3_1p7b", "tiny")])
def test_noalloc_route_matches_route_on_two_calls_in_a_row(first, second):
    B, f = _fn()
    c1 = I.CONFIGS[first]
    c2 = I.CONFIGS[second]
    a1 = _inputs(c1)
    a2 = _inputs(c2)
    r1 = _ref(B, c1, *a1)
    r2 = _ref(B, c2, *a2)
    o1 = _noalloc(B, f, c1, *a1)
    o2 = _noalloc(B, f, c2, *a2)
    _same(o1, r1)
    _same(o2, r2)


def test_noalloc_route_same_shape_twice_and_ragged():
    B, f = _fn()
    cfg = I.small_config("noalloc_ragged", T=333, d=384, N=13, F=192, F_shared=64, K=5, M=9, config_id=920)
    a = _inputs(cfg)
    b = _inputs(cfg, null_bias=-0.7)
    ra, rb = _ref(B, cfg, *a), _ref(B, cfg, *b)
    oa = _noalloc(B, f, cfg, *a)
    ob = _noalloc(B, f, cfg, *b)
    _same(oa, ra)
    _same(ob, rb)


def test_noalloc_route_rejects_shapes_beyond_its_scratch():
    B, f = _fn()
    dm = B.dims(1 << 20, 1024, 64, 64, 8, 768, 768)  # needs ~41 MB of scratch
    assert B.workspace_bytes(dm) > (8 << 20)
    nul = C.c_void_p(0)
    d = C.c_void_p(16)  # never dereferenced: the size check comes first
    rc = f(C.byref(dm), d, d, None, None, None, d, d, d, nul)
    assert rc == B.ERR_UNSUPPORTED
