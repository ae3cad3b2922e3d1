"""moe_route_noalloc: the routing entry point that takes no workspace.

It exists for callers that cannot allocate device memory (plugin-style
interfaces that receive only input and output buffers, hot paths that must
not call cudaMalloc). It must return exactly what moe_route returns for the
same inputs. Two calls in a row on different inputs check that the shared,
persistent scratch array does not leak one call's state into the next; the
router paths that lay out that scratch differently (the fp32 CUDA-core router,
a MoE++ pool with copy and constant experts) alternate with the default one.
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
FP32_CORES = 1   # MOE_FLAG_ROUTER_FP32_CORES


def _B():
    from token_choice_routing_b200 import binding as B
    return B


def _dims(B, cfg, flags=0):
    return B.dims(cfg.T, cfg.d, cfg.N, cfg.M, cfg.K, cfg.F, cfg.F_shared, flags, cfg.C, cfg.V)


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
    T, K = cfg.T, cfg.K
    return dict(logits=torch.empty((T, cfg.router_rows), dtype=torch.float32, device="cuda"),
                idx=torch.empty((T, K), dtype=torch.int32, device="cuda"),
                gate=torch.empty((T, K), dtype=torch.float32, device="cuda"),
                n_real=torch.empty((T,), dtype=torch.int32, device="cuda"))


def _ref(B, cfg, x, w, b, tnb, flags=0):
    dm = _dims(B, cfg, flags)
    ws = torch.empty(B.workspace_bytes(dm), dtype=torch.uint8, device="cuda")
    o = _outputs(cfg)
    B.route(dm, x, w, b, tnb, o["logits"], o["idx"], o["gate"], o["n_real"], ws)
    return o


def _noalloc(B, cfg, x, w, b, tnb, flags=0):
    dm = _dims(B, cfg, flags)
    o = _outputs(cfg)
    p = lambda t: None if t is None else C.c_void_p(t.data_ptr())
    s = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = B.LIB.moe_route_noalloc(C.byref(dm), p(x), p(w), p(b), p(tnb), p(o["logits"]), p(o["idx"]),
                                 p(o["gate"]), p(o["n_real"]), s)
    assert rc == B.OK, B.status_string(rc)
    return o


def _status(B):
    return B.LIB.moe_route_noalloc_device_status(C.c_void_p(torch.cuda.current_stream().cuda_stream))


def _same(o, r):
    torch.cuda.synchronize()
    assert torch.equal(o["idx"], r["idx"])
    assert torch.equal(o["n_real"], r["n_real"])
    assert torch.equal(o["logits"], r["logits"])
    np.testing.assert_allclose(o["gate"].cpu().numpy(), r["gate"].cpu().numpy(), rtol=GATE_REL, atol=1e-7)


@pytest.mark.parametrize("first,second", [("tiny", "qwen3_0p6b"), ("qwen3_1p7b", "tiny")])
def test_noalloc_route_matches_route_on_two_calls_in_a_row(first, second):
    B = _B()
    c1 = I.CONFIGS[first]
    c2 = I.CONFIGS[second]
    a1 = _inputs(c1)
    a2 = _inputs(c2)
    r1 = _ref(B, c1, *a1)
    r2 = _ref(B, c2, *a2)
    o1 = _noalloc(B, c1, *a1)
    o2 = _noalloc(B, c2, *a2)
    _same(o1, r1)
    _same(o2, r2)
    assert _status(B) == B.OK


def test_noalloc_route_same_shape_twice_and_ragged():
    B = _B()
    cfg = I.small_config("noalloc_ragged", T=333, d=384, N=13, F=192, F_shared=64, K=5, M=9, config_id=920)
    a = _inputs(cfg)
    b = _inputs(cfg, null_bias=-0.7)
    ra, rb = _ref(B, cfg, *a), _ref(B, cfg, *b)
    oa = _noalloc(B, cfg, *a)
    ob = _noalloc(B, cfg, *b)
    _same(oa, ra)
    _same(ob, rb)


# The fp32 CUDA-core router (64-token blocks, its own header clear) and a MoE++ pool (an
# 80-row router tile, copy/constant counts in the histogram) place their data in the
# shared array differently from the default path: each runs between two default-path
# calls of another shape, so stale scratch of one layout would show in the next call.
_LAYOUTS = [
    ("fp32_cores", I.small_config("noalloc_f32", T=777, d=512, N=24, F=128, F_shared=64, K=6, M=18,
                                  config_id=921), FP32_CORES),
    ("moepp", I.small_config("noalloc_pp", T=611, d=256, N=16, F=128, F_shared=64, K=4, M=16, C=3, V=2,
                             config_id=922), 0),
]


@pytest.mark.parametrize("name,cfg,flags", _LAYOUTS, ids=[l[0] for l in _LAYOUTS])
def test_noalloc_route_other_scratch_layouts_alternate_with_the_default(name, cfg, flags):
    B = _B()
    dflt = I.CONFIGS["qwen3_0p6b"]
    ad, a = _inputs(dflt), _inputs(cfg)
    rd, r = _ref(B, dflt, *ad), _ref(B, cfg, *a, flags=flags)
    o0 = _noalloc(B, dflt, *ad)
    o1 = _noalloc(B, cfg, *a, flags=flags)
    o2 = _noalloc(B, dflt, *ad)
    o3 = _noalloc(B, cfg, *a, flags=flags)
    for o, e in ((o0, rd), (o1, r), (o2, rd), (o3, r)):
        _same(o, e)
    assert _status(B) == B.OK


def test_noalloc_device_status_reports_a_recorded_timeout_and_the_next_call_clears_it():
    """A device-side failure recorded in the entry point's own scratch is visible to the
    caller: the self-test wait runs out (no GPU fault; the context stays usable), the status
    reader returns MOE_ERR_TIMEOUT, and the next routing call starts from a clean word."""
    B = _B()
    cfg = I.CONFIGS["tiny"]
    a = _inputs(cfg)
    r = _ref(B, cfg, *a)
    _same(_noalloc(B, cfg, *a), r)
    assert _status(B) == B.OK
    s = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert B.LIB.moe_route_noalloc_selftest_bounded_wait(100000, s) == B.OK
    assert _status(B) == B.ERR_TIMEOUT
    _same(_noalloc(B, cfg, *a), r)
    assert _status(B) == B.OK


def test_noalloc_route_rejects_shapes_beyond_its_scratch():
    B = _B()
    dm = B.dims(1 << 20, 1024, 64, 64, 8, 768, 768)  # needs ~41 MB of scratch
    assert B.workspace_bytes(dm) > (8 << 20)
    nul = C.c_void_p(0)
    d = C.c_void_p(16)  # never dereferenced: the size check comes first
    rc = B.LIB.moe_route_noalloc(C.byref(dm), d, d, None, None, None, d, d, d, nul)
    assert rc == B.ERR_UNSUPPORTED
