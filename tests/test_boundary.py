"""The C-ABI library: it loads, exports every entry point the header declares,
and rejects bad arguments on the host (no GPU needed for any call here)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_null.h")
LIB = os.path.join(ROOT, "token_choice_routing_b200", "libmoe_null.so")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from token_choice_routing_b200 import build
        build.build()
    from token_choice_routing_b200 import binding
    return binding


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_aux", "moe_forward",
                 "moe_workspace_bytes", "moe_get_device_status", "moe_aux_sums", "moe_aux_finalize"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    so = C.CDLL(LIB)
    for name in declared_functions():
        assert hasattr(so, name), name


def test_abi_version_and_status_strings(lib):
    assert lib.LIB.moe_abi_version() == 6
    for code in (0, -1, -2, -3, -4, -5, 7):
        assert isinstance(lib.status_string(code), str) and lib.status_string(code)


def good():
    from token_choice_routing_b200 import binding as B
    return B.dims(256, 128, 8, 8, 4, 64, 64)


def test_check_dims(lib):
    B = lib
    assert B.check_dims(good()) == B.OK
    bad_arg = [dict(T=-1), dict(K=0), dict(M=-1), dict(N=0), dict(K=17 + 0, N=8, M=8), dict(d=0), dict(F=0)]
    for kw in bad_arg:
        v = dict(T=256, d=128, N=8, M=8, K=4, F=64, F_shared=64)
        v.update(kw)
        assert B.check_dims(B.dims(**v)) == B.ERR_INVALID_ARG, kw
    unsupported = [dict(N=65, M=0, K=4), dict(K=17, N=64, M=64), dict(d=192), dict(d=16384), dict(F=96),
                   dict(F_shared=32), dict(T=1 << 29, K=8)]
    for kw in unsupported:
        v = dict(T=256, d=128, N=8, M=8, K=4, F=64, F_shared=64)
        v.update(kw)
        assert B.check_dims(B.dims(**v)) == B.ERR_UNSUPPORTED, kw
    # MoE++ copy/constant experts: at most 16 of them and 80 router rows, tensor-core router only
    ok = dict(T=256, d=128, N=8, M=8, K=4, F=64, F_shared=64)
    assert B.check_dims(B.dims(**ok, C=2, V=3)) == B.OK
    assert B.check_dims(B.dims(**dict(ok, N=64, M=0, K=4), C=10, V=5)) == B.OK  # 80 rows
    assert B.check_dims(B.dims(**dict(ok, N=64), C=10, V=6)) == B.ERR_UNSUPPORTED  # 81 rows
    assert B.check_dims(B.dims(**ok, C=9, V=8)) == B.ERR_UNSUPPORTED  # 17 > 16
    assert B.check_dims(B.dims(**ok, flags=B.FLAG_ROUTER_FP32_CORES, C=1)) == B.ERR_UNSUPPORTED
    assert B.check_dims(B.dims(**ok, C=-1)) == B.ERR_INVALID_ARG
    assert B.check_dims(B.dims(**dict(ok, M=0, K=9), C=0, V=0)) == B.ERR_INVALID_ARG  # K > N+M
    assert B.check_dims(B.dims(**dict(ok, M=0, K=9), C=1, V=0)) == B.OK  # K <= N+M+C+V
    dm = good()
    for f in (B.FLAG_ROUTER_FP32_CORES, B.FLAG_FFN_CTA_PAIR, B.FLAG_ROUTER_FP32_CORES | B.FLAG_FFN_CTA_PAIR,
              B.FLAG_WGRAD_CTA_PAIR, B.FLAG_FFN_CTA_PAIR | B.FLAG_WGRAD_CTA_PAIR):
        dm.flags = f
        assert B.check_dims(dm) == B.OK, f
    for f in (8, 16, 0x80000000, B.FLAG_ROUTER_FP32_CORES | 8):
        dm.flags = f
        assert B.check_dims(dm) == B.ERR_INVALID_ARG, f


def test_workspace_depends_on_router_path(lib):
    """The fp32 CUDA-core route keeps per-block statistics over 64-token blocks
    and a transposed fp32 W_r; the tensor-core route over 128-token blocks and
    a bf16 three-term split of W_r. Both layouts are sized by the library."""
    B = lib
    for T, d, N, K in ((1, 128, 1, 1), (16384, 1024, 64, 4), (131072, 2048, 64, 8), (777, 256, 15, 3)):
        tc = B.workspace_bytes(B.dims(T, d, N, 64, K, 64, 64))
        fp = B.workspace_bytes(B.dims(T, d, N, 64, K, 64, 64, B.FLAG_ROUTER_FP32_CORES))
        assert tc > 0 and fp > 0 and tc % 256 == 0 and fp % 256 == 0
        npw = (N + 1 + 15) // 16 * 16
        npad = 8 if N <= 8 else 16 if N <= 16 else 32 if N <= 32 else 64
        # the weight buffers alone differ by exactly this much (both 256-aligned regions)
        al = lambda v: (v + 255) // 256 * 256
        assert tc - al(2 * 3 * npw * d) >= 0 and fp - al(4 * d * (npad + 4)) >= 0


def test_workspace_and_sizes(lib):
    B = lib
    assert B.workspace_bytes(good()) > 0
    assert B.workspace_bytes(B.dims(-1, 128, 8, 8, 4, 64, 64)) == 0
    small = B.workspace_bytes(B.dims(1000, 1024, 64, 64, 4, 768, 768))
    big = B.workspace_bytes(B.dims(100000, 1024, 64, 64, 4, 768, 768))
    assert big > small and big % 256 == 0
    assert B.aux_sums_count(good()) == 8 + 5 + 9 + 2
    # with C + V = 5: five more slot counts and five more probability sums
    assert B.aux_sums_count(B.dims(256, 128, 8, 8, 4, 64, 64, C=2, V=3)) == 8 + 10 + 14 + 2
    assert B.packed_gate_up_elems(good(), False) == 8 * 2 * 64 * 128
    assert B.packed_gate_up_elems(good(), True) == 2 * 64 * 128


def test_host_side_rejections_touch_no_device(lib):
    B = lib
    L = B.LIB
    dm = good()
    nul = None
    # null pointers with valid dims -> INVALID_ARG before any CUDA call
    assert L.moe_route(C.byref(dm), nul, nul, nul, nul, nul, nul, nul, nul, nul, nul) == B.ERR_INVALID_ARG
    assert L.moe_dispatch(C.byref(dm), nul, nul, nul, nul, nul, nul, nul, nul, nul) == B.ERR_INVALID_ARG
    assert L.moe_combine(C.byref(dm), nul, nul, nul, nul, nul, nul, nul, nul, nul) == B.ERR_INVALID_ARG
    assert L.moe_combine_inplace(C.byref(dm), *([nul] * 9)) == B.ERR_INVALID_ARG
    # the in-place combine needs the route's workspace (its token list): a missing one is refused
    fake = C.c_void_p(16)
    assert L.moe_combine_inplace(C.byref(dm), fake, fake, fake, nul, nul, nul, fake, nul, nul) == B.ERR_INVALID_ARG
    assert L.moe_aux(C.byref(dm), nul, nul, nul, nul, nul) == B.ERR_INVALID_ARG
    assert L.moe_forward(C.byref(dm), nul, nul, nul, nul, nul, nul) == B.ERR_INVALID_ARG
    assert L.moe_get_device_status(nul, nul) == B.ERR_INVALID_ARG
    assert L.moe_selftest_bounded_wait(nul, 1000, nul) == B.ERR_INVALID_ARG
    # invalid dims are rejected first
    bad = B.dims(256, 100, 8, 8, 4, 64, 64)
    assert L.moe_route(C.byref(bad), nul, nul, nul, nul, nul, nul, nul, nul, nul, nul) == B.ERR_UNSUPPORTED
    assert L.moe_check_dims(None) == B.ERR_INVALID_ARG
    # T = 0 is a no-op
    zero = B.dims(0, 128, 8, 8, 4, 64, 64)
    assert L.moe_route(C.byref(zero), nul, nul, nul, nul, nul, nul, nul, nul, nul, nul) == B.OK


def test_backward_workspace_and_host_side_rejections(lib):
    B = lib
    L = B.LIB
    dm = good()
    T, d, K, F, Fs = 256, 128, 4, 64, 64
    bw = B.backward_workspace_bytes(dm)
    assert bw > 0 and bw % 256 == 0
    # holds at least the gate/up pre-activations and their gradients (routed and shared) and
    # the routed rows' upstream and input gradients (the shared expert's input gradient goes
    # straight into the caller's dx)
    assert bw >= 2 * (2 * (T * K * 2 * F + T * 2 * Fs)) + 2 * 2 * T * K * d
    assert B.backward_workspace_bytes(B.dims(-1, 128, 8, 8, 4, 64, 64)) == 0
    big = B.backward_workspace_bytes(B.dims(16384, 1024, 64, 64, 4, 768, 768))
    assert big > bw
    nul = None
    inv = B.ERR_INVALID_ARG
    assert L.moe_combine_backward(C.byref(dm), *([nul] * 11)) == inv
    assert L.moe_router_backward(C.byref(dm), nul, nul, nul, nul, nul, T, 0.02, 0.001, nul, nul, nul, nul) == inv
    assert L.moe_router_weight_grad(C.byref(dm), nul, nul, nul, nul, nul) == inv
    assert L.moe_expert_ffn_backward(C.byref(dm), nul, nul, nul, nul, nul, nul, nul, nul, nul) == inv
    assert L.moe_input_grad(C.byref(dm), *([nul] * 9)) == inv
    assert L.moe_expert_dgrad_down(C.byref(dm), *([nul] * 7)) == inv
    assert L.moe_expert_swiglu_backward(C.byref(dm), *([nul] * 7)) == inv
    assert L.moe_expert_swiglu_backward_saved(C.byref(dm), *([nul] * 5)) == inv
    assert L.moe_expert_wgrad_down(C.byref(dm), *([nul] * 9)) == inv
    assert L.moe_expert_dgrad_gate_up(C.byref(dm), *([nul] * 8)) == inv
    assert L.moe_expert_wgrad_gate_up(C.byref(dm), *([nul] * 9)) == inv
    assert L.moe_backward(C.byref(dm), nul, nul, nul, 0.02, 0.001, nul, nul, nul) == inv
    # a token total smaller than this call's tokens is never valid (pointers set to a dummy value)
    fake = C.c_void_p(256)
    assert L.moe_router_backward(C.byref(dm), fake, fake, fake, fake, fake, T - 1, 0.02, 0.001, fake, nul,
                                 fake, nul) == inv
    # invalid dims first; T = 0 is a no-op
    bad = B.dims(256, 100, 8, 8, 4, 64, 64)
    assert L.moe_backward(C.byref(bad), nul, nul, nul, 0.02, 0.001, nul, nul, nul) == B.ERR_UNSUPPORTED
    zero = B.dims(0, 128, 8, 8, 4, 64, 64)
    assert L.moe_backward(C.byref(zero), nul, nul, nul, 0.02, 0.001, nul, nul, nul) == B.OK


def test_struct_layouts_match_header(tmp_path, lib):
    """The binding's ctypes structures have the C header's field offsets and sizes (compiled
    with the host C compiler against include/moe_null.h)."""
    import shutil
    import subprocess
    B = lib
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    structs = {
        "moe_dims_t": (B.Dims, [f for f, _ in B.Dims._fields_]),
        "moe_weights_t": (B.Weights, [f for f, _ in B.Weights._fields_]),
        "moe_outputs_t": (B.Outputs, [f for f, _ in B.Outputs._fields_]),
        "moe_saved_t": (B.Saved, [f for f, _ in B.Saved._fields_]),
        "moe_grads_t": (B.Grads, [f for f, _ in B.Grads._fields_]),
    }
    src = ['#include <stdio.h>', '#include <stddef.h>', '#include "moe_null.h"', "int main(void) {"]
    for name, (_, fields) in structs.items():
        src.append(f'  printf("{name} sizeof %zu\\n", sizeof({name}));')
        for f in fields:
            src.append(f'  printf("{name} {f} %zu\\n", offsetof({name}, {f}));')
    src += ["  return 0;", "}"]
    c = tmp_path / "layout.c"
    c.write_text("\n".join(src) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {}
    for line in out:
        if line.strip():
            name, field, val = line.split()
            got[(name, field)] = int(val)
    for name, (cls, fields) in structs.items():
        assert got[(name, "sizeof")] == C.sizeof(cls), name
        for f in fields:
            assert got[(name, f)] == getattr(cls, f).offset, (name, f)
