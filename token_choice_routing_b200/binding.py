"""ctypes binding of libmoe_null.so (include/moe_null.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. Tensors are torch CUDA tensors; their data pointers and the current
CUDA stream are passed through the C ABI. There is no CPU fallback: if the
library is missing this module raises on import.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_null.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE_BOUNDS = 0, -1, -2, -3, -4, -5


class MoEError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {code} ({status_string(code)})")
        self.code = code


class Dims(C.Structure):
    _fields_ = [("T", C.c_int32), ("d", C.c_int32), ("N", C.c_int32), ("M", C.c_int32),
                ("K", C.c_int32), ("F", C.c_int32), ("F_shared", C.c_int32), ("flags", C.c_uint32),
                ("C", C.c_int32), ("V", C.c_int32)]


class Weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("w_router", "router_bias", "gate_up", "w_down",
                                           "shared_gate_up", "shared_down", "const_vectors", "router_split")]


OUTPUT_FIELDS = ("logits", "topk_idx", "topk_gate", "n_real", "counts", "offsets", "perm_tok",
                 "slot_row", "xs", "h", "h_shared", "ys", "shared_out", "y", "counts_ext", "P",
                 "losses", "z", "z_shared")


class Outputs(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in OUTPUT_FIELDS]


SAVED_FIELDS = ("x", "logits", "topk_idx", "topk_gate", "offsets", "slot_row", "xs", "h", "h_shared", "ys",
                "counts_ext")


class Saved(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in SAVED_FIELDS] + [("t_total", C.c_int64), ("z", C.c_void_p),
                                                          ("z_shared", C.c_void_p)]


GRAD_FIELDS = ("dx", "dw_router", "dbias", "dtok_null_bias", "dw_gate", "dw_up", "dw_down", "dws_gate",
               "dws_up", "dws_down", "dconst")


class Grads(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in GRAD_FIELDS]


def _load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"CUDA library not built: {LIB_PATH} is missing "
                          "(run python -m token_choice_routing_b200.build)")
    lib = C.CDLL(LIB_PATH)
    vp, i32, sz = C.c_void_p, C.c_int, C.c_size_t
    pd = C.POINTER(Dims)
    sig = {
        "moe_abi_version": (i32, []),
        "moe_status_string": (C.c_char_p, [i32]),
        "moe_check_dims": (i32, [pd]),
        "moe_workspace_bytes": (sz, [pd]),
        "moe_packed_gate_up_elems": (sz, [pd, i32]),
        "moe_pack_gate_up": (i32, [pd, vp, vp, vp, vp, vp, vp, vp]),
        "moe_router_split_elems": (sz, [pd]),
        "moe_prepare_router": (i32, [pd, vp, vp, vp]),
        "moe_route": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_route_prepared": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_dispatch": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_expert_ffn": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_expert_gate_up": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_expert_gate_up_gather": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_expert_down": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_combine": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_combine_inplace": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_expert_down_combine": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_expert_gate_up_rows": (i32, [pd, C.c_int64, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_expert_down_rows": (i32, [pd, C.c_int64, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_aux_sums_count": (sz, [pd]),
        "moe_aux_sums": (i32, [pd, vp, vp, vp]),
        "moe_aux_sums_accumulate": (i32, [pd, vp, vp, vp]),
        "moe_aux_finalize": (i32, [pd, vp, vp, vp, vp, vp]),
        "moe_aux": (i32, [pd, vp, vp, vp, vp, vp]),
        "moe_forward": (i32, [pd, C.POINTER(Weights), vp, vp, C.POINTER(Outputs), vp, vp]),
        "moe_get_device_status": (i32, [vp, vp]),
        "moe_clear_device_status": (i32, [vp, vp]),
        "moe_selftest_bounded_wait": (i32, [vp, C.c_uint64, vp]),
        "moe_route_noalloc": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_route_noalloc_device_status": (i32, [vp]),
        "moe_route_noalloc_selftest_bounded_wait": (i32, [C.c_uint64, vp]),
        "moe_backward_workspace_bytes": (sz, [pd]),
        "moe_combine_backward": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_router_backward": (i32, [pd, vp, vp, vp, vp, vp, C.c_int64, C.c_float, C.c_float, vp, vp, vp, vp]),
        "moe_router_weight_grad": (i32, [pd, vp, vp, vp, vp, vp]),
        "moe_expert_ffn_backward": (i32, [pd, C.POINTER(Weights), C.POINTER(Saved), vp, vp, vp, vp,
                                          C.POINTER(Grads), vp, vp]),
        "moe_input_grad": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_expert_swiglu_backward": (i32, [pd, vp, vp, vp, vp, vp, vp, vp]),
        "moe_expert_swiglu_backward_saved": (i32, [pd, vp, vp, vp, vp, vp]),
        "moe_expert_dgrad_down": (i32, [pd, vp, vp, vp, vp, vp, vp, vp]),
        "moe_expert_wgrad_down": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_expert_dgrad_gate_up": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_expert_wgrad_gate_up": (i32, [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_backward": (i32, [pd, C.POINTER(Weights), C.POINTER(Saved), vp, C.c_float, C.c_float,
                               C.POINTER(Grads), vp, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    if lib.moe_abi_version() != 6:
        raise ImportError("libmoe_null ABI version mismatch")
    return lib


LIB = _load()


def status_string(code: int) -> str:
    return LIB.moe_status_string(int(code)).decode()


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return C.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _check(fn: str, code: int):
    if code != OK:
        raise MoEError(fn, code)


# moe_dims_t.flags: router product on the fp32 CUDA cores instead of the tensor cores;
# expert GEMMs on CTA pairs instead of single-CTA tiles; the backward's weight gradients on
# CTA pairs
FLAG_ROUTER_FP32_CORES = 1
FLAG_FFN_CTA_PAIR = 2
FLAG_WGRAD_CTA_PAIR = 4


def dims(T, d, N, M, K, F, F_shared, flags=0, C=0, V=0) -> Dims:
    return Dims(int(T), int(d), int(N), int(M), int(K), int(F), int(F_shared), int(flags), int(C), int(V))


def check_dims(dm: Dims) -> int:
    return LIB.moe_check_dims(C.byref(dm))


def workspace_bytes(dm: Dims) -> int:
    return int(LIB.moe_workspace_bytes(C.byref(dm)))


def aux_sums_count(dm: Dims) -> int:
    return int(LIB.moe_aux_sums_count(C.byref(dm)))


def packed_gate_up_elems(dm: Dims, shared: bool) -> int:
    return int(LIB.moe_packed_gate_up_elems(C.byref(dm), 1 if shared else 0))


def pack_gate_up(dm, w_gate, w_up, ws_gate, ws_up, gate_up, shared_gate_up, stream=None):
    _check("moe_pack_gate_up", LIB.moe_pack_gate_up(C.byref(dm), _p(w_gate), _p(w_up), _p(ws_gate),
                                                     _p(ws_up), _p(gate_up), _p(shared_gate_up),
                                                     _stream(stream)))


def router_split_elems(dm: Dims) -> int:
    return int(LIB.moe_router_split_elems(C.byref(dm)))


def prepare_router(dm, w_router, router_split, stream=None):
    _check("moe_prepare_router", LIB.moe_prepare_router(C.byref(dm), _p(w_router), _p(router_split),
                                                         _stream(stream)))


def route(dm, x, w_router, bias, tok_null_bias, logits, topk_idx, topk_gate, n_real, ws, stream=None):
    _check("moe_route", LIB.moe_route(C.byref(dm), _p(x), _p(w_router), _p(bias), _p(tok_null_bias),
                                      _p(logits), _p(topk_idx), _p(topk_gate), _p(n_real), _p(ws),
                                      _stream(stream)))


def route_prepared(dm, x, router_split, bias, tok_null_bias, logits, topk_idx, topk_gate, n_real, ws, stream=None):
    _check("moe_route_prepared",
           LIB.moe_route_prepared(C.byref(dm), _p(x), _p(router_split), _p(bias), _p(tok_null_bias), _p(logits),
                                  _p(topk_idx), _p(topk_gate), _p(n_real), _p(ws), _stream(stream)))


def dispatch(dm, x, topk_idx, ws, counts, offsets, perm_tok, slot_row, xs, stream=None):
    _check("moe_dispatch", LIB.moe_dispatch(C.byref(dm), _p(x), _p(topk_idx), _p(ws), _p(counts),
                                            _p(offsets), _p(perm_tok), _p(slot_row), _p(xs),
                                            _stream(stream)))


def expert_ffn(dm, xs, x, offsets, gate_up, w_down, shared_gate_up, shared_down, h, h_shared, ys,
               shared_out, ws, stream=None):
    _check("moe_expert_ffn", LIB.moe_expert_ffn(C.byref(dm), _p(xs), _p(x), _p(offsets), _p(gate_up),
                                                _p(w_down), _p(shared_gate_up), _p(shared_down), _p(h),
                                                _p(h_shared), _p(ys), _p(shared_out), _p(ws),
                                                _stream(stream)))


def expert_gate_up(dm, xs, x, offsets, gate_up, shared_gate_up, h, h_shared, ws, stream=None):
    _check("moe_expert_gate_up", LIB.moe_expert_gate_up(C.byref(dm), _p(xs), _p(x), _p(offsets), _p(gate_up),
                                                        _p(shared_gate_up), _p(h), _p(h_shared), _p(ws),
                                                        _stream(stream)))


def expert_gate_up_gather(dm, x, perm_tok, offsets, gate_up, shared_gate_up, h, h_shared, ws, stream=None):
    _check("moe_expert_gate_up_gather",
           LIB.moe_expert_gate_up_gather(C.byref(dm), _p(x), _p(perm_tok), _p(offsets), _p(gate_up),
                                         _p(shared_gate_up), _p(h), _p(h_shared), _p(ws), _stream(stream)))


def expert_down(dm, offsets, h, h_shared, w_down, shared_down, ys, shared_out, ws, stream=None):
    _check("moe_expert_down", LIB.moe_expert_down(C.byref(dm), _p(offsets), _p(h), _p(h_shared), _p(w_down),
                                                  _p(shared_down), _p(ys), _p(shared_out), _p(ws),
                                                  _stream(stream)))


def expert_gate_up_rows(dm, rows_cap, xs, x, offsets, gate_up, shared_gate_up, h, h_shared, ws, stream=None):
    """Gate/up grouped GEMM of an expert shard over rows_cap received rows (expert parallelism)."""
    _check("moe_expert_gate_up_rows",
           LIB.moe_expert_gate_up_rows(C.byref(dm), int(rows_cap), _p(xs), _p(x), _p(offsets), _p(gate_up),
                                       _p(shared_gate_up), _p(h), _p(h_shared), _p(ws), _stream(stream)))


def expert_down_rows(dm, rows_cap, offsets, h, h_shared, w_down, shared_down, ys, shared_out, ws, stream=None):
    """Down grouped GEMM of an expert shard over rows_cap received rows (expert parallelism)."""
    _check("moe_expert_down_rows",
           LIB.moe_expert_down_rows(C.byref(dm), int(rows_cap), _p(offsets), _p(h), _p(h_shared), _p(w_down),
                                    _p(shared_down), _p(ys), _p(shared_out), _p(ws), _stream(stream)))


def expert_down_combine(dm, offsets, h, h_shared, w_down, shared_down, ys, topk_gate, slot_row, y, ws,
                        stream=None, topk_idx=None, x=None, const_vectors=None):
    """Down GEMM with the combine in its shared-expert tiles (topk_idx, x and const_vectors
    are needed only with MoE++ copy/constant experts)."""
    _check("moe_expert_down_combine",
           LIB.moe_expert_down_combine(C.byref(dm), _p(offsets), _p(h), _p(h_shared), _p(w_down), _p(shared_down),
                                       _p(ys), _p(topk_gate), _p(slot_row), _p(topk_idx), _p(x),
                                       _p(const_vectors), _p(y), _p(ws), _stream(stream)))


def combine(dm, ys, shared_out, topk_gate, slot_row, y, stream=None, topk_idx=None, x=None,
            const_vectors=None):
    """topk_idx, x and const_vectors are needed only with MoE++ copy/constant experts."""
    _check("moe_combine", LIB.moe_combine(C.byref(dm), _p(ys), _p(shared_out), _p(topk_gate), _p(slot_row),
                                          _p(topk_idx), _p(x), _p(const_vectors), _p(y), _stream(stream)))


def combine_inplace(dm, ys, topk_gate, slot_row, y, ws, stream=None, topk_idx=None, x=None, const_vectors=None):
    """y holds the shared expert's output; adds the routed rows of the tokens the route listed in ws."""
    _check("moe_combine_inplace",
           LIB.moe_combine_inplace(C.byref(dm), _p(ys), _p(topk_gate), _p(slot_row), _p(topk_idx), _p(x),
                                   _p(const_vectors), _p(y), _p(ws), _stream(stream)))


def aux(dm, ws, counts_ext, P, losses, stream=None):
    _check("moe_aux", LIB.moe_aux(C.byref(dm), _p(ws), _p(counts_ext), _p(P), _p(losses), _stream(stream)))


def aux_sums(dm, ws, sums, stream=None):
    _check("moe_aux_sums", LIB.moe_aux_sums(C.byref(dm), _p(ws), _p(sums), _stream(stream)))


def aux_sums_accumulate(dm, ws, sums, stream=None):
    _check("moe_aux_sums_accumulate", LIB.moe_aux_sums_accumulate(C.byref(dm), _p(ws), _p(sums), _stream(stream)))


def aux_finalize(dm, sums, counts_ext, P, losses, stream=None):
    _check("moe_aux_finalize", LIB.moe_aux_finalize(C.byref(dm), _p(sums), _p(counts_ext), _p(P),
                                                    _p(losses), _stream(stream)))


def forward(dm, weights: Weights, x, tok_null_bias, outputs: Outputs, ws, stream=None):
    _check("moe_forward", LIB.moe_forward(C.byref(dm), C.byref(weights), _p(x), _p(tok_null_bias),
                                          C.byref(outputs), _p(ws), _stream(stream)))


def get_device_status(ws, stream=None) -> int:
    return LIB.moe_get_device_status(_p(ws), _stream(stream))


def clear_device_status(ws, stream=None):
    _check("moe_clear_device_status", LIB.moe_clear_device_status(_p(ws), _stream(stream)))


def selftest_bounded_wait(ws, limit_ns: int, stream=None):
    _check("moe_selftest_bounded_wait", LIB.moe_selftest_bounded_wait(_p(ws), int(limit_ns), _stream(stream)))


# ------------------------------------------------------------------------------ backward


def backward_workspace_bytes(dm: Dims) -> int:
    return int(LIB.moe_backward_workspace_bytes(C.byref(dm)))


def combine_backward(dm, dy, ys, topk_gate, slot_row, dys, dg, bws, stream=None, topk_idx=None, x=None,
                     const_vectors=None):
    _check("moe_combine_backward",
           LIB.moe_combine_backward(C.byref(dm), _p(dy), _p(ys), _p(topk_gate), _p(slot_row), _p(topk_idx), _p(x),
                                    _p(const_vectors), _p(dys), _p(dg), _p(bws), _stream(stream)))


def router_backward(dm, logits, topk_idx, topk_gate, dg, counts_ext, t_total, alpha, beta, ds, bws,
                    dtok_null_bias=None, stream=None):
    _check("moe_router_backward",
           LIB.moe_router_backward(C.byref(dm), _p(logits), _p(topk_idx), _p(topk_gate), _p(dg), _p(counts_ext),
                                   int(t_total), float(alpha), float(beta), _p(ds), _p(dtok_null_bias), _p(bws),
                                   _stream(stream)))


def router_weight_grad(dm, x, dw_router, dbias, bws, stream=None):
    _check("moe_router_weight_grad",
           LIB.moe_router_weight_grad(C.byref(dm), _p(x), _p(dw_router), _p(dbias), _p(bws), _stream(stream)))


def expert_ffn_backward(dm, weights: Weights, saved: Saved, dys, dy, dxs, dx_shared, grads: Grads, bws,
                        stream=None):
    _check("moe_expert_ffn_backward",
           LIB.moe_expert_ffn_backward(C.byref(dm), C.byref(weights), C.byref(saved), _p(dys), _p(dy), _p(dxs),
                                       _p(dx_shared), C.byref(grads), _p(bws), _stream(stream)))


def input_grad(dm, dx_shared, dxs, slot_row, topk_idx, topk_gate, dy, dx, bws, stream=None):
    _check("moe_input_grad",
           LIB.moe_input_grad(C.byref(dm), _p(dx_shared), _p(dxs), _p(slot_row), _p(topk_idx), _p(topk_gate),
                              _p(dy), _p(dx), _p(bws), _stream(stream)))


def backward(dm, weights: Weights, saved: Saved, dy, alpha, beta, grads: Grads, bws, stream=None):
    _check("moe_backward", LIB.moe_backward(C.byref(dm), C.byref(weights), C.byref(saved), _p(dy), float(alpha),
                                            float(beta), C.byref(grads), _p(bws), _stream(stream)))


def expert_swiglu_backward(dm, xs, x, offsets, gate_up, shared_gate_up, bws, stream=None):
    _check("moe_expert_swiglu_backward",
           LIB.moe_expert_swiglu_backward(C.byref(dm), _p(xs), _p(x), _p(offsets), _p(gate_up), _p(shared_gate_up),
                                          _p(bws), _stream(stream)))


def expert_dgrad_down(dm, offsets, dys, dy, w_down, shared_down, bws, stream=None):
    _check("moe_expert_dgrad_down", LIB.moe_expert_dgrad_down(C.byref(dm), _p(offsets), _p(dys), _p(dy),
                                                              _p(w_down), _p(shared_down), _p(bws),
                                                              _stream(stream)))


def expert_wgrad_down(dm, offsets, dys, dy, h, h_shared, dw_down, dws_down, bws, stream=None):
    _check("moe_expert_wgrad_down", LIB.moe_expert_wgrad_down(C.byref(dm), _p(offsets), _p(dys), _p(dy), _p(h),
                                                              _p(h_shared), _p(dw_down), _p(dws_down), _p(bws),
                                                              _stream(stream)))


def expert_dgrad_gate_up(dm, offsets, gate_up, shared_gate_up, w_router, dxs, dx_shared, bws, stream=None):
    """w_router (or None): add the router's input gradient ds W_r to dx_shared."""
    _check("moe_expert_dgrad_gate_up",
           LIB.moe_expert_dgrad_gate_up(C.byref(dm), _p(offsets), _p(gate_up), _p(shared_gate_up), _p(w_router),
                                        _p(dxs), _p(dx_shared), _p(bws), _stream(stream)))


def expert_wgrad_gate_up(dm, offsets, xs, x, dw_gate, dw_up, dws_gate, dws_up, bws, stream=None):
    _check("moe_expert_wgrad_gate_up",
           LIB.moe_expert_wgrad_gate_up(C.byref(dm), _p(offsets), _p(xs), _p(x), _p(dw_gate), _p(dw_up),
                                        _p(dws_gate), _p(dws_up), _p(bws), _stream(stream)))


def expert_swiglu_backward_saved(dm, offsets, z, z_shared, bws, stream=None):
    _check("moe_expert_swiglu_backward_saved",
           LIB.moe_expert_swiglu_backward_saved(C.byref(dm), _p(offsets), _p(z), _p(z_shared), _p(bws),
                                                _stream(stream)))
