"""A null-expert MoE layer object over the C ABI.

Holds the device weights (gate/up packed once by the library), allocates the
caller-owned buffers and workspace with torch, and runs the forward through
``moe_forward``. PyTorch is used for device memory and streams only.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Tuple

import numpy as np
import torch

from . import binding as B


def bf16_tensor(bits: np.ndarray, device) -> torch.Tensor:
    """uint16 bf16 bit array (host) -> torch.bfloat16 tensor on ``device``."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def chunk_bounds(T: int, chunk: int) -> List[Tuple[int, int]]:
    """Token ranges [a, b) of the host-buffer forward's chunks, none longer than ``chunk``.

    Nothing overlaps the first chunk's copy in or the last chunk's copy out, so the batch
    starts and ends with short chunks (chunk/8, chunk/4, chunk/2, ... and the same in reverse),
    and the tokens between them are split into equal chunks of at most ``chunk``. A batch too
    short for both ramps is split into equal chunks of at most chunk/8 (or one chunk)."""
    if T <= 0:
        return []
    chunk = max(1, int(chunk))
    ramp = []
    s = max(1, chunk // 8)
    while s < chunk:
        ramp.append(s)
        s *= 2
    middle = T - 2 * sum(ramp)
    if ramp and middle >= 1:
        m = -(-middle // chunk)
        sizes = ramp + [middle // m + (1 if i < middle % m else 0) for i in range(m)] + ramp[::-1]
    else:
        piece = max(1, chunk // 8) if ramp else chunk
        n = -(-T // piece)
        sizes = [T // n + (1 if i < T % n else 0) for i in range(n)]
    bounds, a = [], 0
    for sz in sizes:
        bounds.append((a, a + sz))
        a += sz
    assert a == T
    return bounds


class MoENullLayer:
    def __init__(self, d: int, N: int, M: int, K: int, F: int, F_shared: int, *,
                 w_router: torch.Tensor, router_bias: Optional[torch.Tensor],
                 w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor,
                 ws_gate: torch.Tensor, ws_up: torch.Tensor, ws_down: torch.Tensor,
                 router: str = "tensor", ffn: str = "auto", C: int = 0, V: int = 0,
                 const_vectors: Optional[torch.Tensor] = None, wgrad: str = "pair"):
        """router: "tensor" (router product on the tensor cores, fp32 weights split
        exactly into three bf16 terms) or "fp32_cores" (fp32 FMA on the CUDA cores).
        ffn: "single" (single-CTA tiles), "pair" (expert GEMMs on CTA pairs where the
        shape allows) or "auto" (pairs for calls of at least PAIR_MIN_TOKENS tokens,
        where they measured faster; single-CTA tiles below). wgrad: the backward's weight
        gradients on CTA pairs where the shape allows ("pair", the default: faster on every
        measured workload) or on single CTAs ("single"); the results are the same bit for
        bit. C, V: MoE++ copy and constant experts (router rows N+1 .. N+C+V after the null
        logit; const_vectors [V, d] bf16)."""
        if router not in ("tensor", "fp32_cores"):
            raise ValueError(f"router must be 'tensor' or 'fp32_cores', not {router!r}")
        if ffn not in ("pair", "single", "auto"):
            raise ValueError(f"ffn must be 'pair', 'single' or 'auto', not {ffn!r}")
        if wgrad not in ("pair", "single"):
            raise ValueError(f"wgrad must be 'pair' or 'single', not {wgrad!r}")
        self.d, self.N, self.M, self.K, self.F, self.F_shared = d, N, M, K, F, F_shared
        self.C, self.V = C, V
        self.router, self.ffn, self.wgrad = router, ffn, wgrad
        if V > 0 and (const_vectors is None or tuple(const_vectors.shape) != (V, d)):
            raise ValueError("const_vectors [V, d] bf16 is required when V > 0")
        self.const_vectors = None if V == 0 else const_vectors.contiguous()
        self.flags = ((B.FLAG_ROUTER_FP32_CORES if router == "fp32_cores" else 0) |
                      (B.FLAG_FFN_CTA_PAIR if ffn == "pair" else 0) |
                      (B.FLAG_WGRAD_CTA_PAIR if wgrad == "pair" else 0))
        dev = w_router.device
        self.device = dev
        self.w_router = w_router.contiguous()
        self.router_bias = None if router_bias is None else router_bias.contiguous()
        self.w_down = w_down.contiguous()
        self.shared_down = ws_down.contiguous()
        dm = self.dims(1)
        code = B.check_dims(dm)
        if code != B.OK:
            raise B.MoEError("moe_check_dims", code)
        self.gate_up = torch.empty(B.packed_gate_up_elems(dm, False), dtype=torch.bfloat16, device=dev)
        self.shared_gate_up = torch.empty(B.packed_gate_up_elems(dm, True), dtype=torch.bfloat16, device=dev)
        B.pack_gate_up(dm, w_gate.contiguous(), w_up.contiguous(), ws_gate.contiguous(), ws_up.contiguous(),
                       self.gate_up, self.shared_gate_up)
        # the tensor-core router's three-term split of W_r, prepared once (moe_prepare_router)
        self.router_split = None
        if router == "tensor":
            self.router_split = torch.empty(B.router_split_elems(dm), dtype=torch.bfloat16, device=dev)
            B.prepare_router(dm, self.w_router, self.router_split)
        self._weights = B.Weights(self.w_router.data_ptr(),
                                  None if self.router_bias is None else self.router_bias.data_ptr(),
                                  self.gate_up.data_ptr(), self.w_down.data_ptr(),
                                  self.shared_gate_up.data_ptr(), self.shared_down.data_ptr(),
                                  None if self.const_vectors is None else self.const_vectors.data_ptr(),
                                  None if self.router_split is None else self.router_split.data_ptr())

    @classmethod
    def from_inputs(cls, inp, device="cuda", router: str = "tensor", ffn: str = "auto",
                    wgrad: str = "pair") -> "MoENullLayer":
        c = inp.cfg
        f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        cv = None if c.V == 0 else bf16_tensor(inp.const_vectors, device)
        return cls(c.d, c.N, c.M, c.K, c.F, c.F_shared,
                   w_router=f32(inp.w_router), router_bias=f32(inp.bias),
                   w_gate=bf16_tensor(inp.w_gate, device), w_up=bf16_tensor(inp.w_up, device),
                   w_down=bf16_tensor(inp.w_down, device), ws_gate=bf16_tensor(inp.ws_gate, device),
                   ws_up=bf16_tensor(inp.ws_up, device), ws_down=bf16_tensor(inp.ws_down, device),
                   router=router, ffn=ffn, C=c.C, V=c.V, const_vectors=cv, wgrad=wgrad)

    # With ffn="auto", calls of at least this many tokens run the expert GEMMs on CTA pairs:
    # on the 131072-token skewed workload they measured ~4.5% faster per forward, on 16384-token
    # workloads 1-2% slower (pair tiles round each expert up to 256 rows).
    PAIR_MIN_TOKENS = 65536

    def dims(self, T: int) -> B.Dims:
        flags = self.flags
        if self.ffn == "auto" and T >= self.PAIR_MIN_TOKENS:
            flags |= B.FLAG_FFN_CTA_PAIR
        return B.dims(T, self.d, self.N, self.M, self.K, self.F, self.F_shared, flags, self.C, self.V)

    def alloc(self, T: int, logits: bool = True, xs: bool = True, save_preact: bool = False,
              combine: str = "inplace") -> Dict[str, torch.Tensor]:
        """Caller-owned buffers for a T-token call (R_cap = T*K rows). xs=False
        leaves out the gathered copy of the routed rows: the forward then gathers
        rows of x inside the gate/up GEMM and dispatch writes no copies.
        save_preact=True (training) adds z/z_shared: the forward keeps the gate/up
        pre-activations and the backward does not recompute them.
        combine: where the shared expert's output goes and how the routed outputs are
        added to it.
          "inplace" (default): the down GEMM writes it into y and the combine adds the
            gated routed rows in place, skipping tokens without any (their y is done);
          "separate": a buffer of its own (out["shared_out"]), read by the combine;
          "fused": the combine runs in the down GEMM's shared-expert tiles
            (moe_expert_down_combine) and that output never goes to memory.
        All three give bit-identical y."""
        if combine not in ("inplace", "separate", "fused"):
            raise ValueError(f"combine must be 'inplace', 'separate' or 'fused', not {combine!r}")
        dev, d, N, M, K, F, Fs = self.device, self.d, self.N, self.M, self.K, self.F, self.F_shared
        R = T * K
        i32, f32, bf = torch.int32, torch.float32, torch.bfloat16
        out = dict(
            logits=torch.empty((T, N + 1 + self.C + self.V), dtype=f32, device=dev) if logits else None,
            topk_idx=torch.empty((T, K), dtype=i32, device=dev),
            topk_gate=torch.empty((T, K), dtype=f32, device=dev),
            n_real=torch.empty((T,), dtype=i32, device=dev),
            counts=torch.empty((N,), dtype=i32, device=dev),
            offsets=torch.empty((N + 1,), dtype=i32, device=dev),
            perm_tok=torch.empty((max(R, 1),), dtype=i32, device=dev),
            slot_row=torch.empty((T, K), dtype=i32, device=dev),
            xs=torch.empty((max(R, 1), d), dtype=bf, device=dev) if xs else None,
            h=torch.empty((max(R, 1), F), dtype=bf, device=dev),
            h_shared=torch.empty((max(T, 1), Fs), dtype=bf, device=dev),
            ys=torch.empty((max(R, 1), d), dtype=bf, device=dev),
            shared_out=torch.empty((max(T, 1), d), dtype=bf, device=dev) if combine == "separate" else None,
            y=torch.empty((max(T, 1), d), dtype=bf, device=dev),
            counts_ext=torch.empty((N + M + self.C + self.V,), dtype=i32, device=dev),
            P=torch.empty((N + M + self.C + self.V,), dtype=f32, device=dev),
            losses=torch.empty((2,), dtype=f32, device=dev),
            z=torch.empty((max(R, 1), 2 * F), dtype=bf, device=dev) if save_preact else None,
            z_shared=torch.empty((max(T, 1), 2 * Fs), dtype=bf, device=dev) if save_preact else None,
        )
        if combine == "inplace":
            out["shared_out"] = out["y"]
        out["workspace"] = torch.empty((max(B.workspace_bytes(self.dims(T)), 256),), dtype=torch.uint8, device=dev)
        return out

    def alloc_grads(self, T: int) -> Dict[str, torch.Tensor]:
        """Gradient buffers and the backward workspace for a T-token backward."""
        dev, d, N, F, Fs = self.device, self.d, self.N, self.F, self.F_shared
        rows = N + 1 + self.C + self.V
        bf, f32 = torch.bfloat16, torch.float32
        g = dict(
            dx=torch.empty((max(T, 1), d), dtype=bf, device=dev),
            dw_router=torch.empty((rows, d), dtype=f32, device=dev),
            dbias=torch.empty((rows,), dtype=f32, device=dev),
            dtok_null_bias=torch.empty((max(T, 1),), dtype=f32, device=dev),
            dw_gate=torch.empty((N, F, d), dtype=bf, device=dev),
            dw_up=torch.empty((N, F, d), dtype=bf, device=dev),
            dw_down=torch.empty((N, d, F), dtype=bf, device=dev),
            dws_gate=torch.empty((Fs, d), dtype=bf, device=dev),
            dws_up=torch.empty((Fs, d), dtype=bf, device=dev),
            dws_down=torch.empty((d, Fs), dtype=bf, device=dev),
            dconst=torch.empty((self.V, d), dtype=f32, device=dev) if self.V else None,
        )
        g["workspace"] = torch.empty((max(B.backward_workspace_bytes(self.dims(T)), 256),), dtype=torch.uint8,
                                     device=dev)
        return g

    def saved(self, x: torch.Tensor, out: Dict[str, torch.Tensor], counts_ext: Optional[torch.Tensor] = None,
              t_total: Optional[int] = None) -> B.Saved:
        """The forward tensors the backward reads. counts_ext and t_total default to this
        call's own (one data-parallel rank); pass the all-reduced ones otherwise."""
        if out.get("logits") is None or out.get("xs") is None:
            raise ValueError("the backward needs the forward's logits and xs")
        ce = out["counts_ext"] if counts_ext is None else counts_ext
        ptr = lambda t: t.data_ptr()
        z, zs = out.get("z"), out.get("z_shared")
        return B.Saved(ptr(x), ptr(out["logits"]), ptr(out["topk_idx"]), ptr(out["topk_gate"]),
                       ptr(out["offsets"]), ptr(out["slot_row"]), ptr(out["xs"]), ptr(out["h"]),
                       ptr(out["h_shared"]), ptr(out["ys"]), ptr(ce),
                       int(x.shape[0] if t_total is None else t_total),
                       None if z is None else ptr(z), None if zs is None else ptr(zs))

    def backward(self, x: torch.Tensor, out: Dict[str, torch.Tensor], dy: torch.Tensor, alpha: float = 2e-2,
                 beta: float = 1e-3, grads: Optional[Dict[str, torch.Tensor]] = None,
                 counts_ext: Optional[torch.Tensor] = None, t_total: Optional[int] = None,
                 stream=None) -> Dict[str, torch.Tensor]:
        """Gradients of <y, dy> + alpha L_bal + beta L_z through ``moe_backward``."""
        T = x.shape[0]
        if grads is None:
            grads = self.alloc_grads(T)
        sv = self.saved(x, out, counts_ext, t_total)
        g = B.Grads(*[None if grads.get(n) is None else grads[n].data_ptr() for n in B.GRAD_FIELDS])
        B.backward(self.dims(T), self._weights, sv, dy, alpha, beta, g, grads["workspace"], stream)
        return grads

    def alloc_host_pipeline(self, chunk: int, nsets: int = 2) -> Dict[str, object]:
        """Device buffers for forward_host with token chunks of at most ``chunk``: ``nsets``
        chunk-sized output sets and input stagings (one chunk computes while the next is copied
        in and the previous one copied out), the summed statistics and the batch's counts, P
        and losses, and the two copy streams."""
        dev = self.device
        sets = [self.alloc(chunk, logits=False) for _ in range(max(2, int(nsets)))]
        for o in sets:
            o["x_stage"] = torch.empty((chunk, self.d), dtype=torch.bfloat16, device=dev)
        n = B.aux_sums_count(self.dims(1))
        pool = self.N + self.M + self.C + self.V
        return dict(chunk=chunk, sets=sets,
                    sums=torch.empty((n,), dtype=torch.float64, device=dev),
                    counts_ext=torch.empty((pool,), dtype=torch.int32, device=dev),
                    P=torch.empty((pool,), dtype=torch.float32, device=dev),
                    losses=torch.empty((2,), dtype=torch.float32, device=dev),
                    copy_in=torch.cuda.Stream(device=dev), copy_out=torch.cuda.Stream(device=dev))

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, pipe: Dict[str, object],
                     tok_null_bias_host: Optional[torch.Tensor] = None,
                     reduce_sums=None) -> Dict[str, torch.Tensor]:
        """The forward from and to host memory (pinned, for asynchronous copies), in token
        chunks (``chunk_bounds``): while chunk i runs on the current stream, chunk i+1's tokens
        are copied in on one stream and chunk i-1's y copied out on another. Every step of the layer is per
        token, so y is bit-identical to one forward over the whole batch; the statistics of
        L_bal and L_z, which are means over the whole batch, are summed over the chunks on the
        device (moe_aux_sums / moe_aux_sums_accumulate) and finalised once. Returns the device
        counts_ext, P and losses of the batch. The current stream is ordered after the last
        copy, so synchronising it makes y_host complete. The per-token null offsets (4 B a
        token) are copied in once for the whole batch, ahead of the first chunk, into a device
        buffer the pipeline keeps (allocated by the first call that needs it, grown with T):
        one small copy per chunk would leave a gap in the copy-in stream each time. reduce_sums (data parallel: e.g.
        dist.allreduce_aux_sums) is applied to the summed statistics before they are
        finalised, so the losses are the whole job's."""
        T = x_host.shape[0]
        chunk = pipe["chunk"]
        comp = torch.cuda.current_stream(self.device)
        cin, cout = pipe["copy_in"], pipe["copy_out"]
        sets = pipe["sets"]
        cin.wait_stream(comp)  # nothing is copied in before earlier work on this stream
        ev_in = [torch.cuda.Event() for _ in sets]
        ev_done = [torch.cuda.Event() for _ in sets]
        ev_out = [torch.cuda.Event() for _ in sets]
        ns = len(sets)
        tnb_dev = None
        if tok_null_bias_host is not None:
            tnb_dev = pipe.get("tnb_batch")
            if tnb_dev is None or tnb_dev.numel() < T:
                tnb_dev = torch.empty((T,), dtype=torch.float32, device=self.device)
                pipe["tnb_batch"] = tnb_dev
            with torch.cuda.stream(cin):
                tnb_dev[:T].copy_(tok_null_bias_host, non_blocking=True)
        for c, (a, b) in enumerate(chunk_bounds(T, chunk)):
            k = c % ns
            o = sets[k]
            Tc = b - a
            with torch.cuda.stream(cin):
                if c >= ns:
                    cin.wait_event(ev_done[k])  # the set's previous chunk no longer reads this staging
                o["x_stage"][:Tc].copy_(x_host[a:b], non_blocking=True)
                ev_in[k].record(cin)  # also covers the offsets' copy, issued before chunk 0's
            comp.wait_event(ev_in[k])
            if c >= ns:
                comp.wait_event(ev_out[k])  # the set's previous chunk's y has been copied out
            dm = self.dims(Tc)
            x = o["x_stage"][:Tc]
            tnb = None if tnb_dev is None else tnb_dev[a:b]
            ob = B.Outputs(*[None if o.get(f) is None else o[f].data_ptr() for f in B.OUTPUT_FIELDS])
            B.forward(dm, self._weights, x, tnb, ob, o["workspace"], comp)
            if c == 0:
                B.aux_sums(dm, o["workspace"], pipe["sums"], comp)
            else:
                B.aux_sums_accumulate(dm, o["workspace"], pipe["sums"], comp)
            ev_done[k].record(comp)
            with torch.cuda.stream(cout):
                cout.wait_event(ev_done[k])
                y_host[a:b].copy_(o["y"][:Tc], non_blocking=True)
                ev_out[k].record(cout)
        if reduce_sums is not None:
            reduce_sums(pipe["sums"])
        B.aux_finalize(self.dims(T), pipe["sums"], pipe["counts_ext"], pipe["P"], pipe["losses"], comp)
        comp.wait_stream(cout)
        return dict(counts_ext=pipe["counts_ext"], P=pipe["P"], losses=pipe["losses"])

    def capture_forward(self, x: torch.Tensor, tok_null_bias: Optional[torch.Tensor],
                        out: Dict[str, torch.Tensor]) -> "torch.cuda.CUDAGraph":
        """A CUDA graph of one forward over fixed buffers. replay() recomputes ``out`` from the
        current contents of x (and tok_null_bias) with no host-side launch work, which is what
        bounds a decode-sized step: seven launches of a few microseconds of GPU work each. The
        graph holds the addresses of x, tok_null_bias, the weights and every buffer of ``out``,
        so new tokens are copied into x in place between replays, and the buffers must outlive
        the graph. One eager forward runs first, so that one-time work (kernel attributes,
        cached device properties) happens outside the capture."""
        self.forward(x, tok_null_bias, out)
        cur = torch.cuda.current_stream(self.device)
        side = torch.cuda.Stream(device=self.device)
        side.wait_stream(cur)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            self.forward(x, tok_null_bias, out)
        cur.wait_stream(side)
        return g

    def forward(self, x: torch.Tensor, tok_null_bias: Optional[torch.Tensor] = None,
                out: Optional[Dict[str, torch.Tensor]] = None, stream=None) -> Dict[str, torch.Tensor]:
        T = x.shape[0]
        if out is None:
            out = self.alloc(T)
        o = B.Outputs(*[None if out.get(n) is None else out[n].data_ptr() for n in B.OUTPUT_FIELDS])
        B.forward(self.dims(T), self._weights, x, tok_null_bias, o, out["workspace"], stream)
        return out
