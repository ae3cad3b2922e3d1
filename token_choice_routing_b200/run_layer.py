"""Run a few forwards (and backwards) of one seeded workload through the C ABI.

    python -m token_choice_routing_b200.run_layer [--config qwen3_0p6b] [--tokens T] [--forwards 3]
        [--backwards 0] [--save-preact] [--router tensor|fp32_cores] [--ffn single|pair]
        [--combine inplace|separate|fused]

--tokens T draws only T tokens of the workload (the skewed one keeps its span pattern per
8192-token sequence), for captures whose inputs should exceed L2 but stay a few GB.

With --backwards N the forwards keep the logits and the gathered rows, and N backward
passes of <y, dy> + 2e-2 L_bal + 1e-3 L_z (seeded dy) follow them. --save-preact runs the
training mode: the forwards also save the gate/up pre-activations and the backwards take the
SwiGLU derivative from them.

Used as the target of profiler captures (ncu -k <kernel> -s/-c selects the
launch). Exits non-zero if the device status word reports an error.
"""
import argparse
import sys

import torch

from . import binding as B
from . import inputs as I
from .layer import MoENullLayer, bf16_tensor


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="qwen3_0p6b", choices=sorted(I.CONFIGS))
    ap.add_argument("--tokens", type=int, default=0, help="draw only this many tokens (0: the workload's T)")
    ap.add_argument("--combine", default="inplace", choices=["inplace", "separate", "fused"])
    ap.add_argument("--forwards", type=int, default=3)
    ap.add_argument("--router", default="tensor", choices=["tensor", "fp32_cores"])
    ap.add_argument("--ffn", default="auto", choices=["auto", "single", "pair"])
    ap.add_argument("--backwards", type=int, default=0)
    ap.add_argument("--save-preact", action="store_true")
    a = ap.parse_args(argv)
    cfg = I.CONFIGS[a.config]
    if a.tokens > 0:
        import dataclasses
        seqs = max(1, cfg.seqs * a.tokens // cfg.T) if cfg.skew else cfg.seqs
        cfg = dataclasses.replace(cfg, T=a.tokens, seqs=seqs)
    inp = I.make_inputs(cfg)
    layer = MoENullLayer.from_inputs(inp, "cuda", router=a.router, ffn=a.ffn)
    x = bf16_tensor(inp.x, "cuda")
    tnb = None if inp.tok_null_bias is None else torch.from_numpy(inp.tok_null_bias).cuda()
    out = layer.alloc(inp.cfg.T, logits=a.backwards > 0, save_preact=a.save_preact, combine=a.combine)
    for _ in range(a.forwards):
        layer.forward(x, tnb, out)
    torch.cuda.synchronize()
    st = B.get_device_status(out["workspace"])
    print(f"{a.config} (T={inp.cfg.T}): {a.forwards} forwards, R={int(out['offsets'][-1])}, "
          f"status={B.status_string(st)}")
    if st != B.OK or a.backwards <= 0:
        return 0 if st == B.OK else 1
    dy = bf16_tensor(I.upstream_grad(inp.cfg), "cuda")
    grads = layer.alloc_grads(inp.cfg.T)
    for _ in range(a.backwards):
        layer.backward(x, out, dy, 2e-2, 1e-3, grads=grads)
    torch.cuda.synchronize()
    st = B.get_device_status(grads["workspace"])
    print(f"{a.config}: {a.backwards} backwards, status={B.status_string(st)}")
    return 0 if st == B.OK else 1


if __name__ == "__main__":
    sys.exit(main())
