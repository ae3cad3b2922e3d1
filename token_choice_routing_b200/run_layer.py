"""Run a few forwards of one seeded workload through the C ABI.

    python -m token_choice_routing_b200.run_layer [--config qwen3_0p6b] [--forwards 3]
        [--router tensor|fp32_cores] [--ffn single|pair]

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
    ap.add_argument("--forwards", type=int, default=3)
    ap.add_argument("--router", default="tensor", choices=["tensor", "fp32_cores"])
    ap.add_argument("--ffn", default="single", choices=["single", "pair"])
    a = ap.parse_args(argv)
    inp = I.make_inputs(I.CONFIGS[a.config])
    layer = MoENullLayer.from_inputs(inp, "cuda", router=a.router, ffn=a.ffn)
    x = bf16_tensor(inp.x, "cuda")
    tnb = None if inp.tok_null_bias is None else torch.from_numpy(inp.tok_null_bias).cuda()
    out = layer.alloc(inp.cfg.T, logits=False)
    for _ in range(a.forwards):
        layer.forward(x, tnb, out)
    torch.cuda.synchronize()
    st = B.get_device_status(out["workspace"])
    print(f"{a.config}: {a.forwards} forwards, R={int(out['offsets'][-1])}, status={B.status_string(st)}")
    return 0 if st == B.OK else 1


if __name__ == "__main__":
    sys.exit(main())
