"""Calibrate the null-logit bias of each workload; writes null_bias.json.

For a workload with M null copies and top-K, the null bias b is the scalar
added to the null logit so that the mean number of real experts per token is
as close as possible to rho*K, rho = N/(N+M) (the paper's data-sparsity target
E[K] = rho*k_max: "Improving MoE Compute Efficiency by Composing Weight and
Data Sparsity", review page, section 三 / 期望活跃专家数). The mean real count
is non-increasing in b, so b is found by 60 bisection steps on [-30, 30] over
the oracle's float64 logits of the seeded inputs, using the oracle's threshold
count. Only the oracle and the input generator are used.

Run:  python tests/golden/calibrate_null_bias.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle as O  # noqa: E402
from token_choice_routing_b200.inputs import CONFIGS, make_inputs, bf16_to_f32  # noqa: E402


def mean_real(s, M, K, b):
    sb = s.copy()
    sb[:, -1] += b
    return float(O.threshold_real_count(sb, M, K).mean())


def calibrate(cfg, steps=60):
    inp = make_inputs(cfg, weights=False, null_bias=0.0)
    s = O.router_logits(bf16_to_f32(inp.x), inp.w_router, inp.bias)
    target = cfg.rho * cfg.K
    lo, hi = -30.0, 30.0
    for _ in range(steps):
        mid = 0.5 * (lo + hi)
        if mean_real(s, cfg.M, cfg.K, mid) > target:
            lo = mid
        else:
            hi = mid
    cands = [float(np.float32(lo)), float(np.float32(hi))]
    errs = [abs(mean_real(s, cfg.M, cfg.K, c) - target) for c in cands]
    b = cands[int(np.argmin(errs))]
    return b, mean_real(s, cfg.M, cfg.K, b), target


def calibrated_names():
    return [n for n, c in CONFIGS.items() if c.M > 0 and not c.skew]


if __name__ == "__main__":
    out = {}
    for name in calibrated_names():
        b, r, target = calibrate(CONFIGS[name])
        out[name] = {"null_bias": b, "mean_real": r, "target": target}
        print(name, out[name], flush=True)
    with open(os.path.join(HERE, "null_bias.json"), "w") as f:
        json.dump(out, f, indent=1, sort_keys=True)
