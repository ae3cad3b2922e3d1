#!/usr/bin/env python
"""Benchmark of the null-expert MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config skew] [--no-backward] [--no-per-config] [--no-cpu-baseline]

A step is one full forward of the layer (route -> dispatch + aux -> grouped
gate/up SwiGLU GEMM -> grouped down GEMM -> combine) over one batch of T
synthetic tokens that is already resident in HBM. L2 is flushed (a 256 MiB
write) between timed steps; each step is timed with CUDA events on the
launching stream. Prints one JSON line (rank 0).

The default workload is the largest single-GPU one: the skewed batch of
16 x 8192 tokens on the 1.7B-shaped layer (d=2048, N=64, F=1536, K=8, M=64).
Beside it, one GPU also measures the training-mode backward on the same
workload (`backward`) and forward-only steps of the 0.6B- and 1.7B-shaped layers
and of the four points of the matched E[K]=2 sparsity sweep (`per_config`).

Metric: real (token, expert) slots per second for the layer forward, i.e. R /
t_step summed over ranks (null slots are not counted). Multi-GPU runs are data
parallel (each rank its own T tokens, weak scaling) with one NCCL all-reduce
of the additive aux statistics per step, the layer's only exchange.

`e2e` is the same metric through the layer's public forward with host buffers:
every step copies x in from pinned host memory and y, the losses and the slot
counts back to pinned host memory, inside the timed region.

--impl reference times the CPU oracle (the float64 NumPy restatement used by
the tests) on a bounded sample of the same workload's tokens, on the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "real-slot tokens/s per MoE layer fwd; grouped-GEMM TFLOP/s vs BF16 peak"
UNIT = "real-slot tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# Sources whose change invalidates a recorded ncu traffic figure of the grouped GEMM.
GEMM_SOURCES = ("token_choice_routing_b200/csrc/expert_ffn.cu", "token_choice_routing_b200/csrc/moe_internal.cuh")
PAIR_GEMM_SOURCES = ("token_choice_routing_b200/csrc/expert_ffn_pair.cu",
                     "token_choice_routing_b200/csrc/moe_internal.cuh")
GEMM_PROFILE = "profiles/grouped_gemm_qwen3_0p6b.md"
GEMM_PROFILES = (GEMM_PROFILE, "profiles/grouped_gemm_skew.md")
BWD_GEMM_SOURCES = ("token_choice_routing_b200/csrc/expert_ffn_bwd.cu", "token_choice_routing_b200/csrc/moe_internal.cuh")
BWD_GEMM_PROFILE = "profiles/bwd_gemm_kernel_qwen3_0p6b.md"
BWD_GEMM_PROFILES = (BWD_GEMM_PROFILE, "profiles/wgrad_pair_kernel_qwen3_0p6b.md", "profiles/wgrad_pair_kernel_skew.md")


def gemm_source_digest(sources=GEMM_SOURCES) -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in sources:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(workload: str, kernel: str, profile=GEMM_PROFILE, sources=GEMM_SOURCES):
    """DRAM bytes (read + write) of one launch of `kernel` from a committed ncu summary:
    its line 'traffic-record: workload=W kernel=K dram_bytes_per_launch=B source_sha256=H'.
    None unless it was taken on this workload from the current kernel sources. `profile`
    is one summary file or a tuple of them."""
    lines = []
    for prof in ((profile,) if isinstance(profile, str) else profile):
        try:
            with open(os.path.join(ROOT, prof)) as f:
                lines += [l.strip() for l in f if l.strip().startswith("traffic-record:")]
        except OSError:
            pass
    if not lines:
        return None
    digest = gemm_source_digest(sources)
    for l in lines:
        kv = dict(p.split("=", 1) for p in l.split()[1:] if "=" in p)
        if kv.get("workload") == workload and kv.get("kernel") == kernel and kv.get("source_sha256") == digest:
            return float(kv["dram_bytes_per_launch"])
    return None


def recorded_gate_up_traffic(workload: str, pair: bool = False):
    """The gate/up launch's recorded DRAM bytes: the single-CTA kernel ("gate_up") or the
    CTA-pair kernel ("gate_up_pair"), each pinned to its own sources."""
    if pair:
        return recorded_traffic(workload, "gate_up_pair", GEMM_PROFILES, PAIR_GEMM_SOURCES)
    return recorded_traffic(workload, "gate_up", GEMM_PROFILES)


class ClockSampler:
    """Samples the GPU's SM clock and clock-event (throttle) reasons through NVML
    from a background thread while the timed region runs."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device_index: int, period_s: float = 0.002):
        self.idx = torch_device_index
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False

    def __enter__(self):
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(self.idx).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode() if isinstance(uuid, str) else uuid)
            self.nv = pynvml
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self._ok = True
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
            time.sleep(0.05)
            self.samples.clear()  # keep only what is sampled while the measured work runs
        except Exception as e:  # NVML missing: the line says so
            self.err = repr(e)
        return self

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
                self.samples.append((sm, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        self._stop.set()
        if self._ok:
            self.t.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        reasons = set()
        for _, rs in self.samples:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the cpu_baseline object)

def sample_tokens(T: int, S: int):
    """S token indices spread evenly over the batch, so that a sample of a workload with
    token spans of different kinds (the skewed one) holds each kind in its proportion."""
    import numpy as np
    S = max(1, min(T, S))
    return np.unique(np.linspace(0, T - 1, S).round().astype(np.int64))


_F64_WEIGHTS = {}


def f64_weights(inp):
    """The expert weights widened to float64 once per workload (outside the timed region, as
    the GPU arm's weights are resident before its timing starts)."""
    import numpy as np
    from token_choice_routing_b200 import inputs as I
    key = inp.cfg.name
    if key not in _F64_WEIGHTS:
        _F64_WEIGHTS.clear()
        f = lambda b: I.bf16_to_f32(b).astype(np.float64)
        _F64_WEIGHTS[key] = ((f(inp.w_gate), f(inp.w_up), f(inp.w_down)),
                             (f(inp.ws_gate), f(inp.ws_up), f(inp.ws_down)))
    return _F64_WEIGHTS[key]


def oracle_sample_run(inp, S):
    """Full oracle forward on S tokens spread over the batch, stage by stage.
    Returns (seconds, real slots, {stage: seconds}); the stages are the oracle's own
    functions: route (router logits, pool, top-K, gates), dispatch, experts (the SwiGLU
    experts and the gated sum, one oracle function) and aux."""
    import numpy as np
    import oracle as O
    from token_choice_routing_b200 import inputs as I
    cfg = inp.cfg
    f = lambda b: I.bf16_to_f32(b).astype(np.float64)
    experts, shared = f64_weights(inp)
    tok = sample_tokens(cfg.T, S)
    st = {}
    t0 = time.perf_counter()
    x = f(inp.x[tok])
    tnb = None if inp.tok_null_bias is None else inp.tok_null_bias[tok]
    s = O.router_logits(x, inp.w_router, inp.bias, tnb)
    r = O.route(s, cfg.M, cfg.K)
    t1 = time.perf_counter()
    O.dispatch(r["idx"], cfg.N)
    t2 = time.perf_counter()
    O.layer_output(x, r["idx"], r["gates"], cfg.N, experts, shared)
    t3 = time.perf_counter()
    O.aux_stats(r["idx"], r["p"], r["lse"], cfg.N, cfg.M)
    t4 = time.perf_counter()
    st = {"route": t1 - t0, "dispatch": t2 - t1, "experts_and_combine": t3 - t2, "aux": t4 - t3}
    return t4 - t0, int(r["n_real"].sum()), st


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def calibrate_sample(inp, target_s):
    S0 = min(inp.cfg.T, 512)
    dt, _, _ = oracle_sample_run(inp, S0)
    S = int(S0 * target_s / max(dt, 1e-3))
    return max(64, min(inp.cfg.T, S))


def oracle_steps(inp, S, steps):
    """`steps` oracle forwards of the same S-token sample; per-step seconds, per-stage medians."""
    per_step, stages, tot_r = [], {}, 0
    for _ in range(steps):
        dt, R, st = oracle_sample_run(inp, S)
        per_step.append(dt)
        tot_r += R
        for k, v in st.items():
            stages.setdefault(k, []).append(v)
    return per_step, tot_r, {k: statistics.median(v) for k, v in stages.items()}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from token_choice_routing_b200 import inputs as I
    cfg = I.CONFIGS[args.config]
    inp = I.make_inputs(cfg)
    S = calibrate_sample(inp, args.ref_step_seconds)
    for _ in range(args.warmup):
        oracle_sample_run(inp, S)
    per_step, tot_r, stages = oracle_steps(inp, S, args.steps)
    tot_t = sum(per_step)
    value = tot_r / tot_t
    cores = blas_threads()
    sample = (f"{len(sample_tokens(cfg.T, S))} of {cfg.T} tokens per step, spread evenly over the batch "
              "(full oracle forward: route, dispatch, experts, aux)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) tokens, N(0,1/fan_in) weights)",
        "config": workload_config(cfg, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                         "stage_s_median": stages, "step_s": per_step},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


BWD_ALPHA, BWD_BETA = 2e-2, 1e-3  # load-balance and Z-loss weights of the paper's training runs


def measure_backward(args, cfg, layer, x, tnb, flush, peaks, peak_kind):
    """Backward pass of the same layer: gradients of <y, dy> + alpha L_bal + beta L_z with a
    seeded dy, the forward's tensors resident. Training mode: the forward keeps the gate/up
    pre-activations (its time is reported as forward_training_ms) and the backward takes the
    SwiGLU derivative from them. The timed step is one moe_backward call (L2 flushed before
    each). The backward that recomputes the pre-activations instead is timed too
    (backward_recompute_ms). The stages are then timed one by one through their entry points."""
    import numpy as np
    import torch
    from token_choice_routing_b200 import binding as B
    from token_choice_routing_b200 import inputs as I
    from token_choice_routing_b200.layer import bf16_tensor

    dev = x.device
    T, d, F, Fs, N, K = cfg.T, cfg.d, cfg.F, cfg.F_shared, cfg.N, cfg.K
    rows = N + 1 + cfg.C + cfg.V
    bout = layer.alloc(T, logits=True, xs=True, save_preact=True)   # training forward
    rout = layer.alloc(T, logits=True, xs=True)                      # no saved pre-activations
    layer.forward(x, tnb, rout)
    dy = bf16_tensor(I.upstream_grad(cfg), dev)
    grads = layer.alloc_grads(T)
    bws = grads["workspace"]

    def timed(fn):
        for _ in range(args.warmup):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for e0, e1 in evs:
            flush.zero_()
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize()
        return sum(e0.elapsed_time(e1) for e0, e1 in evs)

    fwd_train_ms = timed(lambda: layer.forward(x, tnb, bout)) / args.steps
    recompute_ms = timed(lambda: layer.backward(x, rout, dy, BWD_ALPHA, BWD_BETA, grads=grads)) / args.steps
    total_ms = timed(lambda: layer.backward(x, bout, dy, BWD_ALPHA, BWD_BETA, grads=grads))
    st = B.get_device_status(bws)
    if st != B.OK:
        raise SystemExit(f"backward device status: {B.status_string(st)}")
    R = int(bout["offsets"][-1].item())

    # stages one by one, CUDA events between them
    dm = layer.dims(T)
    Rc = T * K
    dys = torch.empty((Rc, d), dtype=torch.bfloat16, device=dev)
    dg = torch.empty((T, K), dtype=torch.float32, device=dev)
    ds = torch.empty((T, rows), dtype=torch.float32, device=dev)
    dxs = torch.empty((Rc, d), dtype=torch.bfloat16, device=dev)
    o = bout
    stages = [
        ("combine_bwd", lambda: B.combine_backward(dm, dy, o["ys"], o["topk_gate"], o["slot_row"], dys, dg, bws,
                                                   topk_idx=o["topk_idx"], x=x, const_vectors=layer.const_vectors)),
        ("router_bwd", lambda: B.router_backward(dm, o["logits"], o["topk_idx"], o["topk_gate"], dg, o["counts_ext"],
                                                 T, BWD_ALPHA, BWD_BETA, ds, bws, grads["dtok_null_bias"])),
        ("router_wgrad", lambda: B.router_weight_grad(dm, x, grads["dw_router"], grads["dbias"], bws)),
        ("dgrad_down", lambda: B.expert_dgrad_down(dm, o["offsets"], dys, dy, layer.w_down, layer.shared_down, bws)),
        ("swiglu_bwd", lambda: B.expert_swiglu_backward_saved(dm, o["offsets"], o["z"], o["z_shared"], bws)),
        ("swiglu_bwd_recompute", lambda: B.expert_swiglu_backward(dm, o["xs"], x, o["offsets"], layer.gate_up,
                                                                  layer.shared_gate_up, bws)),
        ("wgrad_down", lambda: B.expert_wgrad_down(dm, o["offsets"], dys, dy, o["h"], o["h_shared"],
                                                   grads["dw_down"], grads["dws_down"], bws)),
        # as moe_backward runs them: the shared expert's input gradient written straight into dx,
        # then the input gradient gather in place over the tokens with a real or copy-expert slot
        ("dgrad_gate_up", lambda: B.expert_dgrad_gate_up(dm, o["offsets"], layer.gate_up, layer.shared_gate_up,
                                                         layer.w_router, dxs, grads["dx"], bws)),
        ("wgrad_gate_up", lambda: B.expert_wgrad_gate_up(dm, o["offsets"], o["xs"], x, grads["dw_gate"],
                                                         grads["dw_up"], grads["dws_gate"], grads["dws_up"], bws)),
        ("input_grad", lambda: B.input_grad(dm, grads["dx"], dxs, o["slot_row"], o["topk_idx"], o["topk_gate"], dy,
                                            grads["dx"], bws)),
    ]
    acc = {n: [] for n, _ in stages}
    nb = max(5, min(args.steps, 11))
    for _ in range(nb):
        flush.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)]
        ev[0].record()
        for i, (_, fn) in enumerate(stages):
            fn()
            ev[i + 1].record()
        torch.cuda.synchronize()
        for i, (n, _) in enumerate(stages):
            acc[n].append(ev[i].elapsed_time(ev[i + 1]))
    st = B.get_device_status(bws)
    if st != B.OK:
        raise SystemExit(f"backward device status: {B.status_string(st)}")
    kms = {n: statistics.median(acc[n]) for n in acc}  # median over the passes
    bf16_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    # the in-place input gradient reads and writes dx only for the tokens with a real or copy slot
    idx = o["topk_idx"][:T]
    t_src = int(((idx < cfg.N) | ((idx >= cfg.N + cfg.M) & (idx < cfg.N + cfg.M + cfg.C))).any(dim=1).sum().item())
    # the router's input gradient ds W_r rides in dgrad_gate_up (extra k-blocks of the shared tiles)
    fl = {"swiglu_bwd_recompute": 4.0 * d * (F * R + Fs * T), "dgrad_down": 2.0 * d * (F * R + Fs * T),
          "wgrad_down": 2.0 * d * (F * R + Fs * T), "dgrad_gate_up": 4.0 * d * (F * R + Fs * T) + 2.0 * rows * d * T,
          "wgrad_gate_up": 4.0 * d * (F * R + Fs * T), "router_wgrad": 2.0 * rows * d * T}
    # the saved-pre-activation SwiGLU backward reads z (4F B) and dh (2F B) and writes dz (4F B) per row
    by = {"swiglu_bwd": 10.0 * (F * R + Fs * T), "combine_bwd": 2.0 * d * T + 4.0 * d * R + 12.0 * K * T,
          "router_bwd": 8.0 * rows * T + 12.0 * K * T,
          "input_grad": 4.0 * d * t_src + 2.0 * d * R + 8.0 * K * T}
    kernels = {}
    for n, ms in kms.items():
        k = {"ms": ms}
        if n in ("swiglu_bwd_recompute", "dgrad_down", "wgrad_down", "dgrad_gate_up", "wgrad_gate_up", "router_wgrad"):
            k.update(bound="tensor", **{"TFLOP/s": fl[n] / (ms * 1e9)})
            k["frac"] = k["TFLOP/s"] / bf16_peak
        elif n in by:
            k.update(bound="hbm", **{"GB/s": by[n] / (ms * 1e6)})
            k["frac"] = k["GB/s"] / hbm_peak
        else:
            k.update(bound="alu", **{"TFLOP/s": fl[n] / (ms * 1e9)})
        kernels[n] = k
    gemm = ["dgrad_down", "wgrad_down", "dgrad_gate_up", "wgrad_gate_up"]
    top = max(gemm, key=lambda n: kms[n])
    # the weight gradients ran on CTA pairs (the layer's default) where the shape allows
    pair_ok = {"wgrad_down": d % 256 == 0 and F % 256 == 0 and Fs % 256 == 0,
               "wgrad_gate_up": d % 256 == 0 and (2 * F) % 256 == 0 and (2 * Fs) % 256 == 0}
    top_pair = layer.wgrad == "pair" and pair_ok.get(top, False)
    gemm_ms = sum(kms[n] for n in gemm)
    gemm_flops = sum(fl[n] for n in gemm)
    # combine_bwd, router_bwd, router wgrad (+ its reduce), W_r split, dgrad down, SwiGLU backward,
    # wgrad down, dgrad gate/up, wgrad gate/up, input_grad (+ the constant experts' gradient)
    launches = 11 + (1 if cfg.V else 0)
    return {
        "metric": "real-slot tokens/s per MoE layer bwd", "value": R * args.steps / (total_ms * 1e-3),
        "unit": UNIT, "ms_per_step": total_ms / args.steps, "steps": args.steps,
        "objective": f"<y, dy> + {BWD_ALPHA} L_bal + {BWD_BETA} L_z (dy seeded N(0,1) bf16)",
        "preactivations": "saved by the forward (training mode); the SwiGLU derivative is an elementwise pass",
        "forward_training_ms": fwd_train_ms, "backward_recompute_ms": recompute_ms,
        "ffn_tflops_real_rows": gemm_flops / (gemm_ms * 1e9),
        "roofline": {"kernel": f"{top} grouped GEMM (tcgen05" + (", CTA pairs)" if top_pair else ")"),
                     "bound": "tensor",
                     "achieved": fl[top] / (kms[top] * 1e9), "peak": bf16_peak, "unit": "TFLOP/s",
                     "frac": fl[top] / (kms[top] * 1e9) / bf16_peak, "peak_kind": f"{peak_kind} bf16 burst",
                     "traffic": recorded_traffic(cfg.name, top + ("_pair" if top_pair else ""), BWD_GEMM_PROFILES,
                                                 BWD_GEMM_SOURCES),
                     "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                     "flops_per_launch": fl[top], "ms_per_launch": kms[top]},
        "kernels": kernels,
        "gpu_launches": launches * args.steps,
    }


def workload_config(cfg, args):
    pp = f" C={cfg.C} V={cfg.V}" if cfg.C + cfg.V else ""
    return {"workload": f"{cfg.name}: MoE layer fwd T={cfg.T} d={cfg.d} N={cfg.N} F={cfg.F} "
                        f"F_shared={cfg.F_shared} K={cfg.K} M={cfg.M}{pp} rho={cfg.rho:.3g}",
            "T": cfg.T, "d": cfg.d, "N": cfg.N, "M": cfg.M, "K": cfg.K, "F": cfg.F, "F_shared": cfg.F_shared,
            "C": cfg.C, "V": cfg.V,
            "global_batch_tokens": cfg.T * args.gpus, "parallelism": f"dp{args.gpus}",
            "router": getattr(args, "router", "tensor"), "ffn": getattr(args, "ffn", "auto"),
            "routed_rows": "gathered from x inside gate/up (cp.async row gathers)" if getattr(args, "gather", False)
            else "copied into xs by dispatch",
            "combine": {"inplace": "shared expert written into y, routed rows added in place",
                        "separate": "shared expert output in its own buffer, then the combine launch",
                        "fused": "inside the down GEMM's shared-expert tiles"}[getattr(args, "combine", "inplace")],
            "l2": "flushed between timed steps (256 MiB write)"}


# ----------------------------------------------------------------------------------------
# GPU arm

# Forward-only workloads measured beside the headline (the per_config object): the 0.6B- and
# 1.7B-shaped layers and the four points of the matched E[K] = 2 data-sparsity sweep.
PER_CONFIG = ("qwen3_0p6b", "qwen3_1p7b", "sweep_k2_m0", "sweep_k3_m32", "sweep_k4_m64", "sweep_k8_m192")

# launches of one forward: header clear (the router weight itself is split once, when the layer
# is built), route, scan, dispatch(+aux), gate/up, down, combine (with --combine fused the combine
# runs inside the down GEMM: one launch fewer)
FWD_LAUNCHES = 7


def timed_events(fn, steps, warmup, flush, sync_before=None):
    """Per-step device milliseconds of `fn` (CUDA events on the current stream, L2 flushed
    by a 256 MiB write before every step, warm-up steps untimed)."""
    import torch
    for _ in range(warmup):
        flush.zero_()
        fn()
    torch.cuda.synchronize()
    if sync_before is not None:
        sync_before()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in evs:
        flush.zero_()
        e0.record()
        fn()
        e1.record()
    torch.cuda.synchronize()
    return [e0.elapsed_time(e1) for e0, e1 in evs]


def forward_stage_ms(layer, dm, x, tnb, out, flush, nb):
    """Median device ms of the forward's stages over nb passes, each stage launched through its
    own entry point in the forward's order with CUDA events between them (L2 flushed before
    each pass; the median, so that a pass disturbed by a clock dip does not set it). With no
    shared_out buffer the combine runs inside the down GEMM ("down_combine"), as in the
    forward; otherwise "down" and "combine" are separate launches."""
    import torch
    from token_choice_routing_b200 import binding as B
    fused = out.get("shared_out") is None
    names = ["route", "dispatch", "gate_up"] + (["down_combine"] if fused else ["down", "combine"])
    acc = {n: [] for n in names}
    for _ in range(nb):
        flush.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
        ev[0].record()
        # "route" = header clear + route + scan launches from the prepared router weight, as in the
        # forward (the fp32 CUDA-core router transposes its weight per call instead)
        if layer.router_split is not None:
            B.route_prepared(dm, x, layer.router_split, layer.router_bias, tnb, None, out["topk_idx"],
                             out["topk_gate"], out["n_real"], out["workspace"])
        else:
            B.route(dm, x, layer.w_router, layer.router_bias, tnb, None, out["topk_idx"], out["topk_gate"],
                    out["n_real"], out["workspace"])
        ev[1].record()
        B.dispatch(dm, x, out["topk_idx"], out["workspace"], out["counts"], out["offsets"], out["perm_tok"],
                   out["slot_row"], out["xs"])  # the aux reduction rides in this launch, as in moe_forward
        ev[2].record()
        if out["xs"] is None:
            B.expert_gate_up_gather(dm, x, out["perm_tok"], out["offsets"], layer.gate_up, layer.shared_gate_up,
                                    out["h"], out["h_shared"], out["workspace"])
        else:
            B.expert_gate_up(dm, out["xs"], x, out["offsets"], layer.gate_up, layer.shared_gate_up, out["h"],
                             out["h_shared"], out["workspace"])
        ev[3].record()
        if fused:
            B.expert_down_combine(dm, out["offsets"], out["h"], out["h_shared"], layer.w_down, layer.shared_down,
                                  out["ys"], out["topk_gate"], out["slot_row"], out["y"], out["workspace"],
                                  topk_idx=out["topk_idx"], x=x, const_vectors=layer.const_vectors)
            ev[4].record()
        else:
            B.expert_down(dm, out["offsets"], out["h"], out["h_shared"], layer.w_down, layer.shared_down,
                          out["ys"], out["shared_out"], out["workspace"])
            ev[4].record()
            if out["shared_out"].data_ptr() == out["y"].data_ptr():
                # in place, as moe_forward runs it: only the tokens the route listed
                B.combine_inplace(dm, out["ys"], out["topk_gate"], out["slot_row"], out["y"], out["workspace"],
                                  topk_idx=out["topk_idx"], x=x, const_vectors=layer.const_vectors)
            else:
                B.combine(dm, out["ys"], out["shared_out"], out["topk_gate"], out["slot_row"], out["y"],
                          topk_idx=out["topk_idx"], x=x, const_vectors=layer.const_vectors)
            ev[5].record()
        torch.cuda.synchronize()
        for i, n in enumerate(names):
            acc[n].append(ev[i].elapsed_time(ev[i + 1]))
    return {n: statistics.median(acc[n]) for n in names}


def forward_figures(cfg, R, kms, peaks, args, out):
    """Per-kernel throughput and roofline fractions of one forward from its stage times.
    GEMM FLOPs count real rows only (routed real slots and the shared expert's T rows);
    route, dispatch and combine count the bytes the method must move. The down GEMM with
    the combine inside it is reported against the tensor peak (its FLOPs) and, beside
    that, the combine's own bytes over the same time."""
    T, d, F, Fs, N, K = cfg.T, cfg.d, cfg.F, cfg.F_shared, cfg.N, cfg.K
    flops_gu = 4.0 * d * F * R + 4.0 * d * Fs * T
    flops_dn = 2.0 * d * F * R + 2.0 * d * Fs * T
    bytes_route = 2.0 * d * T + (8.0 * K + 4.0) * T
    # dispatch: topk_idx and in-block ranks read, slot_row written (4 B each per slot), perm_tok per real
    # slot; plus, when it copies rows into xs, 2d B read and 2d B written per real slot
    bytes_dispatch = 12.0 * K * T + 4.0 * R + (0.0 if args.gather else 4.0 * d * R)
    # combine: each real slot's row of ys (2d B); the shared expert's row read and y written (4d B)
    # for every token, or in place only for the tokens that have a source at all
    if getattr(args, "combine", "separate") == "inplace":
        t_src = int((out["n_real"][:T] > 0).sum().item()) if cfg.C + cfg.V == 0 else T
        bytes_combine = 2.0 * d * R + 4.0 * d * t_src
    else:
        bytes_combine = 2.0 * d * R + 4.0 * d * T
    if cfg.C + cfg.V > 0:  # MoE++ copy/constant slots read a row of x or a constant vector
        bytes_combine += 2.0 * d * float(out["counts_ext"][cfg.N + cfg.M:].sum().item())
    bf16_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    fp32_peak = 148 * 128 * 2 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12
    b = {
        "route": {"ms": kms["route"], "bound": "alu" if args.router == "fp32_cores" else "hbm",
                  "TFLOP/s": 2.0 * (N + 1) * d * T / (kms["route"] * 1e9),
                  "GB/s": bytes_route / (kms["route"] * 1e6)},
        "dispatch": {"ms": kms["dispatch"], "bound": "hbm", "GB/s": bytes_dispatch / (kms["dispatch"] * 1e6)},
        "gate_up": {"ms": kms["gate_up"], "bound": "tensor", "TFLOP/s": flops_gu / (kms["gate_up"] * 1e9)},
    }
    if args.router == "fp32_cores":  # the CUDA-core product: its bound is the fp32 FMA rate
        b["route"]["frac_fp32_alu"] = b["route"]["TFLOP/s"] / fp32_peak
    else:  # on the tensor cores the route is bound by reading x from HBM
        b["route"]["frac"] = b["route"]["GB/s"] / hbm_peak
    b["route"]["frac_hbm"] = b["route"]["GB/s"] / hbm_peak
    b["dispatch"]["frac"] = b["dispatch"]["GB/s"] / hbm_peak
    b["gate_up"]["frac"] = b["gate_up"]["TFLOP/s"] / bf16_peak
    if "down_combine" in kms:
        ms = kms["down_combine"]
        # the fused launch writes y (2d B per token) instead of the shared output, and reads each
        # real slot's ys row (2d B) from L2 or HBM: those are the combine's bytes inside it
        b["down_combine"] = {"ms": ms, "bound": "tensor", "TFLOP/s": flops_dn / (ms * 1e9),
                             "frac": flops_dn / (ms * 1e9) / bf16_peak,
                             "combine_bytes": 2.0 * d * R + 2.0 * d * T}
        ffn_ms = kms["gate_up"] + ms
    else:
        b["down"] = {"ms": kms["down"], "bound": "tensor", "TFLOP/s": flops_dn / (kms["down"] * 1e9)}
        b["down"]["frac"] = b["down"]["TFLOP/s"] / bf16_peak
        b["combine"] = {"ms": kms["combine"], "bound": "hbm", "GB/s": bytes_combine / (kms["combine"] * 1e6)}
        b["combine"]["frac"] = b["combine"]["GB/s"] / hbm_peak
        ffn_ms = kms["gate_up"] + kms["down"]
    ffn_tflops = (6.0 * d * F * R + 6.0 * d * Fs * T) / (ffn_ms * 1e9)
    return b, ffn_tflops, flops_gu


def measure_per_config(args, names, dev, flush, peaks):
    """Forward-only measurement of further workloads (one at a time, buffers freed between):
    median step time over `steps` timed forwards, real slots per second, stage times."""
    import torch
    from token_choice_routing_b200 import inputs as I
    from token_choice_routing_b200.layer import MoENullLayer, bf16_tensor
    res = {}
    steps, warmup = max(3, min(args.steps, 10)), max(3, min(args.warmup, 5))
    for name in names:
        cfg = I.CONFIGS[name]
        inp = I.make_inputs(cfg)
        layer = MoENullLayer.from_inputs(inp, dev, router=args.router, ffn=args.ffn)
        x = bf16_tensor(inp.x, dev)
        tnb = None if inp.tok_null_bias is None else torch.from_numpy(inp.tok_null_bias).to(dev)
        out = layer.alloc(cfg.T, logits=False, xs=not args.gather, combine=args.combine)
        ms = timed_events(lambda: layer.forward(x, tnb, out), steps, warmup, flush)
        R = int(out["offsets"][-1].item())
        kms = forward_stage_ms(layer, layer.dims(cfg.T), x, tnb, out, flush, 9)  # median of 9 passes
        b, ffn_tflops, _ = forward_figures(cfg, R, kms, peaks, args, out)
        med = statistics.median(ms)
        res[name] = {"T": cfg.T, "K": cfg.K, "M": cfg.M, "rho": cfg.rho, "real_slots_per_step": R,
                     "ms_per_step_median": med, "ms_per_step_mean": sum(ms) / len(ms), "steps": steps,
                     "value": R / (med * 1e-3), "tokens_per_s": cfg.T / (med * 1e-3),
                     "ffn_tflops_real_rows": ffn_tflops,
                     "kernels": {k: {kk: vv for kk, vv in v.items() if kk in ("ms", "frac", "frac_hbm", "GB/s")}
                                 for k, v in b.items()}}
        del layer, out, x, tnb, inp
        torch.cuda.empty_cache()
    sw = [n for n in names if n.startswith("sweep_")]
    if len(sw) > 1:
        base = res[sw[0]]["ms_per_step_median"]
        res["sweep_time_vs_rho1"] = {n: res[n]["ms_per_step_median"] / base for n in sw}
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="skew",
                    help="headline workload (default: skew, the largest single-GPU workload)")
    ap.add_argument("--router", default="tensor", choices=["tensor", "fp32_cores"],
                    help="router product on the tensor cores (default) or the fp32 CUDA cores")
    ap.add_argument("--ffn", default="auto", choices=["auto", "single", "pair"],
                    help="expert GEMMs on single-CTA tiles, CTA pairs where the shape allows, or auto "
                         "(default: pairs from 65536 tokens per call)")
    ap.add_argument("--gather", action="store_true",
                    help="no xs copy: gate/up gathers the routed rows of x by TMA (default: dispatch copies them)")
    ap.add_argument("--combine", default="inplace", choices=["inplace", "separate", "fused"],
                    help="inplace (default): the down GEMM writes the shared expert's output into y and "
                         "the combine adds the routed rows there; separate: its own buffer; fused: the "
                         "combine inside the down GEMM's shared-expert tiles")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward-pass measurement")
    ap.add_argument("--no-per-config", action="store_true", help="skip the forward-only per_config workloads")
    ap.add_argument("--e2e-chunk", type=int, default=16384,
                    help="tokens per chunk of the host-buffer forward that e2e times")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target oracle time of the cpu_baseline")
    ap.add_argument("--cpu-steps", type=int, default=3, help="oracle steps of the cpu_baseline")
    ap.add_argument("--ref-step-seconds", type=float, default=2.0, help="oracle seconds per reference step")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import numpy as np
    import torch
    import torch.distributed as dist

    from token_choice_routing_b200 import binding as B
    from token_choice_routing_b200 import inputs as I
    from token_choice_routing_b200.dist import allreduce_aux_sums, dp_forward
    from token_choice_routing_b200.layer import MoENullLayer, bf16_tensor, chunk_bounds

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    assert world == args.gpus or world == 1, "launch with torchrun for --gpus > 1"

    cfg = I.CONFIGS[args.config]
    inp = I.make_inputs(cfg)
    layer = MoENullLayer.from_inputs(inp, dev, router=args.router, ffn=args.ffn)
    x = bf16_tensor(inp.x, dev)
    tnb = None if inp.tok_null_bias is None else torch.from_numpy(inp.tok_null_bias).to(dev)
    T = cfg.T
    out = layer.alloc(T, logits=False, xs=not args.gather, combine=args.combine)
    dm = layer.dims(T)
    nsum = B.aux_sums_count(dm)
    sums = torch.zeros(nsum, dtype=torch.float64, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        if world == 1:
            layer.forward(x, tnb, out)
        else:
            dp_forward(layer, x, tnb, out, sums)

    # one forward, plus the aux sums and their finalize when data parallel
    # (with the fp32 CUDA-core router its per-call weight transpose takes the header clear's place)
    kernels_per_step = FWD_LAUNCHES - (1 if args.combine == "fused" else 0) + (2 if world > 1 else 0)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    st = B.get_device_status(out["workspace"])
    if st != B.OK:
        raise SystemExit(f"device status after warm-up: {B.status_string(st)}")

    with ClockSampler(local) as clk:
        step_ms = timed_events(step, args.steps, 0, flush, sync_before=dist.barrier if world > 1 else None)
    if world > 1:
        dist.barrier()
    total_ms = sum(step_ms)
    med_ms = statistics.median(step_ms)
    if world > 1:
        t = torch.tensor([total_ms, med_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms, med_ms = float(t[0].item()), float(t[1].item())
    R = int(out["offsets"][-1].item())
    value = world * R * args.steps / (total_ms * 1e-3)
    st = B.get_device_status(out["workspace"])
    if st != B.OK:
        raise SystemExit(f"device status after timing: {B.status_string(st)}")

    # ---- the same forward replayed from a CUDA graph (one GPU): no host launch work per step,
    # which is what bounds decode-sized steps; same buffers, same L2 flush between steps
    graph = None
    if world == 1:
        y_eager = out["y"].clone()
        try:
            g = layer.capture_forward(x, tnb, out)
        except RuntimeError as e:  # a capture the runtime refuses: report it, keep the rest of the line
            g = None
            graph = {"unavailable": f"CUDA graph capture failed: {e}"[:300]}
            torch.cuda.synchronize()
        if g is not None:
            with ClockSampler(local) as g_clk:  # it runs after the eager steps: the power cap may differ
                g_ms = timed_events(g.replay, args.steps, args.warmup, flush)
            torch.cuda.synchronize()
            if not torch.equal(out["y"], y_eager) or B.get_device_status(out["workspace"]) != B.OK:
                raise SystemExit("graph replay: y differs from the eager forward's, or the device status is set")
            graph = {"value": R * args.steps / (sum(g_ms) * 1e-3), "unit": UNIT,
                     "ms_per_step": sum(g_ms) / args.steps, "ms_per_step_median": statistics.median(g_ms),
                     "what": "the forward captured once in a CUDA graph (torch.cuda.graph) and replayed",
                     "clocks": g_clk.summary()}
        del g, y_eager

    # ---- per-kernel breakdown (separately timed passes, same launches, CUDA events between them);
    # the SM clock is sampled here too: under the 1000 W cap it can settle lower than in the step loop
    with ClockSampler(local) as stage_clk:
        kms = forward_stage_ms(layer, dm, x, tnb, out, flush, max(5, min(args.steps, 11)))
    peaks, peak_kind = load_peaks()
    breakdown, ffn_tflops, flops_gu = forward_figures(cfg, R, kms, peaks, args, out)
    bf16_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    d, F, Fs = cfg.d, cfg.F, cfg.F_shared

    achieved = breakdown["gate_up"]["TFLOP/s"]
    pair = (args.ffn == "pair" or (args.ffn == "auto" and T >= MoENullLayer.PAIR_MIN_TOKENS)) \
        and cfg.F % 128 == 0 and cfg.F_shared % 128 == 0
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    roofline = {"kernel": "grouped gate/up SwiGLU GEMM (tcgen05, %s)" % ("CTA pairs" if pair else "single CTA"),
                "bound": "tensor", "achieved": achieved,
                "peak": bf16_peak, "unit": "TFLOP/s", "frac": achieved / bf16_peak,
                "peak_kind": f"{peak_kind} bf16 burst",
                # context: the kernel is timed inside back-to-back forwards, where the power cap
                # applies; against the sustained bf16 figure
                "peak_sustained": sustained, "frac_of_sustained": achieved / sustained,
                "stage_clocks": stage_clk.summary(),
                "traffic": None if args.gather else recorded_gate_up_traffic(cfg.name, pair),
                "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                "flops_per_launch": flops_gu, "ms_per_launch": kms["gate_up"]}

    if cfg.name.startswith("decode"):
        # a few rows per expert: the gate/up GEMM streams the weights of the experts that some
        # token chose (the others are never read), so its bound is HBM on those bytes
        used = int((out["counts"] > 0).sum().item())
        bytes_gu = (2.0 * 2 * F * d * used + 2.0 * 2 * Fs * d + 2.0 * d * (R + T) + 2.0 * F * R + 2.0 * Fs * T)
        gbs = bytes_gu / (kms["gate_up"] * 1e6)
        roofline = {"kernel": "grouped gate/up SwiGLU GEMM (weight streaming, tcgen05)", "bound": "hbm",
                    "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                    "peak_kind": f"{peak_kind} HBM copy", "traffic": None, "bytes_per_launch": bytes_gu,
                    "experts_used": used, "ms_per_launch": kms["gate_up"]}

    # ---- end to end through the public API with host buffers: every step copies x (and the
    # per-token null offsets) in from pinned host memory and y, the losses and the slot counts back
    # to pinned host memory; the layer's host forward runs in token chunks so the copies in and
    # out overlap each other and the compute
    x_pin = torch.from_numpy(np.ascontiguousarray(inp.x).view(np.int16)).view(torch.bfloat16).pin_memory()
    tnb_pin = None if inp.tok_null_bias is None else torch.from_numpy(inp.tok_null_bias).pin_memory()
    y_pin = torch.empty((T, d), dtype=torch.bfloat16).pin_memory()
    loss_pin = torch.empty(2, dtype=torch.float32).pin_memory()
    cext_pin = torch.empty(out["counts_ext"].numel(), dtype=torch.int32).pin_memory()
    chunk = min(T, args.e2e_chunk)
    pipe = layer.alloc_host_pipeline(chunk, nsets=3)

    def e2e_step():
        st = layer.forward_host(x_pin, y_pin, pipe, tnb_pin, reduce_sums=allreduce_aux_sums if world > 1 else None)
        loss_pin.copy_(st["losses"], non_blocking=True)
        cext_pin.copy_(st["counts_ext"], non_blocking=True)

    e2e_ms = timed_events(e2e_step, args.steps, args.warmup, flush, sync_before=dist.barrier if world > 1 else None)
    if world > 1:
        dist.barrier()
    e2e_total = sum(e2e_ms)
    if world > 1:
        t = torch.tensor([e2e_total], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_total = float(t.item())
    torch.cuda.synchronize()
    if not torch.equal(y_pin.to(dev), out["y"][:T]):
        raise SystemExit("e2e: the y copied back differs from the device forward's y")
    h2d = x_pin.numel() * 2 + (0 if tnb_pin is None else tnb_pin.numel() * 4)
    e2e = {"value": world * R * args.steps / (e2e_total * 1e-3), "unit": UNIT,
           "h2d_bytes_per_step": int(h2d),
           "d2h_bytes_per_step": int(y_pin.numel() * 2 + 4 * loss_pin.numel() + 4 * cext_pin.numel()),
           "ms_per_step": e2e_total / args.steps, "ms_per_step_median": statistics.median(e2e_ms),
           "chunk_tokens": chunk, "chunks_per_step": len(chunk_bounds(T, chunk)),
           "launches_per_step": (FWD_LAUNCHES + 1) * len(chunk_bounds(T, chunk)) + 1}
    del x_pin, y_pin, pipe

    backward = None
    if not args.no_backward and world == 1 and not args.gather:
        backward = measure_backward(args, cfg, layer, x, tnb, flush, peaks, peak_kind)

    per_config = None
    if world == 1 and not args.no_per_config:
        del layer, out, x, tnb
        torch.cuda.empty_cache()
        per_config = measure_per_config(args, [n for n in PER_CONFIG if n != cfg.name], dev, flush, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        S = calibrate_sample(inp, args.cpu_seconds / max(1, args.cpu_steps))
        per_step, Rs, stages = oracle_steps(inp, S, max(1, args.cpu_steps))
        cpu = {"value": Rs / sum(per_step), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{len(sample_tokens(T, S))} of {T} tokens spread evenly over the batch, "
                         f"{len(per_step)} full oracle forwards ({sum(per_step):.1f} s)",
               "step_s": per_step, "stage_s_median": stages}

    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "ms_per_step_median": med_ms,
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 tokens, N(0,1/fan_in) bf16 weights, fp32 router)",
            "config": workload_config(cfg, args),
            "real_slots_per_step": R, "tokens_per_s": world * T * args.steps / (total_ms * 1e-3),
            "ffn_tflops_real_rows": ffn_tflops, "ffn_frac_of_bf16_peak": ffn_tflops / bf16_peak,
            # the FLOPs behind it: routed real slots and the shared expert's T rows (one launch each GEMM)
            "ffn_gflop_per_step": {"routed": 6.0 * cfg.d * cfg.F * R / 1e9,
                                   "shared": 6.0 * cfg.d * cfg.F_shared * cfg.T / 1e9},
            "roofline": roofline, "kernels": breakdown, "cpu_baseline": cpu, "e2e": e2e, "graph": graph,
            "gpu_launches": kernels_per_step * args.steps,
            "clocks": clk.summary(),
            "backward": backward,
            "per_config": per_config,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
