"""Seeded synthetic workloads for the null-expert MoE layer.

This module only draws numbers. It holds none of the layer's arithmetic: no
router product, no softmax, no selection. Both the CUDA path's tests/bench and
the CPU oracle's tests take their inputs from here, and nothing else is shared
between the two.

Recipe (one numpy SeedSequence per tensor, spawned from SeedSequence(20260000 +
config id) in the fixed order of ``_STREAMS``; bf16 tensors are drawn in row
chunks of 2^22 elements, chunk c from the tensor's c-th child PCG64 stream):

* x ~ N(0, 1), drawn in fp32 and rounded to bf16 (round to nearest even).
* routed and shared expert weights ~ N(0, 1/fan_in), fan_in = d for gate/up and
  F (or F_shared) for down, rounded to bf16.
* router weight W_r ~ N(0, 1/d), fp32, shape [N+1, d]; row N is the null logit
  (Kilian et al., "Improving MoE Compute Efficiency by Composing Weight and Data
  Sparsity", review page, section 三 "Null Expert 机制": the router emits N+1
  logits, the last one for the null expert).
* router bias [N+1]: zero for real experts, and for the null logit a scalar
  that was calibrated (bisection on the oracle's fp64 logits) so that the mean
  number of real experts per token is close to rho*K with rho = N/(N+M).  The
  calibrated scalars live in ``NULL_BIAS`` below and are written by
  ``tests/golden/calibrate_null_bias.py``, which calls only the oracle.
* the skewed workload (the 16 x 8192 token batch) has, in each 8192-token
  sequence, a contiguous low-information span of round(0.6*8192) tokens at its
  start (x ~ 0.3*N(0,1), per-token null-logit offset +1.5) followed by dense
  tokens (x ~ N(0,1), offset 0), and a Zipf(1.1) real-expert bias
  b_i = -1.1*ln(i+1).  This stands in for the vision-then-text layout the
  paper's per-token compute figure shows (sciencestack page, Figure 5).
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Optional

import numpy as np

SEED_BASE = 20260000

# Order of the per-tensor sub-streams; never reorder (it would change inputs). New
# streams go at the end: the earlier ones keep their draws.
_STREAMS = ("x", "w_router", "w_gate", "w_up", "w_down",
            "ws_gate", "ws_up", "ws_down", "spans", "const_vectors", "dy")


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    config_id: int
    T: int
    d: int
    N: int
    F: int
    F_shared: int
    K: int
    M: int
    skew: bool = False
    seqs: int = 1
    bias_from: Optional[str] = None  # workload whose calibrated null bias this one uses
    C: int = 0  # MoE++ copy experts (router rows N+1 .. N+C)
    V: int = 0  # MoE++ constant experts (router rows N+C+1 .. N+C+V)

    @property
    def rho(self) -> float:
        return self.N / float(self.N + self.M)

    @property
    def router_rows(self) -> int:
        return self.N + 1 + self.C + self.V

    @property
    def seed(self) -> int:
        return SEED_BASE + self.config_id


# The five workloads (the sweep's four points get ids 30..33).
CONFIGS: Dict[str, LayerConfig] = {c.name: c for c in [
    LayerConfig("tiny", 0, T=256, d=128, N=8, F=64, F_shared=64, K=4, M=8),
    LayerConfig("qwen3_0p6b", 1, T=16384, d=1024, N=64, F=768, F_shared=768, K=4, M=64, seqs=8),
    LayerConfig("qwen3_1p7b", 2, T=16384, d=2048, N=64, F=1536, F_shared=1536, K=8, M=192, seqs=8),
    LayerConfig("sweep_k2_m0", 30, T=65536, d=2048, N=64, F=1536, F_shared=1536, K=2, M=0, seqs=8),
    LayerConfig("sweep_k3_m32", 31, T=65536, d=2048, N=64, F=1536, F_shared=1536, K=3, M=32, seqs=8),
    LayerConfig("sweep_k4_m64", 32, T=65536, d=2048, N=64, F=1536, F_shared=1536, K=4, M=64, seqs=8),
    LayerConfig("sweep_k8_m192", 33, T=65536, d=2048, N=64, F=1536, F_shared=1536, K=8, M=192, seqs=8),
    LayerConfig("skew", 4, T=131072, d=2048, N=64, F=1536, F_shared=1536, K=8, M=64, skew=True, seqs=16),
    # Small-batch (decode-sized) forwards with the 0.6B and 1.7B layers' weights: same
    # config ids, so the router and expert weights are the same draws; ~T rho K / N rows
    # per expert, so the expert GEMMs stream weights (experts no token chose are skipped).
    LayerConfig("decode_0p6b", 1, T=64, d=1024, N=64, F=768, F_shared=768, K=4, M=64, bias_from="qwen3_0p6b"),
    LayerConfig("decode_1p7b", 2, T=64, d=2048, N=64, F=1536, F_shared=1536, K=8, M=192,
                bias_from="qwen3_1p7b"),
    # The 0.6B layer with MoE++ copy and constant experts beside the null expert: the same
    # draws for x, the expert weights and the first N+1 router rows (rows are drawn in order).
    LayerConfig("moepp_0p6b", 1, T=16384, d=1024, N=64, F=768, F_shared=768, K=4, M=64, seqs=8,
                bias_from="qwen3_0p6b", C=4, V=4),
]}

# Null-logit bias per workload, from tests/golden/calibrate_null_bias.py (oracle
# routing on fp64 logits, 60 bisection steps on [-30, 30]).  Target mean real
# count: rho*K = 2 for every workload that has null copies.  The sweep's M=0
# point and the skewed workload take no calibrated bias.
NULL_BIAS: Dict[str, float] = {
    "qwen3_0p6b": 1.9099643230438232,
    "qwen3_1p7b": 2.3808422088623047,
    "sweep_k3_m32": 1.547541856765747,
    "sweep_k4_m64": 1.909210443496704,
    "sweep_k8_m192": 2.3533687591552734,
    "tiny": 0.7090700268745422,
}


SKEW_LOW_INFO_FRACTION = 0.6
SKEW_LOW_INFO_SCALE = 0.3
SKEW_NULL_OFFSET = 1.5
SKEW_ZIPF_S = 1.1


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


_CHUNK = 1 << 22   # elements per independently seeded chunk (fixed: part of the recipe)
_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1)))
    return _POOL


def _streams(seed: int) -> Dict[str, np.random.SeedSequence]:
    children = np.random.SeedSequence(seed).spawn(len(_STREAMS))
    return dict(zip(_STREAMS, children))


def _normal_bf16(ss: np.random.SeedSequence, shape, scale, row_scale=None) -> np.ndarray:
    """N(0, scale^2) draws in fp32, rounded to bf16 (uint16 bits).

    The tensor is cut into row chunks of about ``_CHUNK`` elements; chunk c is
    drawn from the c-th child of ``ss`` (so the result does not depend on how
    many threads draw it). ``row_scale`` (one float per leading-axis row)
    multiplies each row.
    """
    out = np.empty(shape, dtype=np.uint16)
    flat = out.reshape(-1)
    rows = shape[0]
    per = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    step = max(1, _CHUNK // max(per, 1))
    starts = list(range(0, rows, step))
    kids = ss.spawn(len(starts))

    def work(i):
        r0 = starts[i]
        r1 = min(rows, r0 + step)
        g = np.random.Generator(np.random.PCG64(kids[i]))
        v = g.standard_normal((r1 - r0) * per, dtype=np.float32)
        if scale != 1.0:
            v *= np.float32(scale)
        if row_scale is not None:
            v = (v.reshape(r1 - r0, per) * row_scale[r0:r1, None].astype(np.float32)).reshape(-1)
        flat[r0 * per:r1 * per] = bf16_round(v)

    list(_pool().map(work, range(len(starts))))
    return out


@dataclasses.dataclass
class LayerInputs:
    """Host-side inputs of one workload. bf16 tensors are uint16 bit arrays."""
    cfg: LayerConfig
    x: np.ndarray              # [T, d] bf16 bits
    w_router: np.ndarray       # [N+1, d] float32
    bias: np.ndarray           # [N+1] float32
    tok_null_bias: Optional[np.ndarray]  # [T] float32 or None
    w_gate: np.ndarray         # [N, F, d] bf16 bits
    w_up: np.ndarray           # [N, F, d] bf16 bits
    w_down: np.ndarray         # [N, d, F] bf16 bits
    ws_gate: np.ndarray        # [F_s, d] bf16 bits
    ws_up: np.ndarray          # [F_s, d] bf16 bits
    ws_down: np.ndarray        # [d, F_s] bf16 bits
    const_vectors: Optional[np.ndarray] = None  # [V, d] bf16 bits (MoE++ constant experts)


def make_inputs(cfg: LayerConfig, *, T: Optional[int] = None, weights: bool = True,
                null_bias: Optional[float] = None) -> LayerInputs:
    """Draw the seeded inputs of ``cfg``.

    ``T`` overrides the token count (the first T rows of a draw of the full
    stream are NOT guaranteed equal to a smaller draw; use it for test sizes).
    ``weights=False`` leaves the expert weights as empty arrays (routing-only
    tests).  ``null_bias`` overrides the calibrated null-logit bias.
    """
    T = cfg.T if T is None else T
    s = _streams(cfg.seed)
    d, N, F, Fs = cfg.d, cfg.N, cfg.F, cfg.F_shared

    tok_null_bias = None
    if cfg.skew:
        L = max(1, T // cfg.seqs) if T >= cfg.seqs else T
        low = int(round(SKEW_LOW_INFO_FRACTION * L))
        pos = np.arange(T) % L
        is_low = pos < low
        row_scale = np.where(is_low, np.float32(SKEW_LOW_INFO_SCALE), np.float32(1.0))
        x = _normal_bf16(s["x"], (T, d), 1.0, row_scale=row_scale)
        tok_null_bias = np.where(is_low, np.float32(SKEW_NULL_OFFSET), np.float32(0.0)).astype(np.float32)
    else:
        x = _normal_bf16(s["x"], (T, d), 1.0)

    g_r = np.random.Generator(np.random.PCG64(s["w_router"]))
    w_router = (g_r.standard_normal((cfg.router_rows, d)) / math.sqrt(d)).astype(np.float32)

    bias = np.zeros(cfg.router_rows, dtype=np.float32)
    if cfg.skew:
        bias[:N] = (-SKEW_ZIPF_S * np.log(np.arange(N, dtype=np.float64) + 1.0)).astype(np.float32)
    elif cfg.M > 0:
        nb = NULL_BIAS.get(cfg.bias_from or cfg.name, 0.0) if null_bias is None else null_bias
        bias[N] = np.float32(nb)

    if weights:
        w_gate = _normal_bf16(s["w_gate"], (N, F, d), 1.0 / math.sqrt(d))
        w_up = _normal_bf16(s["w_up"], (N, F, d), 1.0 / math.sqrt(d))
        w_down = _normal_bf16(s["w_down"], (N, d, F), 1.0 / math.sqrt(F))
        ws_gate = _normal_bf16(s["ws_gate"], (Fs, d), 1.0 / math.sqrt(d))
        ws_up = _normal_bf16(s["ws_up"], (Fs, d), 1.0 / math.sqrt(d))
        ws_down = _normal_bf16(s["ws_down"], (d, Fs), 1.0 / math.sqrt(Fs))
    else:
        e = np.zeros((0,), dtype=np.uint16)
        w_gate = w_up = w_down = ws_gate = ws_up = ws_down = e

    const_vectors = _normal_bf16(s["const_vectors"], (cfg.V, d), 0.5) if cfg.V else None
    return LayerInputs(cfg, x, w_router, bias, tok_null_bias,
                       w_gate, w_up, w_down, ws_gate, ws_up, ws_down, const_vectors)


def upstream_grad(cfg: LayerConfig, *, T: Optional[int] = None, scale: float = 1.0) -> np.ndarray:
    """Seeded upstream gradient dy of the layer output for the backward pass: N(0, scale^2)
    bf16 bits [T, d], from the config's own "dy" stream."""
    T = cfg.T if T is None else T
    return _normal_bf16(_streams(cfg.seed)["dy"], (T, cfg.d), scale)


def small_config(name: str = "small", *, T: int, d: int, N: int, F: int, F_shared: int,
                 K: int, M: int, config_id: int = 900, skew: bool = False,
                 seqs: int = 1, C: int = 0, V: int = 0) -> LayerConfig:
    """An ad-hoc configuration for tests (edge cases, ragged sizes)."""
    return LayerConfig(name, config_id, T=T, d=d, N=N, F=F, F_shared=F_shared, K=K, M=M,
                       skew=skew, seqs=seqs, C=C, V=V)
