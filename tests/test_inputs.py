"""The seeded input generator: determinism, bf16 rounding, stored calibration."""
import json
import os

import numpy as np
import pytest
import torch

from token_choice_routing_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_same_seed_same_inputs():
    cfg = I.CONFIGS["tiny"]
    a, b = I.make_inputs(cfg), I.make_inputs(cfg)
    for f in ("x", "w_router", "bias", "w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f


def test_shapes_and_scales():
    cfg = I.CONFIGS["tiny"]
    a = I.make_inputs(cfg)
    T, d, N, F, Fs = cfg.T, cfg.d, cfg.N, cfg.F, cfg.F_shared
    assert a.x.shape == (T, d) and a.x.dtype == np.uint16
    assert a.w_router.shape == (N + 1, d) and a.w_router.dtype == np.float32
    assert a.w_gate.shape == (N, F, d) and a.w_down.shape == (N, d, F)
    assert a.ws_gate.shape == (Fs, d) and a.ws_down.shape == (d, Fs)
    x = I.bf16_to_f32(a.x)
    assert abs(x.std() - 1.0) < 0.05
    assert abs(I.bf16_to_f32(a.w_gate).std() * np.sqrt(d) - 1.0) < 0.05
    assert abs(I.bf16_to_f32(a.w_down).std() * np.sqrt(F) - 1.0) < 0.05


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(1)
    v = (rng.standard_normal(100000) * 37).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(I.bf16_round(v), ref)
    assert np.array_equal(I.bf16_to_f32(ref), torch.from_numpy(v).to(torch.bfloat16).float().numpy())


def test_null_bias_table_is_the_calibration_output():
    d = json.load(open(os.path.join(GOLDEN, "null_bias.json")))
    assert set(d) == set(I.NULL_BIAS)
    for k, v in d.items():
        assert I.NULL_BIAS[k] == v["null_bias"]
        assert abs(v["mean_real"] - v["target"]) < 1e-3


def test_calibration_reproduces_tiny():
    import importlib.util
    spec = importlib.util.spec_from_file_location("cal", os.path.join(GOLDEN, "calibrate_null_bias.py"))
    cal = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(cal)
    b, r, target = cal.calibrate(I.CONFIGS["tiny"])
    assert b == I.NULL_BIAS["tiny"]


def test_skew_layout():
    cfg = I.small_config("sk", T=64, d=16, N=8, F=16, F_shared=16, K=4, M=4, skew=True, seqs=2)
    a = I.make_inputs(cfg)
    L = 32
    low = int(round(0.6 * L))
    pos = np.arange(64) % L
    assert np.array_equal(a.tok_null_bias, np.where(pos < low, 1.5, 0.0).astype(np.float32))
    x = I.bf16_to_f32(a.x)
    assert x[pos < low].std() < 0.5 < x[pos >= low].std()
    assert a.bias[0] == 0.0 and a.bias[1] == pytest.approx(-1.1 * np.log(2.0), rel=1e-6)
    assert a.bias[-1] == 0.0
