"""CPU tests of the benchmark's host-side helpers: the source-pinned ncu traffic records and
the reference arm's JSON line shape (no GPU, no kernel launch)."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_traffic_record_is_used_only_with_matching_sources(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    digest = bench.gemm_source_digest(("kernel.cu",))
    prof = tmp_path / "prof.md"
    prof.write_text("# profile\n\ntraffic-record: workload=w1 kernel=gate_up dram_bytes_per_launch=123456 "
                    f"source_sha256={digest}\n"
                    "traffic-record: workload=w1 kernel=down dram_bytes_per_launch=777 source_sha256=deadbeef\n")
    assert bench.recorded_traffic("w1", "gate_up", "prof.md", ("kernel.cu",)) == 123456.0
    assert bench.recorded_traffic("w2", "gate_up", "prof.md", ("kernel.cu",)) is None       # other workload
    assert bench.recorded_traffic("w1", "down", "prof.md", ("kernel.cu",)) is None          # stale digest
    src.write_text("// kernel v2\n")                                                         # sources changed
    assert bench.recorded_traffic("w1", "gate_up", "prof.md", ("kernel.cu",)) is None
    assert bench.recorded_traffic("w1", "gate_up", "missing.md", ("kernel.cu",)) is None


def test_committed_records_parse():
    """The committed profiles carry well-formed records of known workloads."""
    from token_choice_routing_b200 import inputs as I
    n = 0
    for prof in (*bench.GEMM_PROFILES, bench.BWD_GEMM_PROFILE):
        if not os.path.exists(os.path.join(ROOT, prof)):
            continue
        lines = [l for l in open(os.path.join(ROOT, prof)) if l.startswith("traffic-record:")]
        n += len(lines)
        for l in lines:
            kv = dict(p.split("=", 1) for p in l.split()[1:])
            assert kv["workload"] in I.CONFIGS and int(kv["dram_bytes_per_launch"]) > 0
            assert len(kv["source_sha256"]) == 64
    assert n > 0


def test_token_sample_spreads_over_the_batch():
    """The oracle's timing sample takes tokens from every part of the batch (the skewed
    workload's low-information and dense spans alike)."""
    tok = bench.sample_tokens(131072, 1000)
    assert tok[0] == 0 and tok[-1] == 131071 and len(tok) == 1000
    low = (tok % 8192) < round(0.6 * 8192)   # the skewed workload's low-information spans
    assert abs(low.mean() - 0.6) < 0.01
    assert bench.sample_tokens(10, 50).tolist() == list(range(10))


def test_reference_arm_json_line():
    """bench.py --impl reference times the oracle on the host and prints one JSON line with the
    contract's keys (a tiny sample keeps this quick)."""
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "tiny", "--steps", "1",
                        "--warmup", "0", "--ref-step-seconds", "0.2"], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "impl", "cpu_baseline", "e2e", "config"):
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
