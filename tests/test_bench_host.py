"""Host side of bench.py on CPU: the reference arm's JSON line (the fp64 oracle timed on this host)
and the lookup of captured DRAM traffic, which must ignore a capture of another kernel source."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
                          "--cpu-seconds", "0.5", "--workload", "tiny"],
                         cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"].startswith("tiny")
    import bench as b
    import workloads
    assert d["config"] == json.loads(json.dumps(b.run_config(workloads.WORKLOADS["tiny"], 1)))  # same as the GPU arm


def test_traffic_lookup_requires_the_captured_source(tmp_path, monkeypatch):
    sha = bench.file_sha(bench.GEMM_KERNEL_SRC)
    f = tmp_path / "traffic.txt"
    f.write_text("# workload kernel bytes_per_launch source_sha\n"
                 f"image encode_flow_kernel 123456 {sha}\n"
                 "image other_kernel 7 " + sha + "\n"
                 "packed encode_flow_kernel 999 0000000000000000\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.read_traffic("image", "encode_flow_kernel") == 123456.0
    assert bench.read_traffic("packed", "encode_flow_kernel") is None     # captured from other source
    assert bench.read_traffic("offline", "encode_flow_kernel") is None    # never captured
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.txt"))
    assert bench.read_traffic("image", "encode_flow_kernel") is None
