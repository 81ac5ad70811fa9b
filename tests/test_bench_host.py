"""bench.py on the host: the reference arm's JSON line (the oracle timed on
the CPU) carries every key of the bench contract, and the source hash that
keys the recorded DRAM traffic ignores comments but not code."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_line_has_the_contract_keys():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "3", "--warmup", "3"],
                         cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["steps"] == 3 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["config"]["workload"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_kernel_source_sha_ignores_comments_only(tmp_path):
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    c = tmp_path / "c.cu"
    a.write_text("// header\n__global__ void k(int *p) {\n    p[0] = 1;  // one\n}\n")
    b.write_text("/* another\n   header */\n__global__ void k(int *p) {\n  p[0] = 1;\n}\n")
    c.write_text("// header\n__global__ void k(int *p) {\n    p[0] = 2;  // one\n}\n")
    assert bench.kernel_source_sha(str(a)) == bench.kernel_source_sha(str(b))
    assert bench.kernel_source_sha(str(a)) != bench.kernel_source_sha(str(c))
