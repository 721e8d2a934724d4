"""The benchmark's reference arm (the fp64 oracle on the host cores) runs on
the CPU: check the JSON line it prints against the benchmark contract."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True,
                       text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


def test_reference_arm_line():
    d = run_bench("--impl", "reference", "--steps", "1", "--warmup", "3", "--workload", "wan1.3b_framewise_infer")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["dtype"] == "f64" and d["value"] > 0
    assert d["config"]["workload"] == "wan1.3b_framewise_infer"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_warmup_below_three_is_refused():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"], capture_output=True,
                       text=True, timeout=120, cwd=ROOT)
    assert r.returncode != 0 and "warmup" in r.stderr


def test_traffic_key_ignores_comments_but_not_code():
    """The DRAM-traffic tables are keyed by a hash of the kernel's code: a
    comment edit keeps the key, a code edit changes it."""
    import bench
    src = {"a.cu": "int f(int x) { // double it\n  return 2 * x; /* twice */ }\n",
           "kernels.h": "struct P {\n  int n;  // rows\n};\n"}
    files = ["a.cu", "struct P"]
    base = bench.kernel_sources_hash(files, src.get)
    recommented = {"a.cu": "// doubles its argument\nint f(int x) {\n  return 2 * x;\n}\n",
                   "kernels.h": "struct P {\n  int n;\n};\n"}
    assert bench.kernel_sources_hash(files, recommented.get) == base
    changed = dict(src, **{"a.cu": src["a.cu"].replace("2 * x", "3 * x")})
    assert bench.kernel_sources_hash(files, changed.get) != base
    changed = dict(src, **{"kernels.h": "struct P {\n  long n;\n};\n"})
    assert bench.kernel_sources_hash(files, changed.get) != base
