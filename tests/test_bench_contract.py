"""bench.py's output contract, checked on CPU: the reference arm (the oracle
on the host's cores) prints one JSON line with the keys the contract names,
and the kernel-code hash that keys the committed DRAM counters ignores
comment-only edits."""
import json
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def run_reference(*extra):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
           "single_96_64x64", "--steps", "1", "--warmup", "0", "--cpu-seconds", "1", *extra]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout[-2000:]
    return json.loads(lines[0])


def test_reference_arm_prints_one_complete_json_line():
    d = run_reference()
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 0
    assert d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["value"] > 0 and d["unit"] == "TOPS"
    assert d["config"]["workload"] == "single_96_64x64"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    # the time per step is the inverse of the rate on the workload's ops
    ops = 2.0 * 96 * 96 * 9 * 64 * 64
    assert abs(ops / (d["value"] * 1e12) * 1e3 - d["ms_per_step"]) <= 1e-6 * d["ms_per_step"]


def test_kernel_code_hash_ignores_comments():
    import bench
    src = "int a; // one\n/* two\n   lines */ int b;\n\n  // only a comment\nint c;  \n"
    assert bench.code_only(src) == "int a;\n int b;\nint c;"
    h = bench.conv_source_hash()
    assert re.fullmatch(r"[0-9a-f]{16}", h)
