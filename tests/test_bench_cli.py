"""bench.py's command line on the CPU: every documented mode is accepted, and the
reference arm (the fp64 oracle on the host cores, no GPU) prints one JSON line with
the keys the benchmark contract asks for."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args, timeout=300):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, capture_output=True,
                          text=True, timeout=timeout)


def test_help_lists_every_mode():
    r = _run("--help")
    assert r.returncode == 0, r.stderr
    for flag in ("--gpus", "--steps", "--warmup", "--impl", "--case", "--prefill", "--schedule", "--sessions",
                 "--configs", "--library", "--euler-sweep", "--hbm-kernels", "--no-cpu-baseline"):
        assert flag in r.stdout, flag


def test_reference_arm_line():
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-step-seconds", "0.5")
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["unit"] == "TFLOP/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "v02-640x368-unit-40L-4steps-hist64-40x128"
