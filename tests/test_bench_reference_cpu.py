"""The benchmark's reference arm (the fp64 oracle, timed on the host cores):
one JSON line per run with the contract's fields, in each step mode, on CPU."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*extra):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
           "--steps", "2", "--warmup", "1", "--cpu-sample-seconds", "0.4", *extra]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


@pytest.mark.parametrize("mode", ["decode", "spec", "prefill"])
def test_reference_arm_line(mode):
    j = _run("--mode", mode, "--chunk", "4")
    assert j["impl"] == "reference" and j["unit"] == "steps/s" and j["value"] > 0
    assert j["higher_is_better"] is True and j["steps"] == 2 and j["warmup"] == 1
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] == j["value"]
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["value"] == j["value"]
    assert j["config"]["workload"] == "tiny"
    if mode != "decode":
        assert j["config"]["mode"] == mode and j["config"]["chunk"] == 4
        assert ("4 x (decode + append)" if mode == "spec" else "4 appends + decode") in j["cpu_baseline"]["sample"]
