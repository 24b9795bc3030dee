"""The benchmark's reference arm (the fp64 oracle, timed on the host cores):
one JSON line per run with the contract's fields, in each step mode, on CPU;
and the oracle pool behind it."""

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


@pytest.mark.parametrize("mode", ["decode", "spec", "prefill", "strided"])
def test_reference_arm_line(mode):
    import bench
    from syngen import configs as C
    j = _run("--mode", mode, "--chunk", "4")
    assert j["impl"] == "reference" and j["unit"] == "steps/s" and j["value"] > 0
    assert j["higher_is_better"] is True and j["steps"] == 2 and j["warmup"] == 1
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == j["value"]
    assert cb["cores"] >= 1 and cb["extrapolated_from_units"] >= 1 and "extrapolated" in cb["sample"]
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["value"] == j["value"]
    # the same config object as the native arm's line for this workload and mode
    w = C.get_workload("tiny")
    chunk = 4 if mode != "decode" else 1
    _, _, flush = bench.step_bytes_model(w, mode, chunk, w.T0)
    assert j["config"] == bench.workload_config(w, mode, chunk, 1, flush)
    if mode != "decode":
        assert {"spec": "4 x (decode + append)", "prefill": "4 appends + decode",
                "strided": "strided selection (stride 4) + decode + append"}[mode] in cb["sample"]


def test_oracle_pool_keeps_timing_past_its_prepared_tokens():
    """A unit holds 256 prepared tokens; a sample longer than they last starts
    the unit again from T0, so every sample times work and the rate holds."""
    import bench
    from syngen import configs as C
    w = C.get_workload("tiny")
    pool = bench.OraclePool(w, max_appends=16)
    try:
        s1, n1 = pool.sample(1.2)
        s2, n2 = pool.sample(0.3)
    finally:
        pool.close()
    assert n1 > 16 * pool.workers and n2 > 0
    assert 0 < s1 < 1 and 0 < s2 < 1
    assert 0.2 < s1 / s2 < 5
