"""The JSON line bench.py prints, checked on CPU through its reference arm (the float64 oracle on
a bounded row sample), and the ways bench.py refuses to produce a number: a non-zero rank of the
reference arm does no work, too few warm-up steps are rejected, and the device arm without a
CUDA device exits non-zero instead of falling back to the CPU."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args, env=None, timeout=600):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          env=e, capture_output=True, text=True, timeout=timeout)


def _json_lines(stdout):
    return [json.loads(l) for l in stdout.splitlines() if l.startswith("{")]


def test_reference_arm_prints_one_complete_line():
    r = _bench("--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-rows", "4")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    line = lines[0]
    sys.path.insert(0, ROOT)
    import bench
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC
    assert line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["n_gpus"] == 1 and line["steps"] == 1 and line["warmup"] == 3
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    assert line["vs_baseline"] is None
    assert line["dtype"] == "f64" and line["data"] == "synthetic"
    assert line["config"]["workload"] == "wan1.3b_b1_w6_c3"
    assert line["config"]["n_q"] == 4680 and line["config"]["keys_per_query"] == 14040
    assert line["ms_per_step"] > 0 and line["query_tokens_per_s"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert "4 sampled query rows" in cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    # value is the sampled work over the timed oracle time: 832 flop per (row, key, head)
    flops = 4 * 14040 * 12 * 2 * (224 + 192)
    assert line["value"] == pytest.approx(flops / (line["ms_per_step"] * 1e-3) / 1e12, rel=1e-6)


def test_reference_arm_other_ranks_exit_without_work():
    r = _bench("--impl", "reference", "--steps", "1", "--warmup", "3",
               env={"RANK": "1", "WORLD_SIZE": "2"}, timeout=120)
    assert r.returncode == 0
    assert _json_lines(r.stdout) == []


def test_fewer_than_three_warmup_steps_are_refused():
    r = _bench("--impl", "reference", "--steps", "1", "--warmup", "2", timeout=120)
    assert r.returncode != 0
    assert "--warmup must be >= 3" in r.stderr
    assert _json_lines(r.stdout) == []


def test_device_arm_without_a_gpu_fails_instead_of_falling_back():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    r = _bench("--steps", "1", "--warmup", "3", "--no-cpu-baseline", timeout=300)
    assert r.returncode != 0
    assert _json_lines(r.stdout) == []
