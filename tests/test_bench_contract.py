"""The JSON line bench.py prints, checked on CPU through its reference arm (the float64 oracle on
a bounded row sample), and the ways bench.py refuses to produce a number: a non-zero rank of the
reference arm does no work, too few warm-up steps are rejected, and the device arm without a
CUDA device exits non-zero instead of falling back to the CPU."""
import json
import os
import subprocess
import sys

import numpy as np
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


def test_clock_summary_uses_the_samples_stamped_inside_the_timed_region():
    import datetime
    sys.path.insert(0, ROOT)
    import bench
    t0 = datetime.datetime(2026, 1, 2, 3, 4, 5, 0)

    def stamp(ms):
        return (t0 + datetime.timedelta(milliseconds=ms)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]

    clk = bench.ClockSampler(0)
    # idle before and after (1965 MHz, 0 % busy), power-capped inside (1600-1700 MHz)
    clk.lines["stamped"] = (
        [f"{stamp(ms)}, 1965, 1965, 200.0, 0x0000000000000001, 0" for ms in (0, 10, 20)] +
        [f"{stamp(ms)}, {mhz}, 1965, 990.0, 0x0000000000000004, 0"
         for ms, mhz in ((40, 1600), (50, 1650), (60, 1700))] +
        [f"{stamp(ms)}, 1965, 1965, 210.0, 0x0000000000000001, 0" for ms in (90, 100)])
    clk.lines["plain"] = ["1965, 1965, 200.0, 0x0000000000000001, 0"]
    clk.t_begin = (t0 + datetime.timedelta(milliseconds=35)).timestamp()
    clk.t_end = (t0 + datetime.timedelta(milliseconds=65)).timestamp()
    s = clk.summary()
    assert s["sm_mhz"] == 1650 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    assert s["samples"] == 8 and s["samples_in_timed_region"] == 3 and s["from"] == "timed region"
    assert s["power_w_max"] == 990.0
    # a region between two samples falls back to busy samples, then to all of them
    clk.t_begin = clk.t_end = (t0 + datetime.timedelta(milliseconds=75)).timestamp()
    s = clk.summary()
    assert s["from"] == "all samples" and s["samples_in_timed_region"] == 0
    # without stamped samples the unstamped poller's are used
    clk.lines["stamped"] = []
    clk.lines["plain"] = ["1700, 1965, 900.0, 0x0000000000000004, 80",
                          "1965, 1965, 200.0, 0x0000000000000001, 0"]
    s = clk.summary()
    assert s["sm_mhz"] == 1700 and s["from"] == "utilisation >= 50 %" and s["samples"] == 2


def test_reference_split_computes_what_one_oracle_call_does():
    """The reference arm builds the chunk's keys once and evaluates sampled rows per step
    (bench.OracleRows); for the same rows that is exactly oracle.chunk_step's result."""
    import bench
    import oracle
    from mla_latent_kv_attn_b200 import inputs
    cfg = inputs.small_bf16_config()
    sample = bench.OracleSample(cfg)
    prep = bench.OracleRows(sample)
    rows = inputs.sample_rows(cfg.n_q, 37, tag=5)
    got = prep.evaluate(rows)
    ref = oracle.chunk_step(sample.d, sample.lw, sample.x, sample.win,
                            cfg.first_frame(cfg.measured_chunk), rows=rows, append=False)
    for k in ("o", "o_lat", "lse"):
        assert np.array_equal(got[k], ref[k]), k
