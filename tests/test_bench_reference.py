"""CPU tests of bench.py's reference arm (the oracle timed on host cores) and its JSON
contract, on small workloads; plus the host helpers that describe the CPU baseline.  No GPU
is used: the reference arm runs only the oracle."""

import contextlib
import io
import json

import bench

CONTRACT = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
            "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config")


def _run(argv):
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main(argv)
    assert rc in (0, None)
    lines = [x for x in buf.getvalue().splitlines() if x.startswith("{")]
    assert len(lines) == 1, buf.getvalue()
    return json.loads(lines[0])


def _check_line(d, workload):
    for k in CONTRACT:
        assert k in d, k
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["n_gpus"] == 1 and d["steps"] == 1
    assert d["vs_baseline"] is None and d["data"] == "synthetic"
    assert d["config"]["workload"] == workload
    cpu = d["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == d["value"] and cpu["unit"] == d["unit"]
    assert cpu["cores"] >= 1 and cpu["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_attention():
    d = _run(["--impl", "reference", "--workload", "tiny_causal", "--steps", "1",
              "--warmup", "0"])
    _check_line(d, "tiny_causal")
    assert d["higher_is_better"] is True and d["dtype"] == "f64"


def test_reference_arm_windowed():
    d = _run(["--impl", "reference", "--workload", "long_local_sym512", "--steps", "1",
              "--warmup", "0"])
    _check_line(d, "long_local_sym512")


def test_reference_arm_varlen():
    # packed sequences: the sample is drawn from the longest sequence, the config names the
    # packing
    d = _run(["--impl", "reference", "--workload", "varlen3", "--steps", "1", "--warmup", "0"])
    _check_line(d, "varlen3")
    assert d["config"]["num_seqs"] == 3 and d["config"]["total_tokens"] == 896
    assert d["config"]["max_seqlen"] == 512


def test_reference_arm_decode():
    d = _run(["--impl", "reference", "--workload", "decode_q4_l8k", "--steps", "1",
              "--warmup", "0"])
    _check_line(d, "decode_q4_l8k")
    assert d["unit"] == "GB/s"


def test_reference_arm_fp8():
    d = _run(["--impl", "reference", "--workload", "fp8_long_causal", "--steps", "1",
              "--warmup", "0"])
    _check_line(d, "fp8_long_causal")


def test_host_helpers():
    assert bench.oracle_threads() >= 1
    h = bench.host_cpus()
    assert h["logical_cores"] >= 1
    assert h["physical_cores"] is None or 1 <= h["physical_cores"] <= h["logical_cores"]


def test_clock_sampler_without_gpu_returns_nothing_or_a_summary():
    s = bench.ClockSampler(0)
    out = s.stop()
    assert out is None or {"sm_mhz", "sm_max_mhz", "reasons", "samples"} <= set(out)


def test_reference_arm_under_two_ranks_prints_once():
    # launched like the multi-GPU bench (RANK / WORLD_SIZE in the environment): rank 0 runs
    # the oracle and prints the one JSON line, rank 1 exits 0 without work or output
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    outs = []
    for rank in (0, 1):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT="29531")
        r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload",
                            "tiny_causal", "--gpus", "2", "--steps", "1", "--warmup", "0"],
                           cwd=root, env=env, capture_output=True, text=True, timeout=300)
        assert r.returncode == 0, r.stderr
        outs.append([x for x in r.stdout.splitlines() if x.startswith("{")])
    assert len(outs[0]) == 1 and outs[1] == []
    d = json.loads(outs[0][0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
