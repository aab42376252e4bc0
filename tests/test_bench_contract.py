"""The benchmark's command-line contract, checked on the host.

The reference arm (the fp64 oracle on the host cores) must print exactly one
JSON line with the keys the contract names, and report the same `config`
object as the CUDA arm.  Without a GPU, the CUDA arm must fail loudly rather
than fall back to anything else.
"""
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args, timeout=600):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_contract_line():
    r = run_bench("--impl", "reference", "--workload", "tiny_mqa_decode", "--steps", "2", "--warmup", "1")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["value"] > 0 and line["unit"] == "GB/s"
    assert (line["n_gpus"], line["steps"], line["warmup"]) == (1, 2, 1)
    assert line["higher_is_better"] is True and line["scaling"] == "weak" and line["data"] == "synthetic"
    cfg = line["config"]
    assert cfg["workload"] == "tiny_mqa_decode" and cfg["B"] == 1 and cfg["D"] == 64 and cfg["append"] is False
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_both_arms_share_the_config_object():
    sys.path.insert(0, ROOT)
    import bench
    from decode_attention_packed_b200.workloads import make_inputs, workload

    w = workload("gqa_decode")
    inp = make_inputs(w)
    cfg = bench.workload_config(w, bench.algorithmic_bytes(inp), 1)
    assert cfg["workload"] == "gqa_decode" and cfg["kv_bytes_per_call"] == inp.kv_bytes()
    assert cfg["parallelism"].startswith("dp1")


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a GPU")
def test_cuda_arm_fails_loudly_without_a_gpu():
    r = run_bench("--steps", "1", "--warmup", "1", "--no-clocks", timeout=300)
    assert r.returncode != 0
    assert not [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]


def test_default_run_is_the_headline_with_the_suite():
    sys.path.insert(0, ROOT)
    import bench

    a = bench.parse([])
    assert a.workload == bench.HEADLINE == "ragged_varlen" and a.suite and a.gpus == 1
    assert (a.steps, a.warmup) == (20, 5)
    assert set(bench.SUITE) == {"gqa_decode", "spec_mtp_small_q", "long_context_split_kv"}
    b = bench.parse(["--workload", "gqa_decode"])
    assert b.workload == "gqa_decode" and not b.suite
    assert not bench.parse(["--no-suite"]).suite
