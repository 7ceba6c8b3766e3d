"""bench.py's host-side contract, on the CPU: the reference arm (the oracle on the
host cores) prints one JSON line with the contract's keys; under several ranks
only rank 0 prints; fewer than 3 warm-up steps is an error; without a GPU the
product arm fails loudly instead of falling back to the CPU; the DRAM traffic
figure is reported only while the captured kernel sources are unchanged."""
import hashlib
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None, timeout=600):
    env = dict(os.environ)
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=timeout)


def test_gpus_flag_starts_the_ranks_itself():
    """`bench.py --gpus 2` outside a launcher starts two ranks itself; under the
    reference arm only rank 0 works and prints, and it reports both ranks."""
    r = _run(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    assert json.loads(lines[0])["n_gpus"] == 2


def test_reference_arm_json_line():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["higher_is_better"] is True
    assert d["dtype"] == "f64" and d["data"] == "synthetic" and "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "3"],
             {"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_too_few_warmup_steps_is_an_error():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "2"])
    assert r.returncode != 0 and "warm-up" in r.stderr


@pytest.mark.skipif(torch.cuda.is_available(), reason="on a GPU host the product arm runs the real bench")
def test_product_arm_fails_loudly_without_a_gpu():
    r = _run(["--steps", "1", "--warmup", "3"], timeout=300)
    assert r.returncode != 0
    assert not [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_traffic_only_for_the_captured_sources(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    srcs = ["prefill_tc.cu", "prep_body.cuh", "chain_body.cuh"]
    h = hashlib.sha1()
    for f in srcs:
        with open(os.path.join(ROOT, "linear_attention_token_shortconv_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    monkeypatch.setattr(bench, "NCU_TRAFFIC", {
        "now": {"sources": srcs, "sha1": h.hexdigest(), "bytes_per_unit": 2.0},
        "stale": {"sources": srcs, "sha1": "0" * 40, "bytes_per_unit": 2.0},
        "missing": {"sources": ["no_such_file.cu"], "sha1": h.hexdigest(), "bytes_per_unit": 2.0}})
    assert bench.kernel_traffic("now", 10) == 20.0
    assert bench.kernel_traffic("stale", 10) is None
    assert bench.kernel_traffic("missing", 10) is None
    assert bench.kernel_traffic("never_captured", 10) is None
