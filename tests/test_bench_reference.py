"""bench.py's reference arm (CPU): the oracle timed on the host cores prints
one JSON line on the same metric, unit and config as the library's arm, with
its cpu_baseline and an e2e record that moves no bytes; ranks other than 0
print nothing; fewer than 3 warm-up steps are refused."""
import json
import os
import subprocess
import sys

import bench
from mixture_experts_routing_top_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run(args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                          cwd=ROOT, env=e, timeout=600)


def line(args):
    r = run(args)
    assert r.returncode == 0, r.stderr[-2000:]
    out = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(out) == 1
    return json.loads(out[0])


def check_contract(res, steps):
    assert res["impl"] == "reference" and res["metric"] == bench.METRIC and res["unit"] == "tokens/s"
    assert res["higher_is_better"] is True and res["scaling"] == "weak" and res["vs_baseline"] is None
    assert res["steps"] == steps and res["warmup"] == 3 and res["value"] > 0 and res["ms_per_step"] > 0
    cb = res["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] == res["value"] and cb["sample"]
    assert res["e2e"] == {"value": res["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}


def test_reference_line_on_the_tiny_layer():
    res = line(["--impl", "reference", "--workload", "tiny_fp32", "--steps", "4", "--warmup", "3"])
    check_contract(res, 4)
    cfg = dict(res["config"])
    assert cfg.pop("l2")
    assert cfg == bench.workload_config(W.TINY, 1)


def test_reference_line_routing_only():
    res = line(["--impl", "reference", "--workload", "dispatch_combine_sweep_bf16", "--routing-only",
                "--steps", "3", "--warmup", "3"])
    check_contract(res, 3)
    assert res["config"]["workload"].endswith("[routing only]") and res["config"]["E"] == 256


def test_other_ranks_print_nothing():
    r = run(["--impl", "reference", "--workload", "tiny_fp32", "--steps", "3", "--warmup", "3"],
            {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_too_few_warmup_steps_refused():
    r = run(["--impl", "reference", "--workload", "tiny_fp32", "--steps", "3", "--warmup", "2"])
    assert r.returncode != 0 and "warmup" in r.stderr


def test_several_gpus_need_one_process_each():
    r = run(["--impl", "reference", "--workload", "tiny_fp32", "--gpus", "2", "--steps", "3", "--warmup", "3"])
    assert r.returncode != 0 and "one process per GPU" in r.stderr
    r = run(["--impl", "reference", "--workload", "tiny_fp32", "--gpus", "2", "--steps", "3", "--warmup", "3"],
            {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""
