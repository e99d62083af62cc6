"""bench.py's JSON line, checked on CPU through its reference arm (the
oracle timed on the host): one line with the contract's keys on rank 0,
nothing and exit status 0 on the other ranks."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    return p.returncode, [l for l in p.stdout.splitlines() if l.strip()]


@pytest.mark.parametrize("extra", [["--workload", "up"], ["--workload", "up", "--nvfp4"]], ids=["mxfp4", "nvfp4"])
def test_reference_arm_prints_one_contract_line(extra):
    rc, lines = _run(["--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-rows", "2", *extra])
    assert rc == 0 and len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "wan_ffn_up_4096x5120x13824"
    assert d["config"]["format"] == ("nvfp4" if "--nvfp4" in extra else "mxfp4")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_default_workload_is_the_four_block_ffn():
    # the default run measures the largest single-GPU configuration (here one
    # block of it, to keep the CPU oracle short)
    rc, lines = _run(["--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-rows", "8", "--blocks", "1"])
    assert rc == 0 and len(lines) == 1
    d = json.loads(lines[0])
    cfg = d["config"]
    assert cfg["workload"].startswith("wan_ffn_block_x4_32760x5120x13824")
    assert (cfg["M"], cfg["d_model"], cfg["d_ff"], cfg["layers"]) == (32760, 5120, 13824, 1)
    assert d["value"] > 0 and d["impl"] == "reference"


def test_reference_arm_is_silent_on_other_ranks():
    rc, lines = _run(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--ref-rows", "2",
                      "--workload", "up"], {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert rc == 0 and lines == []


def test_gpus_n_starts_n_ranks_and_rank0_alone_prints():
    # without a launcher environment, --gpus 2 starts two ranks itself
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3", "--ref-rows", "2", "--workload", "tiny"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    lines = [l for l in p.stdout.splitlines() if l.strip().startswith("{")]
    assert p.returncode == 0, p.stderr[-2000:]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["impl"] == "reference"


def test_gpus_must_match_the_launcher():
    rc, _ = _run(["--impl", "reference", "--gpus", "4", "--steps", "1", "--warmup", "3", "--workload", "tiny"],
                 {"RANK": "0", "WORLD_SIZE": "2", "LOCAL_RANK": "0"})
    assert rc != 0


def test_bench_rejects_too_few_warmup_steps_and_bad_format_combinations():
    rc, _ = _run(["--impl", "reference", "--steps", "1", "--warmup", "2"])
    assert rc != 0
    rc, _ = _run(["--impl", "reference", "--steps", "1", "--warmup", "3", "--nvfp4", "--hp-fp16"])
    assert rc != 0
