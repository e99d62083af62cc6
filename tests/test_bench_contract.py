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


@pytest.mark.parametrize("extra", [[], ["--nvfp4"]], ids=["mxfp4", "nvfp4"])
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
    assert d["config"]["format"] == ("nvfp4" if extra else "mxfp4")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_is_silent_on_other_ranks():
    rc, lines = _run(["--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-rows", "2"],
                     {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert rc == 0 and lines == []


def test_bench_rejects_too_few_warmup_steps_and_bad_format_combinations():
    rc, _ = _run(["--impl", "reference", "--steps", "1", "--warmup", "2"])
    assert rc != 0
    rc, _ = _run(["--impl", "reference", "--steps", "1", "--warmup", "3", "--nvfp4", "--hp-fp16"])
    assert rc != 0
