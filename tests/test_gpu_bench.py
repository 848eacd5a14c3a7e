"""bench.py on the GPU: the contract line of the tiny workload, plain and through
the data-parallel path on a one-rank process group, carries the keys the
measurement needs and an oracle-consistent loss."""
import json
import os
import subprocess
import sys

import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _line(*args):
    r = subprocess.run([sys.executable, "bench.py", "--config", "0", "--steps", "3", "--warmup", "3",
                        *args], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


@pytest.mark.parametrize("mode", [[], ["--mode", "dp", "--no-cpu-baseline"]])
def test_bench_contract_line(mode):
    d = _line(*mode)
    assert d["unit"] == "tokens/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["config"]["workload"].startswith("tiny") and d["config"]["chunk"] == 64
    assert d["gpu_launches"] > 0
    r = d["roofline"]
    assert r["bound"] in ("tensor", "hbm") and r["achieved"] > 0 and r["frac"] > 0
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] == 4
    o = oracle.oracle_from_inputs(synth.make_inputs(0))
    assert abs(d["loss"] - o["loss"]) <= 1e-3 * abs(o["loss"])
    if mode:
        assert d["config"]["parallelism"].startswith("dp1")
    else:
        assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] > 0
