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


def test_memory_sweep_is_linear_in_rows():
    """bench.py --mem-sweep: peak device memory of one forward+backward call grows
    by the per-row inputs and outputs only (hidden 8 KiB, dH 16 KiB, teacher
    0.78 KiB, two per-row words), and an explicit chunk bounds the rest."""
    r = subprocess.run([sys.executable, "bench.py", "--mem-sweep", "--sweep-chunk", "256",
                        "--sweep-s", "1024,2048,4096"], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    per_row_kib = (4096 * 2 + 4096 * 4 + 100 * 8 + 8) / 1024
    assert abs(d["fit"]["slope_kib_per_row"] - per_row_kib) < 0.05
    assert d["fit"]["r2"] > 0.9999
    # W (1 GiB) + dW (2 GiB) + one 256-row chunk of dlogits and per-chunk buffers
    assert 2.9 < d["fit"]["intercept_gib"] < 3.1
