"""bench.py's oracle arm on CPU: it prints the contract line for a workload and
never loads the CUDA library (its chunk label is restated in Python)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_runs_without_the_library():
    code = ("import sys; sys.argv = ['bench.py', '--impl', 'reference', '--config', '0', "
            "'--steps', '2', '--warmup', '1']; import bench; rc = bench.main(); "
            "print('LIB_LOADED' if any(m.startswith('chunked_kl_loss_tcgen05_b200') "
            "for m in sys.modules) else 'LIB_NOT_LOADED'); sys.exit(rc)")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    lines = r.stdout.strip().splitlines()
    assert lines[-1] == "LIB_NOT_LOADED"
    line = json.loads(lines[-2])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["config"]["workload"].startswith("tiny") and line["config"]["chunk"] == 64
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["higher_is_better"] is True
