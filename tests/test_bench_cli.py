"""bench.py's CPU legs and the binding's failure mode (CPU only).

* ``--impl reference`` (the float64 oracle on the host cores) prints one JSON
  line with the contract's keys; under torchrun the non-zero ranks print
  nothing and exit 0.
* Without the shared library every call of the binding raises: there is no
  fallback path.
"""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None, timeout=300):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_the_contract_line():
    r = _run(["--impl", "reference", "--workload", "head1_t4096", "--steps", "1", "--warmup", "1", "--cpu-seconds", "1"])
    assert r.returncode == 0, r.stderr[-2000:]
    line = r.stdout.strip().splitlines()[-1]
    d = json.loads(line)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"]


def test_reference_arm_other_ranks_exit_quietly():
    r = _run(["--impl", "reference", "--workload", "head1_t4096", "--steps", "1", "--warmup", "0"],
             env_extra={"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_binding_raises_without_the_library(tmp_path):
    code = (
        "import rope_aware_kv_tri_b200 as tri\n"
        f"tri.LIB_PATH = {str(tmp_path / 'missing.so')!r}\n"
        "try:\n"
        "    tri.tri_status_string(0)\n"
        "except RuntimeError as e:\n"
        "    print('raised', 'not built' in str(e))\n"
    )
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == "raised True"
