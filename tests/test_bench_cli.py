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
    r = _run(["--impl", "reference", "--workload", "head1_t4096", "--steps", "1", "--warmup", "0", "--gpus", "2"],
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


def _small_cpu_workload():
    sys.path.insert(0, ROOT)
    from workload import CONFIGS, make_workload
    cfg = CONFIGS["l32h8_t32k"].replace(L=2, Hkv=2, G=2, lens=[3000, 900], budget=512, window=64, n_samples=256)
    wl = make_workload(cfg, device="cpu")
    rblocks = wl.block_table[:, :32].reshape(-1).long()
    return cfg, wl, rblocks


def _args(**kw):
    import argparse
    d = dict(cpu_seconds=0.5, sinks=0, aggregate="mean", trigger=0)
    d.update(kw)
    return argparse.Namespace(**d)


def test_cpu_baseline_covers_the_variants():
    """The CPU baseline of a variant bench line times that variant: the C
    oracle with sinks and the max over the group, and the distance-table step
    for the distance-only mode."""
    import bench
    cfg, wl, rblocks = _small_cpu_workload()
    save_k, save_v = wl.k_pool[:, rblocks].clone(), wl.v_pool[:, rblocks].clone()
    lens = wl.seq_len.tolist()
    for kw in (dict(), dict(sinks=4), dict(aggregate="max")):
        out = bench.run_cpu_baseline(_args(**kw), wl, cfg, save_k, save_v, rblocks, lens)
        assert out["kind"] == "oracle" and out["value"] > 0 and out["cores"] >= 1
        assert out["c_oracle_1_thread"]["value"] > 0 and out["cpu_model"]
    max_dist = int(wl.cur_pos.max().item()) + 1
    out = bench.run_cpu_baseline_distance(_args(), wl, cfg, save_k, save_v, rblocks, lens, max_dist)
    assert out["kind"] == "oracle" and out["value"] > 0 and "table lookup" in out["sample"]


def test_reference_arm_times_the_requested_variant():
    for extra, marker in ((["--aggregate", "max", "--sinks", "2"], "plain C float64 oracle"),
                          (["--score-mode", "distance"], "distance-table lookup")):
        r = _run(["--impl", "reference", "--workload", "head1_t4096", "--steps", "1", "--warmup", "0",
                  "--cpu-seconds", "1"] + extra)
        assert r.returncode == 0, r.stderr[-2000:]
        d = json.loads(r.stdout.strip().splitlines()[-1])
        assert d["value"] > 0 and marker in d["cpu_baseline"]["sample"]
        if "--aggregate" in extra:
            assert d["config"]["aggregate"] == "max" and d["config"]["sinks"] == 2
        else:
            assert d["config"]["score_mode"] == "distance"


def _stub_runner(args, world, rank, local, dist):
    """One rank of ``bench.main`` with the GPU step replaced by a stand-in
    timing (rank r takes 10 + r ms over the timed steps) and a freed count
    derived from the rank's own plan; everything else is bench.py's own
    per-rank plan and job reduction over the process group."""
    import bench
    cfg, seed, heads_mode = bench.rank_plan(args, world, rank)
    keys_per_step = sum(cfg.lens) * cfg.L * cfg.Hkv
    freed_per_step = sum(-(-n // 16) - -(-min(n, cfg.budget) // 16) for n in cfg.lens)
    job = bench.job_summary(dist, 10.0 + rank, keys_per_step, freed_per_step, args.steps, heads_mode)
    plans = [None] * world
    dist.all_gather_object(plans, (cfg.Hkv, seed))
    if rank == 0:
        print(json.dumps({"n_gpus": job["n_gpus"], "scaling": job["scaling"], "value": job["value"],
                          "ms_per_step": job["ms_per_step"], "job_keys": job["job_keys"],
                          "job_freed": job["job_freed"], "freed_same": job["freed_same"], "plans": plans}),
              flush=True)


def _spawned_bench(argv):
    code = ("import sys, json\n"
            f"sys.path.insert(0, {ROOT!r})\n"
            "import bench\n"
            "from tests.test_bench_cli import _stub_runner\n"
            f"bench.main({argv!r}, runner=_stub_runner, backend='gloo')\n")
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    return subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=300)


def test_gpus_flag_spawns_that_many_ranks_with_head_sharding():
    r = _spawned_bench(["--gpus", "2", "--shard", "heads", "--steps", "4"])
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout                # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["scaling"] == "strong"
    # the 32x8-head workload's KV heads split 4 + 4, each rank seeded apart
    assert [p[0] for p in d["plans"]] == [4, 4] and d["plans"][0][1] != d["plans"][1][1]
    assert d["ms_per_step"] == 11.0 / 4                      # the slowest rank's time
    assert d["job_keys"] == 2 * 32768 * 32 * 4              # both ranks' keys
    assert d["freed_same"] is True and d["job_freed"] == 2 * 1920
    assert d["value"] == d["job_keys"] * 4 / 0.011


def test_gpus_flag_with_sequence_sharding_is_weak_scaling():
    r = _spawned_bench(["--gpus", "2", "--steps", "2"])
    assert r.returncode == 0, r.stderr[-3000:]
    d = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][0])
    assert d["n_gpus"] == 2 and d["scaling"] == "weak" and d["freed_same"] is None
    assert [p[0] for p in d["plans"]] == [8, 8] and d["job_keys"] == 2 * 32768 * 32 * 8


def test_world_size_must_match_gpus_flag():
    r = _run(["--gpus", "4", "--steps", "1"], env_extra={"WORLD_SIZE": "2", "RANK": "0", "LOCAL_RANK": "0"})
    assert r.returncode != 0 and "WORLD_SIZE=2" in (r.stderr + r.stdout)


def test_launch_accounting_and_flush_options():
    """The launch count the bench line claims and the kernels it names follow
    the step's shape: three launches when the step selects and compacts in
    one persistent kernel, five with the separate kernels, for either score
    mode; the L2 flush mode is a choice between two documented options."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.launches_per_step(True) == 3
    assert bench.launches_per_step(False) == 5
    assert bench.kernel_list(True, False) == "query_kernel, score kernel, select_compact_kernel"
    assert bench.kernel_list(True, True) == "query_kernel (plan only), distance_score_kernel, select_compact_kernel"
    assert bench.kernel_list(False, False).endswith("evict_kernel, move_kernel x2")
    assert bench.parse_args([]).l2_flush == "clean"
    assert bench.parse_args(["--l2-flush", "dirty"]).l2_flush == "dirty"
