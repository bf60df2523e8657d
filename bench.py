#!/usr/bin/env python
"""Throughput of the TriAttention key-importance + eviction step on B200.

One step = tri_compress_step over one synthetic cache: effective query,
score of every cached key, top-B selection with a recent window, and
forward-packing compaction of the kept K/V rows.  Default workload: 32
layers x 8 KV heads, GQA group 4, one sequence of 32768 cached bf16 keys,
RoPE base 5e5, offsets 1..4096, B = 2048, W = 128.

Metric: cached keys scored+selected+compacted per second (whole job, all
ranks), with the achieved HBM GB/s of the dominant (score) kernel and of the
whole step against the measured B200 copy bandwidth.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...   (one rank per GPU)

--gpus N > 1 without torchrun starts the N ranks itself (one process per
GPU, NCCL); under torchrun WORLD_SIZE must equal --gpus.

Timing: each timed step restores the kept region of the cache and flushes L2
outside CUDA events that bracket only the tri_compress_step launches: a
256 MiB buffer is written, then (default --l2-flush clean) another 256 MiB is
read, so the write's dirty lines reach DRAM before the step instead of during
its first kernels.  The K/V pools (4.3 GB) are larger than L2 as well.  The timed loop
is bracketed by a barrier and a device synchronize; the step time is the
maximum over ranks.  Ranks run independent caches (weak scaling: units
shard across GPUs with no data-path collective).
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "cached keys scored+selected+compacted per sec; achieved HBM GB/s vs peak"
UNIT = "keys/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 7700.0
L2_FLUSH_BYTES = 256 << 20


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="l32h8_t32k", help="head1_t4096 | l32h8_t32k | decode16 | l32h8_t128k | l64h8g8_4x64k")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target oracle sample time")
    ap.add_argument("--sinks", type=int, default=0, help="leading slots always kept (variant)")
    ap.add_argument("--trigger", type=int, default=0, help="compress only sequences longer than this (variant)")
    ap.add_argument("--aggregate", choices=["mean", "max"], default="mean",
                    help="GQA aggregation of the per-head scores (variant)")
    ap.add_argument("--score-mode", choices=["keys", "distance"], default="keys",
                    help="keys: score every cached key (the method); distance: table of the centres (variant)")
    ap.add_argument("--shard", choices=["sequences", "heads"], default="sequences",
                    help="N>1: an independent cache per GPU (weak scaling) or the KV heads of one "
                         "cache split over the GPUs (strong scaling)")
    ap.add_argument("--graph", action="store_true",
                    help="capture one step in a CUDA graph and time its replays")
    ap.add_argument("--phases", action="store_true",
                    help="decode loop: time each round's phases with library events (serialises launches)")
    ap.add_argument("--l2-flush", choices=["clean", "dirty"], default="clean",
                    help="between timed steps write a buffer larger than L2, then (clean) read a second one so "
                         "that the write's dirty lines are written back before the step, or (dirty) not")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the layer count (small profiling cases of the same kernels)")
    return ap.parse_args(argv)


# ----------------------------------------------------------------- helpers

class L2Flush:
    """Evicts the step's data from L2 between timed steps: writes a buffer
    larger than L2; in "clean" mode then reads a second one, so the write's
    dirty lines are written back before the timed step rather than during
    its first kernels (the state after kernels that only read, such as
    attention over the cache)."""

    def __init__(self, mode: str, dev):
        import torch
        self.mode = mode
        self.buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.buf2 = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev) if mode == "clean" else None

    def __call__(self):
        self.buf.zero_()
        if self.buf2 is not None:
            self.buf2.amax()

    def describe(self) -> str:
        mib = L2_FLUSH_BYTES >> 20
        if self.mode == "clean":
            return (f"K/V pools larger than L2; between timed steps {mib} MiB written, then another {mib} MiB "
                    "read (L2 holds no step data and no dirty lines)")
        return f"K/V pools larger than L2; {mib} MiB written between timed steps (L2 left dirty)"


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# Sources of each kernel whose DRAM traffic record is kept under profiles/.
KERNEL_SOURCES = {
    "score_kernel": ["score.cu", "score_device.cuh", "tri_device.cuh", "tri_internal.h"],
    "select_compact_kernel": ["select_compact.cu", "select_device.cuh", "tri_device.cuh", "tri_internal.h"],
}


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "rope_aware_kv_tri_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic_per_launch(kernel: str, keys: int, moved_rows: int):
    """DRAM bytes of one launch of ``kernel`` on this workload, from the
    committed ncu record (bytes per scored key and per moved row, taken on a
    smaller case of the same kernel), if that record was taken on the
    kernel's current source; else None."""
    if kernel not in KERNEL_SOURCES:
        return None
    path = os.path.join(ROOT, "profiles", f"{kernel}_traffic.txt")
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if "=" in line and not line.lstrip().startswith("#"):
                    k, v = line.split("=", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("source_sha256") != kernel_source_hash(kernel):
            return None
        return round(float(kv["dram_bytes_per_key"]) * keys + float(kv.get("dram_bytes_per_moved_row", 0)) * moved_rows)
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None
        self.bus = None
        try:
            import torch
            self.bus = int(torch.cuda.get_device_properties(device_index).pci_bus_id)
        except Exception:
            pass

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu=pci.bus_id,{self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.5)
        self.t0 = time.time()

    def stop(self):
        self.t1 = time.time()
        time.sleep(0.3)
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        if not self.lines:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            try:
                bus = int(f[0].split(":")[1], 16)
            except Exception:
                bus = None
            if self.bus is not None and bus is not None and bus != self.bus:
                continue
            f = f[1:]
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except Exception:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(args, backend="nccl"):
    """Rank, world and process group of this process.  Under torchrun (or a
    rank spawned by ``spawn_ranks``) the world comes from WORLD_SIZE, which
    must equal --gpus; a single process has world 1.  ``backend`` "nccl"
    binds the process to GPU LOCAL_RANK; "gloo" (host-only tests) does not."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if "WORLD_SIZE" in os.environ and world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch one rank per GPU")
    if world > 1:
        import torch.distributed as dist
        if args.impl == "reference":
            return world, rank, local, None
        if backend == "nccl":
            import torch
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return world, rank, local, dist
    return world, rank, local, None


def rank_plan(args, world, rank):
    """The workload one rank runs: (config, seed, heads_mode).

    --shard sequences (default): every rank runs its own independent cache
    of the full workload shape, seeded per rank (weak scaling).  --shard
    heads: the KV heads of one cache are split over the ranks (each keeps
    its slice of heads, and their query heads, for every sequence), every
    rank seeded apart (strong scaling)."""
    from workload import CONFIGS
    from rope_aware_kv_tri_b200.sharding import shard_heads, shard_seed
    cfg = CONFIGS[args.workload]
    if args.layers > 0:
        cfg = cfg.replace(L=args.layers, name=f"{cfg.name} (L={args.layers})")
    heads_mode = args.shard == "heads" and world > 1
    if heads_mode:
        cfg = cfg.replace(Hkv=len(shard_heads(cfg.Hkv, world, rank)))
    seed = shard_seed(cfg.seed, rank) if world > 1 else cfg.seed
    return cfg, seed, heads_mode


def job_summary(dist, step_ms_total, keys_per_step, freed_per_step, steps, heads_mode, device=None):
    """Reduce one rank's timed steps to the job's figures: the slowest
    rank's time, all ranks' keys and freed blocks, and (head sharding)
    whether every rank freed the same number of blocks.  Every rank takes
    the same collective steps in the same order."""
    from rope_aware_kv_tri_b200.sharding import freed_consistent, keys_per_second, reduce_job
    total_ms, job_keys, job_freed = reduce_job(dist, step_ms_total, keys_per_step, freed_per_step, device)
    freed_same = freed_consistent(dist, freed_per_step, device) if heads_mode else None
    world = dist.get_world_size() if dist is not None else 1
    return {"value": keys_per_second(job_keys, steps, total_ms), "ms_per_step": total_ms / steps,
            "job_keys": job_keys, "job_freed": job_freed, "freed_same": freed_same, "n_gpus": world,
            "scaling": "strong" if heads_mode else "weak"}


def _free_port():
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _spawned_rank(rank, world, port, argv, runner, backend):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "LOCAL_WORLD_SIZE": str(world), "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    main(argv, runner=runner, backend=backend)


def spawn_ranks(args, argv, runner=None, backend="nccl"):
    """--gpus N > 1 without torchrun: start N ranks on this node, one process
    per GPU (rank r on GPU r), with the same arguments; rank 0 prints the
    job's line.  Returns the worst exit code."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_spawned_rank, args=(r, args.gpus, port, argv, runner, backend))
             for r in range(args.gpus)]
    for p in procs:
        p.start()
    codes = []
    for p in procs:
        p.join()
        codes.append(p.exitcode if p.exitcode is not None else 1)
    return max(codes, key=abs)


def unit_rows(pool, table_row, length, l, h):
    """Rows [0, length) of (layer l, KV head h) of one sequence of a paged pool."""
    import torch
    nb = -(-length // 16)
    blocks = torch.tensor(table_row[:nb], dtype=torch.long, device=pool.device)
    return pool[l, blocks, h].reshape(nb * 16, pool.shape[-1])[:length]


# ---------------------------------------------------------- oracle sample

def oracle_sample(units, stats_fn, deltas, base, budget, window, seconds, sinks=0, aggregate="mean"):
    """Time the float64 oracle on units until about ``seconds`` have passed.

    ``units`` yields (keys_bf16_cpu [T,128], vals_bf16_cpu, (s, l, h), p).
    Returns (keys scored, seconds, units done).
    """
    import numpy as np
    import torch
    import oracle
    try:
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(1)
    except Exception:
        limit = None
    keys_done, t_used, n = 0, 0.0, 0
    for keys, vals, (s, l, h), p in units:
        qb, qa, r = stats_fn(l, h)
        kf = keys.double().numpy()
        kb, vb = keys.view(torch.int16).numpy(), vals.view(torch.int16).numpy()
        t0 = time.perf_counter()
        oracle.compress_unit(kf, kb, vb, qb, qa, r, p, deltas, base, budget, window, sinks, aggregate)
        t_used += time.perf_counter() - t0
        keys_done += kf.shape[0]
        n += 1
        if t_used >= seconds:
            break
    if limit is not None:
        limit.restore_original_limits()
    return keys_done, t_used, n


def host_cpu_model():
    """The host CPU's model name, as the kernel reports it."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def c_oracle_sample(units, stats_fn, deltas, base, budget, window, seconds, threads, sinks=0, aggregate="mean"):
    """Time the plain C float64 oracle on units, ``threads`` units at a time
    on the host cores, until about ``seconds`` of wall time have passed.
    Unit inputs are prepared outside the timed region.  Returns (keys
    scored, wall seconds, units done)."""
    from concurrent.futures import ThreadPoolExecutor
    import torch
    from oracle.c_oracle import compress_unit_c
    keys_done, t_used, n = 0, 0.0, 0
    with ThreadPoolExecutor(max_workers=threads) as pool:
        while True:
            batch = []
            for keys, vals, (s, l, h), p in units:
                qb, qa, r = stats_fn(l, h)
                batch.append((keys.view(torch.int16).numpy(), vals.view(torch.int16).numpy(), qb, qa, r, p))
                if len(batch) == 2 * threads:
                    break
            if not batch:
                break
            t0 = time.perf_counter()
            list(pool.map(lambda a: compress_unit_c(a[0], a[1], a[2], a[3], a[4], a[5], deltas, base, budget,
                                                    window, sinks, aggregate), batch))
            t_used += time.perf_counter() - t0
            keys_done += sum(a[0].shape[0] for a in batch)
            n += len(batch)
            if t_used >= seconds:
                break
    return keys_done, t_used, n


# --------------------------------------------------------------- our arm

def run_ours(args, world, rank, local, dist):
    import numpy as np
    import torch
    import rope_aware_kv_tri_b200 as tri
    from rope_aware_kv_tri_b200 import build_lib
    from workload import CONFIGS, make_workload

    build_lib.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.workload == "decode16":
        return run_decode(args, world, rank, local, dist, rank_plan(args, world, rank)[0])
    cfg, seed, heads_mode = rank_plan(args, world, rank)
    wl = make_workload(cfg, device=dev, seed=seed)
    L, Hkv, G, Hq, S = cfg.L, cfg.Hkv, cfg.G, cfg.Hq, cfg.S
    B, W = cfg.budget, cfg.window
    stream = torch.cuda.current_stream(dev)

    # statistics: one-time calibration on the device (untimed)
    if wl.qbar is not None:
        qbar, qabs, R = wl.qbar, wl.qabs, wl.R
    else:
        qbar = torch.empty(L, Hq, 128, device=dev)
        qabs = torch.empty(L, Hq, 64, device=dev)
        R = torch.empty(L, Hq, device=dev)
        tri.tri_calibrate_centers(wl.q_samples, qbar, qabs, R)
        torch.cuda.synchronize(dev)

    lens = wl.seq_len.cpu().tolist()
    kept_blocks = [min((n + 15) // 16, (B + 15) // 16) for n in lens]
    trig = max(args.trigger, B)
    keys_per_step = sum(n for n in lens if n > trig) * L * Hkv      # keys of the sequences the step compresses
    cache = tri.KvCache(wl.k_pool, wl.v_pool, wl.block_table, wl.seq_len, wl.cur_pos,
                        torch.zeros(1, dtype=torch.int32, device=dev), G)
    variant = (args.sinks, args.trigger, args.aggregate) != (0, 0, "mean")
    distance = args.score_mode == "distance"
    opt = tri.step_options(B, W, args.sinks, args.trigger,
                           tri.TRI_AGG_MAX if args.aggregate == "max" else tri.TRI_AGG_MEAN)
    fused = tri.tri_step_is_fused(cache, opt)
    ws = tri.alloc_workspace(cache, opt)
    freed = torch.empty(S * wl.max_blocks, dtype=torch.int32, device=dev)
    count = torch.empty(1, dtype=torch.int32, device=dev)

    # the rows a step may rewrite: blocks holding slots [0, B) of each sequence
    rblocks = torch.cat([wl.block_table[s, :kept_blocks[s]].long() for s in range(S)])
    save_k = wl.k_pool[:, rblocks].clone()
    save_v = wl.v_pool[:, rblocks].clone()
    save_len = wl.seq_len.clone()
    flush = L2Flush(args.l2_flush, dev)
    table_ms = None
    if distance:
        # one-time table of the centres (untimed, like the calibration)
        max_dist = int(wl.cur_pos.max().item()) + 1
        dtable = torch.empty(L, Hkv, max_dist + 1, device=dev)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        tri.tri_distance_table(qbar, wl.key_centres.float().contiguous(), cfg.base, wl.deltas,
                               tri.TRI_AGG_MAX if args.aggregate == "max" else tri.TRI_AGG_MEAN, dtable)
        t1.record()
        torch.cuda.synchronize(dev)
        table_ms = t0.elapsed_time(t1)
        max_len = wl.max_blocks * 16
        slot_pos = torch.arange(max_len, dtype=torch.int32, device=dev).repeat(S, L, Hkv, 1).contiguous()
        save_pos = slot_pos[..., :B].clone()

    def restore():
        wl.k_pool[:, rblocks] = save_k
        wl.v_pool[:, rblocks] = save_v
        wl.seq_len.copy_(save_len)
        if distance:
            slot_pos[..., :B] = save_pos
        flush()

    def step(events=None, idx_out=None):
        if distance:
            tri.tri_compress_step_distance(cache, dtable, slot_pos, opt, ws, freed_ids=freed, freed_count=count,
                                           idx_out=idx_out, events=events)
        elif variant:
            tri.tri_compress_step_ex(cache, qbar, qabs, R, cfg.base, wl.deltas, opt, ws, freed_ids=freed,
                                     freed_count=count, idx_out=idx_out, events=events)
        else:
            tri.tri_compress_step(cache, qbar, qabs, R, cfg.base, wl.deltas, B, W, freed, count, ws,
                                  idx_out=idx_out, events=events)

    # census (untimed): how many rows a step moves, from its kept indices
    idx = torch.empty(S, L, Hkv, B, dtype=torch.int32, device=dev)
    restore()
    step(idx_out=idx)
    if tri.tri_sync_status(cache.status) != tri.TRI_OK:
        raise RuntimeError("device status flag raised by the census step")
    moved = 0
    kept_rows = 0      # every kept row of a compressed sequence: the upper bound of the moves
    for s in range(S):
        if lens[s] > trig:
            j = torch.arange(B, device=dev, dtype=torch.int32)
            moved += int((idx[s] != j).sum().item())
            kept_rows += L * Hkv * B
    del idx
    freed_per_step = int(count.item())

    for _ in range(args.warmup):
        restore()
        step()
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()

    # Optionally the step as a CUDA graph: one capture, replayed every timed
    # step (the same device pointers, so the replay redoes the whole step).
    graph = None
    if args.graph:
        restore()
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        torch.cuda.synchronize(dev)
        for _ in range(args.warmup):
            restore()
            graph.replay()
        torch.cuda.synchronize(dev)

    # Timed steps: one event pair around each tri_compress_step (its kernels
    # then overlap their launches programmatically).
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    for k in range(args.steps):
        restore()
        evs[k][0].record()
        if graph is not None:
            graph.replay()
        else:
            step()
        evs[k][1].record()
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    clocks.stop()
    del graph
    if tri.tri_sync_status(cache.status) != tri.TRI_OK:
        raise RuntimeError("device status flag raised during the timed steps")
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]

    # Phase times (live, same workload): the library records events between
    # its kernels, which serialises their launches, so this is a separate loop.
    n_phase = min(args.steps, 200)
    pevs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_phase)]
    for k in range(n_phase):
        restore()
        step(events=pevs[k])
    torch.cuda.synchronize(dev)
    query_ms = [e[0].elapsed_time(e[1]) for e in pevs]
    score_ms = [e[1].elapsed_time(e[2]) for e in pevs]
    evict_ms = [e[2].elapsed_time(e[3]) for e in pevs]
    job = job_summary(dist, sum(step_ms), keys_per_step, freed_per_step, args.steps, heads_mode, dev)
    value, ms_per_step = job["value"], job["ms_per_step"]
    job_freed, freed_same = job["job_freed"], job["freed_same"]

    peak, peak_kind = measured_peak()
    bytes_per_key = 12 if distance else 256     # distance: position + table entry + score; keys: the bf16 key
    k_bytes = keys_per_step * bytes_per_key
    moved_bytes = moved * 4 * 256
    score_mean = statistics.mean(score_ms)
    kernel = "distance_score_kernel" if distance else ("score_mma_kernel" if args.aggregate == "max"
                                                       else "score_kernel")
    kernel_bytes = k_bytes
    what = "the score kernel"
    kernel_ms = score_mean
    achieved = kernel_bytes / (kernel_ms / 1e3) / 1e9
    tpl = recorded_traffic_per_launch(kernel, keys_per_step, moved) if not variant and not distance else None
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": tpl, "kernel": kernel,
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6650 GB/s",
                "algorithmic_bytes_per_launch": kernel_bytes, "ms_per_launch": round(kernel_ms, 5),
                "timing": f"CUDA events around {what}, {n_phase} live steps",
                "nominal_hbm_gbs": NOMINAL_HBM_GBS}
    step_bytes = k_bytes + moved_bytes
    step_achieved = step_bytes / (ms_per_step / 1e3) / 1e9
    phases = {"query": round(statistics.mean(query_ms), 5), "score": round(score_mean, 5),
              "select_compact": round(statistics.mean(evict_ms), 5)}
    select_compact = {"kernel": "select_compact_kernel" if fused else "evict_kernel + move_kernel x2",
                      "ms": round(statistics.mean(evict_ms), 5), "moved_bytes": moved_bytes,
                      "achieved_moved_gbs": round(moved_bytes / (statistics.mean(evict_ms) / 1e3) / 1e9, 1)}
    upper_bytes = k_bytes + kept_rows * 4 * 256
    step_roofline = {"bound": "hbm", "achieved": round(step_achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(step_achieved / peak, 4), "bytes_per_step": step_bytes,
                     "moved_rows": moved, "phase_ms_serialised": phases, "select_compact": select_compact,
                     "upper_bound": {"moved_rows": kept_rows, "bytes_per_step": upper_bytes,
                                     "frac": round(upper_bytes / (ms_per_step / 1e3) / 1e9 / peak, 4),
                                     "note": "every kept row counted as moved"}}

    # ------------------------------------------------------------ e2e
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, tri, cache, wl, qbar, qabs, R, freed, count, save_k, save_v, rblocks,
                      save_len, keys_per_step, dev, world, dist, step)

    # ---------------------------------------------------- cpu baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if distance:
            cpu = run_cpu_baseline_distance(args, wl, cfg, save_k, save_v, rblocks, lens, max_dist)
        else:
            cpu = run_cpu_baseline(args, wl, cfg, save_k, save_v, rblocks, lens)

    clk = clocks.summary()
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": job["n_gpus"], "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": job["scaling"], "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": cfg.name, "L": L, "Hkv": Hkv, "G": G, "D": 128, "seq_lens": lens,
                   "budget": B, "window": W, "rope_base": cfg.base, "deltas": wl.deltas,
                   "sinks": args.sinks, "trigger": trig, "aggregate": args.aggregate,
                   "score_mode": args.score_mode, "distance_table_build_ms": table_ms,
                   "keys_per_step_per_gpu": keys_per_step, "freed_blocks_per_step": job_freed,
                   "parallelism": (f"KV heads split over {world} GPUs ({cfg.Hkv} per GPU), freed-block "
                                   f"counts all-reduced (equal on every rank: {freed_same})" if heads_mode else
                                   f"units sharded: one independent cache per GPU x{world}"),
                   "input_dtype": "bf16 K/V, fp32 arithmetic",
                   "l2": flush.describe(),
                   "launch": "CUDA graph replay of one captured step" if args.graph else "direct calls",
                   "kernels": kernel_list(fused, distance),
                   "timing": "CUDA events around each tri_compress_step; kept-region restore and L2 flush "
                             "untimed; per-phase times from a separate live loop with phase events"},
        "roofline": roofline, "step_roofline": step_roofline,
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step(fused) * args.steps, "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(out), flush=True)


def kernel_list(fused: bool, distance: bool) -> str:
    """The kernels one step launches, in order."""
    first = "query_kernel (plan only)" if distance else "query_kernel"
    middle = "distance_score_kernel" if distance else "score kernel"
    last = "select_compact_kernel" if fused else "evict_kernel, move_kernel x2"
    return f"{first}, {middle}, {last}"


def launches_per_step(fused: bool) -> int:
    """How many of the library's kernels one step launches (the same count
    for both score modes: the plan, one scoring kernel, then compaction)."""
    return 3 if fused else 5


def run_decode(args, world, rank, local, dist, cfg):
    """The decode-loop workload: sequences of drawn lengths in one shared
    paged pool; each round appends cfg.decode_append tokens to every
    sequence (blocks popped from the device free list by tri_reserve_blocks,
    rows written untimed), then one timed tri_compress_step_ex compresses
    every sequence and pushes the freed blocks back on the device list.  The
    host never reads freed ids.  Reports every round."""
    import torch
    import rope_aware_kv_tri_b200 as tri
    from workload import make_workload
    from workload.gen import write_tokens
    from rope_aware_kv_tri_b200.sharding import keys_per_second, reduce_job, shard_seed
    dev = torch.device("cuda", local)
    wl = make_workload(cfg, device=dev, seed=shard_seed(cfg.seed, rank) if world > 1 else cfg.seed)
    L, Hkv, G, Hq, S = cfg.L, cfg.Hkv, cfg.G, cfg.Hq, cfg.S
    B, W = cfg.budget, cfg.window
    qbar = torch.empty(L, Hq, 128, device=dev)
    qabs = torch.empty(L, Hq, 64, device=dev)
    R = torch.empty(L, Hq, device=dev)
    tri.tri_calibrate_centers(wl.q_samples, qbar, qabs, R)
    cache = tri.KvCache(wl.k_pool, wl.v_pool, wl.block_table, wl.seq_len, wl.cur_pos,
                        torch.zeros(1, dtype=torch.int32, device=dev), G)
    opt = tri.step_options(B, W, args.sinks, args.trigger)
    fused = tri.tri_step_is_fused(cache, opt)
    ws = tri.alloc_workspace(cache, opt)
    fl = tri.FreeList.from_ids(wl.free_blocks, wl.num_blocks, dev)
    n_new = torch.full((S,), cfg.decode_append, dtype=torch.int32, device=dev)
    flush = L2Flush(args.l2_flush, dev)
    # kept slots of every unit (an optional output of the step), to count the
    # rows each round moves once the round is over
    idx = torch.empty(S, L, Hkv, B, dtype=torch.int32, device=dev)
    ident = torch.arange(B, dtype=torch.int32, device=dev)
    peak, peak_kind = measured_peak()
    rounds, total_ms, total_keys = [], 0.0, 0
    clocks = ClockSampler(local)
    clocks.start()
    for r in range(cfg.decode_rounds):
        tri.tri_reserve_blocks(cache, n_new, fl)
        lens = wl.seq_len.tolist()
        for s in range(S):
            write_tokens(wl, s, lens[s], cfg.decode_append)
        wl.seq_len += n_new
        wl.cur_pos += cfg.decode_append
        lens = wl.seq_len.tolist()
        free_before = int(fl.count.item())
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        pev = [torch.cuda.Event(enable_timing=True) for _ in range(4)] if args.phases else None
        torch.cuda.synchronize(dev)
        # the flush keeps the GPU busy while the host enqueues the step, as
        # in a decode loop whose host runs ahead of the GPU; without it the
        # round's events would also time the host's launch of the step
        flush()
        a.record()
        tri.tri_compress_step_ex(cache, qbar, qabs, R, cfg.base, wl.deltas, opt, ws, free_list=fl, idx_out=idx,
                                 events=pev)
        b.record()
        torch.cuda.synchronize(dev)
        if tri.tri_sync_status(cache.status) != tri.TRI_OK:
            raise RuntimeError(f"device status flag raised in decode round {r}")
        ms = a.elapsed_time(b)
        trig = max(args.trigger, B)
        compressed = [s for s in range(S) if lens[s] > trig]
        keys = sum(lens[s] for s in compressed) * L * Hkv
        moved = int((idx[compressed] != ident).sum().item()) if compressed else 0
        step_bytes = keys * 256 + moved * 4 * 256
        freed = int(fl.count.item()) - free_before
        rounds.append({"round": r, "keys": keys, "ms": round(ms, 4), "keys_per_s": round(keys / (ms / 1e3), 1),
                       "k_read_gbs": round(keys * 256 / (ms / 1e3) / 1e9, 1), "moved_rows": moved,
                       "step_bytes": step_bytes, "step_gbs": round(step_bytes / (ms / 1e3) / 1e9, 1),
                       "frac": round(step_bytes / (ms / 1e3) / 1e9 / peak, 4), "freed_blocks": freed,
                       "mean_len_before": round(sum(lens) / S, 1),
                       "kept_rows": len(compressed) * L * Hkv * B})
        if pev is not None:
            rounds[-1]["phase_ms"] = {"query": round(pev[0].elapsed_time(pev[1]), 4),
                                      "score": round(pev[1].elapsed_time(pev[2]), 4),
                                      "select_compact": round(pev[2].elapsed_time(pev[3]), 4)}
        total_ms += ms
        total_keys += keys
    clocks.stop()
    t_job, k_job, _ = reduce_job(dist, total_ms, total_keys, 0, dev)
    value = keys_per_second(k_job, 1, t_job)
    steady = rounds[1:] if len(rounds) > 1 else rounds
    steady_ms = sum(x["ms"] for x in steady)
    steady_bytes = sum(x["step_bytes"] for x in steady)
    all_bytes = sum(x["step_bytes"] for x in rounds)
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": cfg.decode_rounds,
        "warmup": 0, "ms_per_step": round(t_job / cfg.decode_rounds, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": cfg.name, "L": L, "Hkv": Hkv, "G": G, "D": 128, "sequences": S,
                   "budget": B, "window": W, "append_per_round": cfg.decode_append,
                   "free_list": "device (tri_reserve_blocks pops, the step pushes; no host read of freed ids)",
                   "l2": flush.describe(),
                   "kernels": kernel_list(fused, False),
                   "timing": "CUDA events around each round's tri_compress_step_ex; appends untimed",
                   "rounds": rounds},
        "roofline": {"bound": "hbm", "achieved": round(all_bytes / (total_ms / 1e3) / 1e9, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(all_bytes / (total_ms / 1e3) / 1e9 / peak, 4),
                     "traffic": None, "kernel": "whole step (score + select + compaction)",
                     "bytes": "per round: cached keys x 256 B read + moved rows x 1024 B (K and V read and "
                              "written), summed over the rounds",
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                     else "fallback 6650 GB/s",
                     "steady_rounds": {"rounds": len(steady), "ms_mean": round(steady_ms / max(len(steady), 1), 4),
                                       "moved_rows_mean": round(sum(x["moved_rows"] for x in steady)
                                                                / max(len(steady), 1), 1),
                                       "achieved": round(steady_bytes / (steady_ms / 1e3) / 1e9, 1),
                                       "frac": round(steady_bytes / (steady_ms / 1e3) / 1e9 / peak, 4),
                                       "frac_upper_bound": round(
                                           sum(x["keys"] * 256 + x["kept_rows"] * 1024 for x in steady)
                                           / (steady_ms / 1e3) / 1e9 / peak, 4) if steady else None},
                     "achieved_k_read_first_round": rounds[0]["k_read_gbs"] if rounds else None},
        "gpu_launches": launches_per_step(fused) * cfg.decode_rounds, "clocks": clocks.summary(),
    }
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_e2e(args, tri, cache, wl, qbar, qabs, R, freed, count, save_k, save_v, rblocks, save_len,
            keys_per_step, dev, world, dist, step):
    """Same step through the C ABI with the cache in pinned HOST memory: the
    timed region copies the inputs in, runs the step, and copies the result
    (the kept region of K/V, new lengths, freed ids and count) back."""
    import torch
    wl.k_pool[:, rblocks] = save_k
    wl.v_pool[:, rblocks] = save_v
    wl.seq_len.copy_(save_len)
    host = {n: t.to("cpu").pin_memory() for n, t in
            (("k", wl.k_pool), ("v", wl.v_pool), ("table", wl.block_table), ("len", save_len),
             ("pos", wl.cur_pos), ("qbar", qbar), ("qabs", qabs), ("R", R))}
    out_k = torch.empty_like(save_k, device="cpu").pin_memory()
    out_v = torch.empty_like(save_v, device="cpu").pin_memory()
    out_len = torch.empty_like(save_len, device="cpu").pin_memory()
    out_freed = torch.empty_like(freed, device="cpu").pin_memory()
    out_count = torch.empty(1, dtype=torch.int32).pin_memory()
    dev_in = {"k": wl.k_pool, "v": wl.v_pool, "table": wl.block_table, "len": wl.seq_len, "pos": wl.cur_pos,
              "qbar": qbar, "qabs": qabs, "R": R}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in (out_k, out_v, out_len, out_freed, out_count))
    times = []
    for k in range(args.e2e_steps + 1):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record()
        for n, t in host.items():
            dev_in[n].copy_(t, non_blocking=True)
        step()
        out_k.copy_(wl.k_pool[:, rblocks], non_blocking=True)
        out_v.copy_(wl.v_pool[:, rblocks], non_blocking=True)
        out_len.copy_(wl.seq_len, non_blocking=True)
        out_freed.copy_(freed, non_blocking=True)
        out_count.copy_(count, non_blocking=True)
        b.record()
        torch.cuda.synchronize(dev)
        if k > 0:                      # first call is a warm-up
            times.append(a.elapsed_time(b))
    if tri.tri_sync_status(cache.status) != tri.TRI_OK:
        raise RuntimeError("device status flag raised during the end-to-end steps")
    from rope_aware_kv_tri_b200.sharding import reduce_job, keys_per_second
    total, job_keys, _ = reduce_job(dist, sum(times), keys_per_step, 0, dev)
    del host
    return {"value": round(keys_per_second(job_keys, len(times), total), 1), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": len(times),
            "ms_per_step": round(total / len(times), 3)}


def run_cpu_baseline(args, wl, cfg, save_k, save_v, rblocks, lens):
    """The float64 oracle on a bounded sample of this workload's units
    (restored, untouched inputs): the plain C oracle one unit per host thread
    on every core, with its one-thread figure and the numpy oracle's beside it."""
    import numpy as np
    import torch
    import oracle
    wl.k_pool[:, rblocks] = save_k
    wl.v_pool[:, rblocks] = save_v
    table = wl.block_table.cpu().tolist()
    rng = np.random.default_rng(1)
    G = cfg.G
    calib = {}

    def stats_fn(l, h):
        if (l, h) not in calib:
            if wl.q_samples is not None:
                calib[(l, h)] = oracle.calibrate(wl.q_samples[:, l, h * G:(h + 1) * G].double().cpu().numpy())
            else:
                sl = slice(h * G, (h + 1) * G)
                calib[(l, h)] = tuple(t[l, sl].double().cpu().numpy() for t in (wl.qbar, wl.qabs, wl.R))
        return calib[(l, h)]

    def units():
        while True:
            s = int(rng.integers(cfg.S))
            l = int(rng.integers(cfg.L))
            h = int(rng.integers(cfg.Hkv))
            n = lens[s]
            yield (unit_rows(wl.k_pool, table[s], n, l, h).cpu(), unit_rows(wl.v_pool, table[s], n, l, h).cpu(),
                   (s, l, h), int(wl.cur_pos[s].item()))

    threads = os.cpu_count() or 1
    keys, secs, n = c_oracle_sample(units(), stats_fn, wl.deltas, cfg.base, cfg.budget, cfg.window,
                                    args.cpu_seconds, threads, args.sinks, args.aggregate)
    c1, cs1, cn1 = c_oracle_sample(units(), stats_fn, wl.deltas, cfg.base, cfg.budget, cfg.window,
                                   min(3.0, args.cpu_seconds), 1, args.sinks, args.aggregate)
    k1, s1, n1 = oracle_sample(units(), stats_fn, wl.deltas, cfg.base, cfg.budget, cfg.window,
                               min(4.0, args.cpu_seconds), args.sinks, args.aggregate)
    return {"value": round(keys / secs, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": (f"{n} random units of this workload ({keys} keys), plain C float64 oracle, one unit per "
                       f"host thread on {threads} threads (wall time; inputs prepared untimed)"),
            "seconds": round(secs, 2), "cpu_model": host_cpu_model(),
            "c_oracle_1_thread": {"value": round(c1 / cs1, 1), "units": cn1, "seconds": round(cs1, 2)},
            "numpy_oracle_1_thread": {"value": round(k1 / s1, 1), "units": n1, "seconds": round(s1, 2)}}


def distance_oracle_sample(wl, cfg, lens, tables, pairs, seconds, sinks, trigger, rng):
    """Time the numpy oracle's distance-table step (lookup, selection,
    compaction of rows and positions) on units of the compressed sequences,
    cycling over the (layer, KV head) pairs whose tables are given, until
    about ``seconds`` have passed.  Returns (keys, seconds, units)."""
    import numpy as np
    import torch
    import oracle
    table = wl.block_table.cpu().tolist()
    trig = max(trigger, cfg.budget)
    seqs = [s for s in range(cfg.S) if lens[s] > trig]
    keys, secs, n = 0, 0.0, 0
    while seqs and secs < seconds:
        s = seqs[int(rng.integers(len(seqs)))]
        l, h = pairs[n % len(pairs)]
        length, p = lens[s], int(wl.cur_pos[s].item())
        kb = unit_rows(wl.k_pool, table[s], length, l, h).cpu().view(torch.int16).numpy()
        vb = unit_rows(wl.v_pool, table[s], length, l, h).cpu().view(torch.int16).numpy()
        pos = np.arange(length, dtype=np.int64)
        t0 = time.perf_counter()
        sc = oracle.distance_scores(tables[(l, h)], p, pos)
        idx = oracle.select(sc, length, cfg.budget, cfg.window, sinks)
        oracle.compact_rows(kb, idx)
        oracle.compact_rows(vb, idx)
        oracle.compact_rows(pos, idx)
        secs += time.perf_counter() - t0
        keys += length
        n += 1
    return keys, secs, n


def run_cpu_baseline_distance(args, wl, cfg, save_k, save_v, rblocks, lens, max_dist):
    """The distance-only variant's step in the float64 numpy oracle on units
    of this workload, one host core: each unit's scores looked up from its
    (layer, KV head) table, selection, and compaction of rows and positions.
    The tables of two sampled (layer, KV head) pairs are built once from the
    oracle's calibration of the query samples and the workload's key centres,
    outside the timed region (as the device builds its tables once)."""
    import numpy as np
    import torch
    import oracle
    wl.k_pool[:, rblocks] = save_k
    wl.v_pool[:, rblocks] = save_v
    rng = np.random.default_rng(1)
    G = cfg.G
    pairs = [(int(rng.integers(cfg.L)), int(rng.integers(cfg.Hkv))) for _ in range(2)]
    tables = {}
    for l, h in pairs:
        if wl.q_samples is not None:
            qb = oracle.calibrate(wl.q_samples[:, l, h * G:(h + 1) * G].double().cpu().numpy())[0]
        else:
            qb = wl.qbar[l, h * G:(h + 1) * G].double().cpu().numpy()
        tables[(l, h)] = oracle.distance_table(qb, wl.key_centres[l, h].double().cpu().numpy(), wl.deltas,
                                               cfg.base, max_dist, args.aggregate)
    keys, secs, n = distance_oracle_sample(wl, cfg, lens, tables, pairs, args.cpu_seconds, args.sinks,
                                           args.trigger, rng)
    if n == 0:
        return None
    return {"value": round(keys / secs, 1), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": (f"{n} units of this workload ({keys} keys) on {len(pairs)} (layer, KV head) tables built "
                       f"once untimed; float64 numpy oracle: table lookup, selection, compaction of rows and "
                       f"positions, 1 thread; host has {os.cpu_count()} cores"),
            "seconds": round(secs, 2), "cpu_model": host_cpu_model()}


# ---------------------------------------------------------- reference arm

def run_reference(args, world, rank):
    """The float64 CPU oracle as the reference arm (no GPU use)."""
    if rank != 0:
        return
    import numpy as np
    import torch
    import oracle
    from workload import CONFIGS, make_workload
    cfg = CONFIGS[args.workload]
    # The same per-unit shape and distributions as the full workload, one
    # layer of it generated on the host.
    small = cfg.replace(L=1, n_samples=min(cfg.n_samples, 1024))
    wl = make_workload(small, device="cpu", seed=0)
    G = cfg.G
    if wl.qbar is not None:
        stats = tuple(t.double().numpy() for t in (wl.qbar, wl.qabs, wl.R))
    else:
        stats = oracle.calibrate(wl.q_samples.double().numpy())
    table = wl.block_table.tolist()
    lens = wl.seq_len.tolist()
    per_step = max(args.cpu_seconds / max(args.steps + args.warmup, 1), 0.5)

    def units():
        h = 0
        while True:
            s = h % cfg.S
            hh = h % cfg.Hkv
            n = lens[s]
            k = oracle.unit_rows(wl.k_pool.view(torch.int16).numpy(), table[s], n, 0, hh)
            v = oracle.unit_rows(wl.v_pool.view(torch.int16).numpy(), table[s], n, 0, hh)
            yield (torch.from_numpy(k).view(torch.bfloat16), torch.from_numpy(v).view(torch.bfloat16),
                   (s, 0, hh), int(wl.cur_pos[s]))
            h += 1

    def stats_fn(l, h):
        return stats[0][0, h * G:(h + 1) * G], stats[1][0, h * G:(h + 1) * G], stats[2][0, h * G:(h + 1) * G]

    it = units()
    threads = os.cpu_count() or 1
    distance = args.score_mode == "distance"
    if distance:
        # the distance-only variant: tables of two KV heads, built once untimed
        threads = 1
        pairs = [(0, h) for h in range(min(2, cfg.Hkv))]
        max_dist = int(wl.cur_pos.max().item()) + 1
        tables = {(l, h): oracle.distance_table(stats_fn(l, h)[0], wl.key_centres[l, h].double().numpy(),
                                                wl.deltas, cfg.base, max_dist, args.aggregate) for l, h in pairs}
        drng = np.random.default_rng(1)

    def sample_once(seconds):
        if distance:
            return distance_oracle_sample(wl, cfg, lens, tables, pairs, seconds, args.sinks, args.trigger, drng)
        return c_oracle_sample(it, stats_fn, wl.deltas, cfg.base, cfg.budget, cfg.window, seconds, threads,
                               args.sinks, args.aggregate)

    for _ in range(args.warmup):
        sample_once(0.0)
    keys = secs = 0.0
    n_units = 0
    for _ in range(args.steps):
        k, s_, n = sample_once(per_step)
        keys += k
        secs += s_
        n_units += n
    value = keys / secs
    kind = ("float64 numpy oracle, distance-table lookup, selection and compaction, 1 thread (tables of "
            f"{len(pairs)} KV heads built once, untimed)" if distance else
            f"plain C float64 oracle, one unit per host thread on {threads} threads")
    sample = f"{n_units} units of the {cfg.name} workload shape over {args.steps} steps, {kind}"
    out = {"impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * secs / args.steps, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": cfg.name, "L": cfg.L, "Hkv": cfg.Hkv, "G": cfg.G, "D": 128,
                      "seq_lens": cfg.lens, "budget": cfg.budget, "window": cfg.window, "sinks": args.sinks,
                      "aggregate": args.aggregate, "score_mode": args.score_mode},
           "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
                            "sample": sample, "cpu_model": host_cpu_model()},
           "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main(argv=None, runner=None, backend="nccl"):
    """``runner(args, world, rank, local, dist)`` runs one rank's measurement
    (default: run_ours)."""
    args = parse_args(argv)
    if args.impl != "reference" and args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        code = spawn_ranks(args, argv if argv is not None else sys.argv[1:], runner, backend)
        if code:
            raise SystemExit(code)
        return
    world, rank, local, dist = dist_setup(args, backend)
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    try:
        (runner or run_ours)(args, world, rank, local, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
