"""The persistent select + compact kernel against the separate kernels (GPU).

After its score pass a step selects and compacts every unit in one
persistent kernel (select_compact.cu): the CTA that takes a unit selects
it, packs its at-risk prefix in place and moves its other kept rows.  With
TRI_UNFUSED_STEP=1 in the environment the same call runs the selection,
copy-out and move kernels one after the other instead.  Both must give the
same result bit for bit: kept slots, freed blocks and their order, new
lengths, every row of both pools, the device free list.  The separate-kernel
run happens in a child process (the switch is read once per process) on the
same seeded workload; pools are compared through exact checksums of every
unit's rows plus a full row-by-row comparison of sampled units.

Both paths are also checked against the oracle elsewhere; this file pins
them to each other on shapes that stress the persistent kernel:
ragged lengths, a shuffled table, several sequences (one short enough to be
left alone), sinks and a trigger, a free list, budgets 1024 to 8192 (one CTA
per SM above 4096), the maximum over the group, the headline 32-layer x
8-head T = 32768 shape, and the distance-table step (where the kernel also
carries each unit's slot positions with its rows).
"""

import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = {
    "ragged_sinks_trigger": dict(base="decode16", L=4, Hkv=8, G=2, lens=[0] * 6, lens_range=(1500, 9000),
                                 budget=1024, window=64, sinks=5, trigger=1200, n_samples=256),
    "short_and_long": dict(base="l32h8_t32k", L=2, Hkv=4, G=2, lens=[5000, 300, 12345, 1025], budget=1024,
                           window=128, sinks=0, trigger=0, n_samples=256),
    "budget_4096": dict(base="l32h8_t128k", L=2, lens=[20000, 70000], budget=4096, window=256, sinks=0,
                        trigger=0, n_samples=256),
    "budget_8192_max": dict(base="l64h8g8_4x64k", L=2, lens=[9000, 30000], budget=8192, window=128, sinks=0,
                            trigger=0, n_samples=256, aggregate="max"),
    "headline_32L_8H_T32768": dict(base="l32h8_t32k", sinks=0, trigger=0),
    "distance_table_step": dict(base="l32h8_t32k", L=4, lens=[32768, 9000, 1500], budget=2048, window=128, sinks=3,
                                trigger=0, n_samples=256, distance=True),
}


def run_case(name: str, out_path: str) -> None:
    """Run one case through tri_compress_step_ex (with a free list) and save
    what the step produced: kept slots, freed ids, lengths, free list,
    per-unit checksums of both pools and the raw rows of sampled units."""
    sys.path.insert(0, ROOT)
    import rope_aware_kv_tri_b200 as tri
    from tests.gpu_helpers import cache_of, gpu_stats, unit_rows
    from workload import CONFIGS, make_workload
    spec = dict(CASES[name])
    base = spec.pop("base")
    sinks, trigger = spec.pop("sinks"), spec.pop("trigger")
    agg = tri.TRI_AGG_MAX if spec.pop("aggregate", "mean") == "max" else tri.TRI_AGG_MEAN
    distance = spec.pop("distance", False)
    cfg = CONFIGS[base].replace(**spec)
    dev = "cuda"
    wl = make_workload(cfg, device=dev, seed=11)
    stats = gpu_stats(wl)
    cache = cache_of(wl)
    S, L, Hkv, B = cfg.S, cfg.L, cfg.Hkv, cfg.budget
    opt = tri.step_options(B, cfg.window, sinks, trigger, agg)
    ws = tri.alloc_workspace(cache, opt)
    fl = tri.FreeList.from_ids([7777777, 8888888], S * wl.max_blocks + 2, dev)
    freed = torch.full((S * wl.max_blocks,), -7, dtype=torch.int32, device=dev)
    count = torch.full((1,), -7, dtype=torch.int32, device=dev)
    idx = torch.full((S, L, Hkv, B), -7, dtype=torch.int32, device=dev)
    lens = wl.seq_len.cpu().tolist()
    slot_pos = None
    if distance:
        # the distance-table step: scores from a table of the centres, positions carried with the rows
        max_dist = int(wl.cur_pos.max().item()) + 1
        table = torch.empty(L, Hkv, max_dist + 1, device=dev)
        tri.tri_distance_table(stats[0], wl.key_centres.float().contiguous(), cfg.base, wl.deltas, tri.TRI_AGG_MEAN,
                               table)
        slot_pos = torch.arange(wl.max_blocks * 16, dtype=torch.int32, device=dev).repeat(S, L, Hkv, 1).contiguous()
        tri.tri_compress_step_distance(cache, table, slot_pos, opt, ws, free_list=fl, freed_ids=freed,
                                       freed_count=count, idx_out=idx)
    else:
        tri.tri_compress_step_ex(cache, *stats, cfg.base, wl.deltas, opt, ws, free_list=fl, freed_ids=freed,
                                 freed_count=count, idx_out=idx)
    code = tri.tri_sync_status(cache.status)
    n = int(count.item())
    table = wl.block_table.cpu().tolist()
    # exact checksums of every unit's first max(len) rows (int64 sums of
    # position-weighted 16-bit words: any moved, missing or extra row changes them)
    gen = torch.Generator(device=dev).manual_seed(5)
    w = torch.randint(1, 1 << 20, (128,), generator=gen, device=dev, dtype=torch.int64)
    sums = {}
    sample = {}
    for s in range(S):
        for l in range(L):
            for h in range(Hkv):
                for nm, pool in (("k", wl.k_pool), ("v", wl.v_pool)):
                    rows = unit_rows(pool, table[s], lens[s], l, h).view(torch.int16).long()
                    pos = torch.arange(rows.shape[0], device=dev, dtype=torch.int64)[:, None] + 1
                    sums[f"{nm}{s}.{l}.{h}"] = int((rows * w[None, :] * pos).sum().item())
                if (s, l, h) in ((0, 0, 0), (S - 1, L - 1, Hkv - 1), (S // 2, L // 2, Hkv // 2)):
                    sample[f"{s}.{l}.{h}"] = unit_rows(wl.k_pool, table[s], lens[s], l, h).view(torch.int16).cpu()
    torch.save({"code": code, "idx": idx.cpu(), "freed": freed[:n].cpu(), "len": wl.seq_len.cpu(),
                "fl": fl.contents(), "sums": sums, "sample": sample,
                "pos": slot_pos.cpu() if slot_pos is not None else None}, out_path)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rope_aware_kv_tri_b200 import build_lib
    build_lib.build()
    torch.cuda.init()


@pytest.mark.parametrize("name", list(CASES))
def test_persistent_compaction_equals_separate_kernels(name, tmp_path):
    fused = str(tmp_path / "fused.pt")
    unfused = str(tmp_path / "unfused.pt")
    run_case(name, fused)
    torch.cuda.synchronize()
    code = f"import sys; sys.path.insert(0, {ROOT!r}); from tests.test_gpu_select_compact import run_case; " \
           f"run_case({name!r}, {unfused!r})"
    env = dict(os.environ, TRI_UNFUSED_STEP="1")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    a, b = torch.load(fused), torch.load(unfused)
    assert a["code"] == 0 and b["code"] == 0
    assert torch.equal(a["idx"], b["idx"]), "kept slots differ"
    assert torch.equal(a["freed"], b["freed"]), "freed blocks differ"
    assert torch.equal(a["len"], b["len"]), "lengths differ"
    assert a["fl"] == b["fl"], "free lists differ"
    bad = [k for k in a["sums"] if a["sums"][k] != b["sums"][k]]
    assert not bad, f"{len(bad)} units' rows differ, e.g. {bad[:4]}"
    for k in a["sample"]:
        assert torch.equal(a["sample"][k], b["sample"][k]), k
    if a["pos"] is not None:
        assert torch.equal(a["pos"], b["pos"]), "carried positions differ"
