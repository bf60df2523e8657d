"""GPU parity of the step's variants against the float64 oracle.

* attention sinks and the compression trigger in the selection (bit-exact on
  the same fp32 scores, every selection path: one-pass, two-pass, streaming);
* the max-over-group aggregation of the score (G = 1, 2, 4, 8);
* tri_compress_step_ex with sinks, trigger and either aggregation, checked
  like the plain step (lengths, freed ids, kept slots, rows moved bit-exact);
* the device free list: the step pushes its freed ids, tri_reserve_blocks pops
  blocks for appended slots (all or nothing), and a decode loop that never
  reads freed ids back on the host stays equal to the oracle's world.
"""

import numpy as np
import pytest
import torch

import oracle
import rope_aware_kv_tri_b200 as tri
from tests.gpu_helpers import (cache_of, check_scores, check_selection, expected_pools_after, freed_expected,
                               gpu_stats, oracle_stats, oracle_unit_scores, status_tensor, unit_rows)
from tests.test_gpu_parity import SMALL, _score_fill
from workload import CONFIGS, make_workload
from workload.decode import append_tokens, recycle_freed

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rope_aware_kv_tri_b200 import build_lib
    build_lib.build()
    torch.cuda.init()


# ------------------------------------------------------------ selection

@pytest.mark.parametrize("budget,window,sinks", [(64, 8, 1), (64, 8, 2), (64, 8, 3), (64, 8, 4), (64, 0, 5),
                                                 (64, 8, 56), (2048, 128, 4), (2048, 128, 7), (1, 0, 1)])
def test_select_sinks_bit_exact_on_same_scores(budget, window, sinks):
    rng = np.random.default_rng(budget * 7 + window * 3 + sinks)
    lens = [0, 1, budget, budget + 1, 3 * budget + 5, 40000, 777, 5000, 140000]
    kinds = ["normal", "ties", "zeros", "wide", "dups"]
    S, L, Hkv = len(lens), 1, len(kinds)
    max_blocks = -(-max(lens) // 16)
    k = torch.zeros(1, 1, Hkv, 16, 128, dtype=torch.bfloat16, device=DEV)
    cache = tri.KvCache(k, k.clone(), torch.zeros(S, max_blocks, dtype=torch.int32, device=DEV),
                        torch.tensor(lens, dtype=torch.int32, device=DEV), torch.zeros(S, dtype=torch.int64, device=DEV),
                        status_tensor(DEV), 1)
    sc = np.full((S, L, Hkv, max_blocks * 16), np.nan, dtype=np.float32)
    for s, n in enumerate(lens):
        for h in range(Hkv):
            sc[s, 0, h, :n] = _score_fill(rng, n, kinds[h])
            if n > 8:
                sc[s, 0, h, :min(sinks, n)] = 1e30        # sinks score highest: must not take a ranked place
    idx = torch.full((S, L, Hkv, budget), -7, dtype=torch.int32, device=DEV)
    kept = torch.full((S,), -7, dtype=torch.int32, device=DEV)
    tri.tri_select_topk_ex(cache, torch.from_numpy(sc).to(DEV), tri.step_options(budget, window, sinks), idx, kept)
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    idx, kept = idx.cpu().numpy(), kept.cpu().numpy()
    for s, n in enumerate(lens):
        assert kept[s] == min(n, budget)
        for h in range(Hkv):
            ref = oracle.select(sc[s, 0, h, :n].astype(np.float64), n, budget, window, sinks)
            assert np.array_equal(idx[s, 0, h, :kept[s]], ref), (s, h, n)


def test_select_trigger_keeps_short_units():
    budget, window, trigger = 64, 8, 200
    lens = [10, 64, 65, 200, 201, 1000]
    rng = np.random.default_rng(11)
    S = len(lens)
    mb = -(-max(lens) // 16)
    k = torch.zeros(1, 1, 1, 16, 128, dtype=torch.bfloat16, device=DEV)
    cache = tri.KvCache(k, k.clone(), torch.zeros(S, mb, dtype=torch.int32, device=DEV),
                        torch.tensor(lens, dtype=torch.int32, device=DEV), torch.zeros(S, dtype=torch.int64, device=DEV),
                        status_tensor(DEV), 1)
    sc = rng.normal(size=(S, 1, 1, mb * 16)).astype(np.float32)
    idx = torch.full((S, 1, 1, budget), -7, dtype=torch.int32, device=DEV)
    kept = torch.full((S,), -7, dtype=torch.int32, device=DEV)
    tri.tri_select_topk_ex(cache, torch.from_numpy(sc).to(DEV), tri.step_options(budget, window, 2, trigger),
                           idx, kept)
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    assert kept.cpu().tolist() == [10, 64, 65, 200, 64, 64]
    idx = idx.cpu().numpy()
    for s, n in enumerate(lens):
        if n <= trigger:
            m = min(n, budget)
            assert np.array_equal(idx[s, 0, 0, :m], np.arange(m))
            assert np.all(idx[s, 0, 0, m:] == -1)
        else:
            ref = oracle.select(sc[s, 0, 0, :n].astype(np.float64), n, budget, window, 2)
            assert np.array_equal(idx[s, 0, 0], ref)


# ----------------------------------------------------------------- score

MAX_CASES = {
    # CUDA-core kernel (G = 1, or KV heads not a multiple of 8)
    "head1_t4096": SMALL["head1_t4096"],
    "hkv4": SMALL["hkv4"],
    "hkv4_g4": CONFIGS["l32h8_t32k"].replace(L=1, Hkv=4, G=4, lens=[1025, 300], n_samples=256, table="shuffled"),
    "hkv2_g8": CONFIGS["l64h8g8_4x64k"].replace(L=1, Hkv=2, G=8, lens=[777, 16, 0], n_samples=256),
    # tensor-core kernel (8 KV heads per tile, G = 2, 4, 8)
    "hkv8_g2": CONFIGS["l32h8_t32k"].replace(L=2, Hkv=8, G=2, lens=[2000, 700, 1], n_samples=256, table="shuffled"),
    "l2h8g4_t3001": SMALL["l2h8g4_t3001"],
    "l2h8g8_ragged6": SMALL["l2h8g8_ragged6"],
    "hkv16_g4": CONFIGS["l32h8_t32k"].replace(L=1, Hkv=16, G=4, lens=[900, 33], n_samples=256, table="shuffled"),
}


@pytest.mark.parametrize("name", list(MAX_CASES))
def test_score_max_over_group_matches_oracle(name):
    wl = make_workload(MAX_CASES[name], device=DEV, seed=4)
    stats = gpu_stats(wl)
    ref_stats = oracle_stats(wl)
    cache = cache_of(wl)
    S, L, Hkv = wl.cfg.S, wl.cfg.L, wl.cfg.Hkv
    max_len = wl.max_blocks * 16
    sentinel = -4321.25
    scores = torch.full((S, L, Hkv, max_len), sentinel, device=DEV)
    ws = tri.alloc_workspace(cache, tri.step_options(1, 0, aggregate=tri.TRI_AGG_MAX))
    tri.tri_score_ex(cache, *stats, wl.cfg.base, wl.deltas, tri.TRI_AGG_MAX, scores, ws)
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    sc = scores.cpu().numpy()
    table = wl.block_table.cpu().tolist()
    worst = 0.0
    for s in range(S):
        n = int(wl.seq_len[s])
        assert np.all(sc[s, :, :, n:] == sentinel)
        for l in range(L):
            for h in range(Hkv):
                keys = unit_rows(wl.k_pool, table[s], n, l, h)
                ref = oracle_unit_scores(wl, keys, ref_stats, s, l, h, aggregate="max")
                worst = max(worst, check_scores(sc[s, l, h, :n], ref))
    print(f"{name}: worst max-score error / floor = {worst:.2e}")


# ---------------------------------------------------------- the step

VARIANTS = [
    dict(sinks=4, trigger=0, aggregate=tri.TRI_AGG_MEAN),
    dict(sinks=3, trigger=600, aggregate=tri.TRI_AGG_MEAN),
    dict(sinks=5, trigger=0, aggregate=tri.TRI_AGG_MAX),
    dict(sinks=0, trigger=1000, aggregate=tri.TRI_AGG_MAX),
    dict(sinks=448, trigger=0, aggregate=tri.TRI_AGG_MEAN),     # sinks + window = budget: nothing ranked
]


@pytest.mark.parametrize("var", VARIANTS, ids=[f"s{v['sinks']}_t{v['trigger']}_a{v['aggregate']}" for v in VARIANTS])
def test_compress_step_ex_matches_oracle(var):
    wl = make_workload(SMALL["l2h8g8_ragged6"], device=DEV, seed=6)
    budget, window = wl.cfg.budget, wl.cfg.window
    opt = tri.step_options(budget, window, **var)
    agg = "max" if var["aggregate"] == tri.TRI_AGG_MAX else "mean"
    trig = max(var["trigger"], budget)
    stats = gpu_stats(wl)
    ref_stats = oracle_stats(wl)
    S, L, Hkv = wl.cfg.S, wl.cfg.L, wl.cfg.Hkv
    lens = wl.seq_len.cpu().tolist()
    kept = [budget if n > trig else n for n in lens]
    table = wl.block_table.cpu().tolist()
    pk, pv = wl.k_pool.clone(), wl.v_pool.clone()
    cache = cache_of(wl)
    ws = tri.alloc_workspace(cache, opt)
    freed = torch.full((S * wl.max_blocks,), -7, dtype=torch.int32, device=DEV)
    count = torch.full((1,), -7, dtype=torch.int32, device=DEV)
    idx = torch.full((S, L, Hkv, budget), -7, dtype=torch.int32, device=DEV)
    tri.tri_compress_step_ex(cache, *stats, wl.cfg.base, wl.deltas, opt, ws, freed_ids=freed, freed_count=count,
                             idx_out=idx)
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    assert wl.seq_len.cpu().tolist() == kept
    n_freed = int(count.item())
    assert freed[:n_freed].cpu().tolist() == freed_expected(wl.block_table, lens, kept)
    differ = 0
    for s, n in enumerate(lens):
        for l in range(L):
            for h in range(Hkv):
                if n <= trig:
                    assert torch.all(idx[s, l, h] == -7), "idx written for an untouched sequence"
                    continue
                ref = oracle_unit_scores(wl, unit_rows(pk, table[s], n, l, h), ref_stats, s, l, h, aggregate=agg)
                differ += check_selection(idx[s, l, h].cpu().numpy(), ref, n, budget, window, sinks=var["sinks"])
    ek, ev = expected_pools_after(pk, pv, wl.block_table, lens, idx, kept)
    assert torch.equal(wl.k_pool.view(torch.int16), ek.view(torch.int16))
    assert torch.equal(wl.v_pool.view(torch.int16), ev.view(torch.int16))
    print(f"{var}: {differ} kept slots differ from the oracle inside the cut band")


def test_compress_step_ex_defaults_equal_plain_step():
    """{B, W, 0, 0, mean} through the _ex entry is the plain step, bit for bit."""
    a = make_workload(SMALL["hkv6"], device=DEV, seed=7)
    b = make_workload(SMALL["hkv6"], device=DEV, seed=7)
    budget, window = a.cfg.budget, a.cfg.window
    outs = []
    for wl, ex in ((a, False), (b, True)):
        cache = cache_of(wl)
        stats = gpu_stats(wl)
        ws = tri.alloc_workspace(cache, budget)
        freed = torch.zeros(wl.cfg.S * wl.max_blocks, dtype=torch.int32, device=DEV)
        count = torch.zeros(1, dtype=torch.int32, device=DEV)
        idx = torch.zeros(wl.cfg.S, wl.cfg.L, wl.cfg.Hkv, budget, dtype=torch.int32, device=DEV)
        if ex:
            tri.tri_compress_step_ex(cache, *stats, wl.cfg.base, wl.deltas, tri.step_options(budget, window), ws,
                                     freed_ids=freed, freed_count=count, idx_out=idx)
        else:
            tri.tri_compress_step(cache, *stats, wl.cfg.base, wl.deltas, budget, window, freed, count, ws,
                                  idx_out=idx)
        assert tri.tri_sync_status(cache.status) == tri.TRI_OK
        outs.append((idx, freed[:int(count.item())].clone(), wl.seq_len.clone()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    assert torch.equal(outs[0][2], outs[1][2])
    assert torch.equal(a.k_pool.view(torch.int16), b.k_pool.view(torch.int16))
    assert torch.equal(a.v_pool.view(torch.int16), b.v_pool.view(torch.int16))


# ------------------------------------------------------------ free list

def _unused_blocks(wl):
    used = set()
    table = wl.block_table.cpu().tolist()
    for s, n in enumerate(wl.seq_len.cpu().tolist()):
        used.update(table[s][:-(-n // 16)])
    return [b for b in range(wl.k_pool.shape[1]) if b not in used]


def _expected_reserve(table, lens, n_new, free):
    """Blocks each sequence takes: the top `total` entries of the stack, in
    sequence order then table order, from the lowest popped entry up."""
    table = [row[:] for row in table]
    needs = [-(-(n + a) // 16) - (-(-n // 16)) for n, a in zip(lens, n_new)]
    total = sum(needs)
    base = len(free) - total
    pos = base
    for s, need in enumerate(needs):
        lo = -(-lens[s] // 16)
        for e in range(need):
            table[s][lo + e] = free[pos]
            pos += 1
    return table, free[:base]


def test_free_list_push_and_reserve():
    wl = make_workload(SMALL["l2h8g8_ragged6"], device=DEV, seed=8)
    budget, window = wl.cfg.budget, wl.cfg.window
    NB = wl.k_pool.shape[1]
    free0 = _unused_blocks(wl)
    fl = tri.FreeList.from_ids(free0, NB, DEV)
    lens = wl.seq_len.cpu().tolist()
    kept = [min(n, budget) for n in lens]
    cache = cache_of(wl)
    stats = gpu_stats(wl)
    ws = tri.alloc_workspace(cache, budget)
    freed = torch.zeros(wl.cfg.S * wl.max_blocks, dtype=torch.int32, device=DEV)
    count = torch.zeros(1, dtype=torch.int32, device=DEV)
    tri.tri_compress_step_ex(cache, *stats, wl.cfg.base, wl.deltas, tri.step_options(budget, window), ws,
                             free_list=fl, freed_ids=freed, freed_count=count)
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    want_freed = freed_expected(wl.block_table, lens, kept)
    assert freed[:int(count.item())].cpu().tolist() == want_freed
    assert fl.contents() == free0 + want_freed
    # grow every sequence; blocks come from the top of the stack
    lens = wl.seq_len.cpu().tolist()
    n_new = [20, 0, 15, 100, 3, 16]
    want_table, want_free = _expected_reserve(wl.block_table.cpu().tolist(), lens, n_new, fl.contents())
    tri.tri_reserve_blocks(cache, torch.tensor(n_new, dtype=torch.int32, device=DEV), fl)
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    assert wl.block_table.cpu().tolist() == want_table
    assert fl.contents() == want_free
    assert wl.seq_len.cpu().tolist() == lens                  # lengths are the caller's to raise
    # too many slots for the list: nothing changes
    before_table, before_free = wl.block_table.clone(), fl.contents()
    lens = wl.seq_len.cpu().tolist()
    huge = [wl.max_blocks * 16 - n for n in lens]             # fills every table, more than the list holds
    assert sum(wl.max_blocks - (-(-n // 16)) for n in lens) > len(before_free)
    tri.tri_reserve_blocks(cache, torch.tensor(huge, dtype=torch.int32, device=DEV), fl)
    assert tri.tri_sync_status(cache.status) == tri.TRI_ERR_FREELIST
    assert torch.equal(wl.block_table, before_table) and fl.contents() == before_free
    # past the table's capacity: nothing changes either
    over = [wl.max_blocks * 16 - lens[0] + 1, 0, 0, 0, 0, 0]
    tri.tri_reserve_blocks(cache, torch.tensor(over, dtype=torch.int32, device=DEV), fl)
    assert tri.tri_sync_status(cache.status) == tri.TRI_ERR_DEVICE_BOUNDS
    assert torch.equal(wl.block_table, before_table) and fl.contents() == before_free


def test_free_list_push_without_room_is_flagged():
    wl = make_workload(SMALL["l2h8g8_ragged6"], device=DEV, seed=9)
    budget, window = wl.cfg.budget, wl.cfg.window
    lens = wl.seq_len.cpu().tolist()
    kept = [min(n, budget) for n in lens]
    want_freed = freed_expected(wl.block_table, lens, kept)
    assert len(want_freed) > 1
    ids = torch.full((len(want_freed) + 1,), -3, dtype=torch.int32, device=DEV)
    fl = tri.FreeList(ids, torch.tensor([2], dtype=torch.int32, device=DEV))   # room for all but one
    cache = cache_of(wl)
    ws = tri.alloc_workspace(cache, budget)
    freed = torch.zeros(wl.cfg.S * wl.max_blocks, dtype=torch.int32, device=DEV)
    count = torch.zeros(1, dtype=torch.int32, device=DEV)
    tri.tri_compress_step_ex(cache, *gpu_stats(wl), wl.cfg.base, wl.deltas, tri.step_options(budget, window), ws,
                             free_list=fl, freed_ids=freed, freed_count=count)
    assert tri.tri_sync_status(cache.status) == tri.TRI_ERR_FREELIST
    assert int(fl.count.item()) == 2 and torch.all(ids == -3)
    assert freed[:int(count.item())].cpu().tolist() == want_freed       # still reported
    assert wl.seq_len.cpu().tolist() == kept                             # still compacted


def test_decode_loop_with_device_free_list_matches_oracle_world():
    """The GPU world grows its sequences with tri_reserve_blocks and
    compresses with a trigger and sinks, pushing freed blocks on the device
    list; the host never reads freed ids.  The oracle world uses the host
    allocator.  The worlds' block ids differ, so the rows of each unit are
    compared through each world's own table."""
    cfg = CONFIGS["decode16"].replace(L=2, Hkv=4, G=2, lens=[0] * 4, lens_range=(300, 700), budget=256, window=32,
                                  decode_append=64, decode_rounds=5, n_samples=256)
    sinks, trigger = 4, 256 + 64
    cpu = make_workload(cfg, device="cpu")
    G, budget, window, S = cfg.G, cfg.budget, cfg.window, cfg.S
    gk, gv = cpu.k_pool.to(DEV), cpu.v_pool.to(DEV)
    gtable, glen, gpos = cpu.block_table.to(DEV), cpu.seq_len.to(DEV), cpu.cur_pos.to(DEV)
    NB = gk.shape[1]
    fl = tri.FreeList.from_ids(list(cpu.free_blocks), NB, DEV)
    qbar = torch.empty(cfg.L, cfg.Hq, 128, device=DEV)
    qabs = torch.empty(cfg.L, cfg.Hq, 64, device=DEV)
    R = torch.empty(cfg.L, cfg.Hq, device=DEV)
    tri.tri_calibrate_centers(cpu.q_samples.to(DEV), qbar, qabs, R)
    rb, ra, rr = oracle.calibrate(cpu.q_samples.double().numpy())
    cache = tri.KvCache(gk, gv, gtable, glen, gpos, torch.zeros(1, dtype=torch.int32, device=DEV), G)
    opt = tri.step_options(budget, window, sinks, trigger)
    ws = tri.alloc_workspace(cache, opt)
    n_new = torch.full((S,), cfg.decode_append, dtype=torch.int32, device=DEV)
    idx = torch.empty(S, cfg.L, cfg.Hkv, budget, dtype=torch.int32, device=DEV)
    compressed_rounds = 0
    for rnd in range(cfg.decode_rounds):
        old = cpu.seq_len.tolist()
        for s in range(S):
            append_tokens(cpu, s, cfg.decode_append)
        tri.tri_reserve_blocks(cache, n_new, fl)
        gt = gtable.cpu()
        for s in range(S):                      # the new rows, into the GPU world's own blocks
            slots = torch.arange(old[s], old[s] + cfg.decode_append)
            cb, gb, row = cpu.block_table[s].long()[slots // 16], gt[s].long()[slots // 16], slots % 16
            gk[:, gb.to(DEV), :, row.to(DEV)] = cpu.k_pool[:, cb, :, row].to(DEV)
            gv[:, gb.to(DEV), :, row.to(DEV)] = cpu.v_pool[:, cb, :, row].to(DEV)
        glen += n_new
        gpos.copy_(cpu.cur_pos.to(DEV))
        lens = cpu.seq_len.tolist()
        tri.tri_compress_step_ex(cache, qbar, qabs, R, cfg.base, cpu.deltas, opt, ws, free_list=fl, idx_out=idx)
        assert tri.tri_sync_status(cache.status) == tri.TRI_OK
        res = oracle.compress_step(cpu.k_pool.double().numpy(), cpu.k_pool.view(torch.int16).numpy(),
                                   cpu.v_pool.view(torch.int16).numpy(), cpu.block_table.numpy(), lens,
                                   cpu.cur_pos.tolist(), rb, ra, rr, G, cpu.deltas, cfg.base, budget, window,
                                   sinks=sinks, trigger=trigger)
        cpu.k_pool.view(torch.int16).copy_(torch.from_numpy(res["k_pool"]))
        cpu.v_pool.view(torch.int16).copy_(torch.from_numpy(res["v_pool"]))
        cpu.seq_len.copy_(torch.tensor(res["seq_len"], dtype=torch.int32))
        recycle_freed(cpu, lens, torch.tensor(res["freed_ids"] + [0], dtype=torch.int32), len(res["freed_ids"]))
        compressed_rounds += any(n > trigger for n in lens)
        assert glen.cpu().tolist() == res["seq_len"]
        differ = 0
        for (s, l, h), sc in res["scores"].items():
            differ += check_selection(idx[s, l, h].cpu().numpy(), sc, lens[s], budget, window, sinks=sinks)
        if differ:
            # an in-tolerance tie at a cut: the worlds now hold different rows
            print(f"round {rnd}: worlds diverged inside the cut band ({differ} slots); stopping")
            return
        # the GPU world's blocks in use and its free list partition the pool
        new_len = res["seq_len"]
        gt = gtable.cpu().tolist()
        in_use = [b for s in range(S) for b in gt[s][:-(-new_len[s] // 16)]]
        assert sorted(in_use + fl.contents()) == list(range(NB))
        # every unit's rows: same content through each world's table
        ct = cpu.block_table.tolist()
        for s in range(S):
            for l in range(cfg.L):
                for h in range(cfg.Hkv):
                    a = unit_rows(gk, gt[s], new_len[s], l, h).cpu().view(torch.int16)
                    b = unit_rows(cpu.k_pool, ct[s], new_len[s], l, h).view(torch.int16)
                    assert torch.equal(a, b)
                    av = unit_rows(gv, gt[s], new_len[s], l, h).cpu().view(torch.int16)
                    bv = unit_rows(cpu.v_pool, ct[s], new_len[s], l, h).view(torch.int16)
                    assert torch.equal(av, bv)
    assert compressed_rounds >= 2
