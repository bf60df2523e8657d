"""GPU parity of the distance-only variant against the float64 oracle.

* tri_distance_table against the oracle's table (mean and max over the
  group), to fp32 rounding of a float64 sum;
* tri_score_distance is a lookup: bit-exact against the same table read on
  the host, with out-of-range distances flagged;
* tri_compress_step_distance on a table made on the host (the oracle's, in
  fp32) that both sides use: selection, compaction, freed blocks and the
  compacted slot positions are bit-exact, for caches whose slots still equal
  their positions and for caches compacted before (positions with gaps);
* the same step at the benchmark's full size (32 layers x 8 KV heads,
  T = 32768), on the table tri_distance_table builds.
"""

import numpy as np
import pytest
import torch

import oracle
import rope_aware_kv_tri_b200 as tri
from tests.gpu_helpers import cache_of, expected_pools_after, freed_expected, gpu_stats
from tests.test_gpu_parity import SMALL
from workload import make_workload

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rope_aware_kv_tri_b200 import build_lib
    build_lib.build()
    torch.cuda.init()


def _centres(L, Hkv, G, seed):
    g = torch.Generator().manual_seed(seed)
    qbar = torch.randn(L, Hkv * G, 128, generator=g, dtype=torch.float64).float()
    kbar = torch.randn(L, Hkv, 128, generator=g, dtype=torch.float64).float()
    return qbar, kbar


@pytest.mark.parametrize("G,agg", [(2, "mean"), (4, "max"), (1, "mean"), (8, "max")])
def test_distance_table_matches_oracle(G, agg):
    L, Hkv, max_dist = 2, 3, 5000
    deltas, base = [1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096], 5e5
    qbar, kbar = _centres(L, Hkv, G, seed=G)
    table = torch.full((L, Hkv, max_dist + 1), np.nan, device=DEV)
    tri.tri_distance_table(qbar.to(DEV), kbar.to(DEV), base, deltas,
                           tri.TRI_AGG_MAX if agg == "max" else tri.TRI_AGG_MEAN, table)
    torch.cuda.synchronize()
    got = table.double().cpu().numpy()
    qb, kb = qbar.double().numpy(), kbar.double().numpy()
    for l in range(L):
        for h in range(Hkv):
            ref = oracle.distance_table(qb[l, h * G:(h + 1) * G], kb[l, h], deltas, base, max_dist, aggregate=agg)
            scale = float(np.max(np.abs(ref)))
            err = np.abs(got[l, h] - ref)
            assert np.all(err <= 1e-6 * np.abs(ref) + 1e-7 * scale), float((err / scale).max())


def _positions(wl, seed, gapped):
    """slot_pos [S][L][Hkv][max_len]: t for a fresh cache; for the sequences in
    `gapped`, sorted distinct positions below a query position moved ahead by
    the gaps (a cache compacted before)."""
    rng = np.random.default_rng(seed)
    S, L, Hkv = wl.cfg.S, wl.cfg.L, wl.cfg.Hkv
    max_len = wl.max_blocks * 16
    lens = wl.seq_len.cpu().tolist()
    pos = np.zeros((S, L, Hkv, max_len), dtype=np.int32)
    cur = wl.cur_pos.cpu().numpy().copy()
    for s in range(S):
        if s in gapped and lens[s] > 0:
            cur[s] = lens[s] + 3 * lens[s] + 7
            for l in range(L):
                for h in range(Hkv):
                    pos[s, l, h, :lens[s]] = np.sort(rng.choice(cur[s], lens[s], replace=False))
        else:
            pos[s, :, :, :lens[s]] = np.arange(lens[s], dtype=np.int32)
    wl.cur_pos.copy_(torch.from_numpy(cur))
    return pos


def test_score_distance_is_a_lookup_and_flags_bad_distances():
    wl = make_workload(SMALL["l2h8g8_ragged6"], device=DEV, seed=11)
    L, Hkv = wl.cfg.L, wl.cfg.Hkv
    pos = _positions(wl, 1, gapped={0, 2})
    max_dist = int(wl.cur_pos.max().item()) + 5
    table = torch.randn(L, Hkv, max_dist + 1, generator=torch.Generator().manual_seed(3)).to(DEV)
    cache = cache_of(wl)
    max_len = wl.max_blocks * 16
    sentinel = 77.25
    scores = torch.full((wl.cfg.S, L, Hkv, max_len), sentinel, device=DEV)
    tri.tri_score_distance(cache, table, torch.from_numpy(pos).to(DEV), scores)
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    tab, sc, p = table.cpu().numpy(), scores.cpu().numpy(), wl.cur_pos.cpu().numpy()
    for s, n in enumerate(wl.seq_len.cpu().tolist()):
        for l in range(L):
            for h in range(Hkv):
                want = tab[l, h, p[s] - pos[s, l, h, :n]]
                assert np.array_equal(sc[s, l, h, :n], want)
                assert np.all(sc[s, l, h, n:] == sentinel)
    # a key cached after the query position is a bounds error
    bad = pos.copy()
    s0 = 0
    bad[s0, 0, 0, 0] = int(p[s0]) + 1
    tri.tri_score_distance(cache, table, torch.from_numpy(bad).to(DEV), scores)
    assert tri.tri_sync_status(cache.status) == tri.TRI_ERR_DEVICE_BOUNDS


@pytest.mark.parametrize("sinks,trigger", [(0, 0), (4, 0), (2, 600)])
def test_compress_step_distance_matches_oracle(sinks, trigger):
    wl = make_workload(SMALL["l2h8g8_ragged6"], device=DEV, seed=12)
    budget, window = wl.cfg.budget, wl.cfg.window
    S, L, Hkv, G = wl.cfg.S, wl.cfg.L, wl.cfg.Hkv, wl.cfg.G
    pos = _positions(wl, 2, gapped={2, 5})
    p = wl.cur_pos.cpu().tolist()
    max_dist = max(p) + 10
    qbar, kbar = _centres(L, Hkv, G, seed=5)
    qb, kb = qbar.double().numpy(), kbar.double().numpy()
    deltas, base = wl.deltas, wl.cfg.base
    tables = np.stack([np.stack([oracle.distance_table(qb[l, h * G:(h + 1) * G], kb[l, h], deltas, base, max_dist)
                                 for h in range(Hkv)]) for l in range(L)]).astype(np.float32)
    lens = wl.seq_len.cpu().tolist()
    trig = max(trigger, budget)
    kept = [budget if n > trig else n for n in lens]
    k_bits = wl.k_pool.view(torch.int16).cpu().numpy()
    v_bits = wl.v_pool.view(torch.int16).cpu().numpy()
    ref = oracle.compress_step_distance(k_bits, v_bits, wl.block_table.cpu().numpy(), lens, p, pos,
                                        tables.astype(np.float64), budget, window, sinks, trigger)
    pk, pv = wl.k_pool.clone(), wl.v_pool.clone()
    cache = cache_of(wl)
    opt = tri.step_options(budget, window, sinks, trigger)
    ws = tri.alloc_workspace(cache, budget)
    freed = torch.full((S * wl.max_blocks,), -7, dtype=torch.int32, device=DEV)
    count = torch.zeros(1, dtype=torch.int32, device=DEV)
    idx = torch.full((S, L, Hkv, budget), -7, dtype=torch.int32, device=DEV)
    gpos = torch.from_numpy(pos).to(DEV)
    tri.tri_compress_step_distance(cache, torch.from_numpy(tables).to(DEV), gpos, opt, ws, freed_ids=freed,
                                   freed_count=count, idx_out=idx)
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    assert wl.seq_len.cpu().tolist() == ref["seq_len"] == kept
    assert freed[:int(count.item())].cpu().tolist() == ref["freed_ids"] == freed_expected(wl.block_table, lens, kept)
    for (s, l, h), want in ref["idx"].items():
        assert np.array_equal(idx[s, l, h].cpu().numpy(), want), (s, l, h)
    assert np.array_equal(gpos.cpu().numpy(), ref["positions"])
    ek, ev = expected_pools_after(pk, pv, wl.block_table, lens, idx, kept)
    assert torch.equal(wl.k_pool.view(torch.int16), ek.view(torch.int16))
    assert torch.equal(wl.v_pool.view(torch.int16), ev.view(torch.int16))
    assert np.array_equal(wl.k_pool.view(torch.int16).cpu().numpy(), ref["k_pool"])
    assert np.array_equal(wl.v_pool.view(torch.int16).cpu().numpy(), ref["v_pool"])


def test_full_size_distance_step_32L_8H_T32768():
    """The benchmark's distance-table step at its full size (32 layers x 8 KV
    heads, one sequence of 32768 slots, B = 2048, W = 128) in the launch
    configuration bench.py times: the table built by tri_distance_table
    (sampled heads against the oracle's table), then one
    tri_compress_step_distance.  Every unit's kept slots, every row of both
    pools and every carried position are checked; sampled units' kept slots
    equal the oracle's selection on the same table values, bit for bit."""
    from workload import CONFIGS
    wl = make_workload(CONFIGS["l32h8_t32k"], device=DEV, seed=0)
    cfg = wl.cfg
    S, L, Hkv, G = cfg.S, cfg.L, cfg.Hkv, cfg.G
    budget, window = cfg.budget, cfg.window
    qbar = gpu_stats(wl)[0]
    kbar = wl.key_centres.float().contiguous()
    max_dist = int(wl.cur_pos.max().item()) + 1
    table = torch.empty(L, Hkv, max_dist + 1, device=DEV)
    tri.tri_distance_table(qbar, kbar, cfg.base, wl.deltas, tri.TRI_AGG_MEAN, table)
    torch.cuda.synchronize()
    tab = table.cpu().numpy()
    for l, h in ((0, 0), (L - 1, Hkv - 1)):
        ref = oracle.distance_table(qbar[l, h * G:(h + 1) * G].double().cpu().numpy(),
                                    kbar[l, h].double().cpu().numpy(), wl.deltas, cfg.base, max_dist)
        scale = float(np.max(np.abs(ref)))
        err = np.abs(tab[l, h].astype(np.float64) - ref)
        assert np.all(err <= 1e-6 * np.abs(ref) + 1e-7 * scale), float((err / scale).max())
    lens = wl.seq_len.cpu().tolist()
    kept = [min(n, budget) for n in lens]
    max_len = wl.max_blocks * 16
    pos0 = torch.arange(max_len, dtype=torch.int32, device=DEV).repeat(S, L, Hkv, 1).contiguous()
    gpos = pos0.clone()
    pk, pv = wl.k_pool.clone(), wl.v_pool.clone()
    cache = cache_of(wl)
    opt = tri.step_options(budget, window)
    ws = tri.alloc_workspace(cache, opt)
    freed = torch.full((S * wl.max_blocks,), -7, dtype=torch.int32, device=DEV)
    count = torch.full((1,), -7, dtype=torch.int32, device=DEV)
    idx = torch.full((S, L, Hkv, budget), -7, dtype=torch.int32, device=DEV)
    tri.tri_compress_step_distance(cache, table, gpos, opt, ws, freed_ids=freed, freed_count=count, idx_out=idx)
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    assert wl.seq_len.cpu().tolist() == kept
    assert freed[:int(count.item())].cpu().tolist() == freed_expected(wl.block_table, lens, kept)
    ek, ev = expected_pools_after(pk, pv, wl.block_table, lens, idx, kept)
    del pk, pv
    assert torch.equal(wl.k_pool.view(torch.int16), ek.view(torch.int16))
    assert torch.equal(wl.v_pool.view(torch.int16), ev.view(torch.int16))
    del ek, ev
    # positions travel with their rows; slots past the kept ones keep theirs
    assert torch.equal(gpos[..., :budget], torch.gather(pos0, -1, idx.long()))
    assert torch.equal(gpos[..., budget:], pos0[..., budget:])
    # every unit: ascending, window kept; sampled units: the oracle's selection
    assert torch.all(idx[..., 1:] > idx[..., :-1])
    cand = lens[0] - window
    assert torch.all(idx[..., budget - window:] == torch.arange(cand, lens[0], device=DEV, dtype=torch.int32))
    p = wl.cur_pos.cpu().tolist()
    rng = np.random.default_rng(1)
    units = [(0, 0, 0), (S - 1, L - 1, Hkv - 1)] + [(0, int(rng.integers(L)), int(rng.integers(Hkv)))
                                                    for _ in range(4)]
    for s, l, h in units:
        n = lens[s]
        scores = oracle.distance_scores(tab[l, h].astype(np.float64), p[s], np.arange(n))
        want = oracle.select(scores, n, budget, window)
        assert np.array_equal(idx[s, l, h].cpu().numpy(), want), (s, l, h)
