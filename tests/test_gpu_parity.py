"""GPU parity of every C-ABI entry point against the float64 oracle.

All calls go through the shared library (rope_aware_kv_tri_b200 -> ctypes ->
libtriattn.so).  Inputs are seeded synthetic workloads shaped like the five
measured configurations, cut down so the oracle finishes in seconds while
still spanning many 16-row blocks, several score work items, ragged tails,
shuffled block tables, and every KV-heads-per-tile variant (8, 4, 2, 1).
"""

import numpy as np
import pytest
import torch

import oracle
import rope_aware_kv_tri_b200 as tri
from tests.gpu_helpers import (SCORE_TOL, cache_of, check_scores, check_selection, expected_pools_after,
                               freed_expected, gpu_stats, oracle_stats, oracle_unit_scores, run_step,
                               status_tensor, unit_rows)
from workload import CONFIGS, make_workload

pytestmark = pytest.mark.gpu

DEV = "cuda"

SMALL = {
    "head1_t4096": CONFIGS["head1_t4096"],
    "l2h8g4_t3001": CONFIGS["l32h8_t32k"].replace(L=2, lens=[3001], budget=512, window=64, n_samples=512),
    "l2h8g8_ragged6": CONFIGS["l64h8g8_4x64k"].replace(L=2, lens=[700, 33, 1001, 16, 0, 530], budget=512, window=64,
                                     n_samples=256, table="shuffled", pool_headroom=0.2),
    "l2h8g4_t5000": CONFIGS["l32h8_t128k"].replace(L=2, lens=[5000], budget=1024, window=256, n_samples=512),
    "hkv6": CONFIGS["l32h8_t32k"].replace(L=2, Hkv=6, G=3, lens=[777, 1500], budget=300, window=20,
                                    n_samples=256, table="shuffled"),
    "hkv4": CONFIGS["l32h8_t32k"].replace(L=1, Hkv=4, G=2, lens=[1025], budget=100, window=0, n_samples=256),
    "hkv3": CONFIGS["l32h8_t32k"].replace(L=1, Hkv=3, G=5, lens=[401, 17], budget=64, window=64, n_samples=128,
                                    table="shuffled"),
    # the largest budget the library takes (its kept-slot list fills 64 KiB of
    # the selection CTA's shared memory); one sequence exactly at the budget
    "l1h2g2_b16384": CONFIGS["l32h8_t32k"].replace(L=1, Hkv=2, G=2, lens=[40000, 16384, 20000], budget=16384,
                                             window=1024, n_samples=256, table="shuffled"),
}


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rope_aware_kv_tri_b200 import build_lib
    build_lib.build()
    torch.cuda.init()


def _workload(name, seed=0):
    return make_workload(SMALL[name], device=DEV, seed=seed)


# --------------------------------------------------------------- calibrate

def test_calibrate_matches_oracle():
    cfg = CONFIGS["l32h8_t32k"].replace(L=2, lens=[16], n_samples=777)
    wl = make_workload(cfg, device=DEV)
    qbar, qabs, R = gpu_stats(wl)
    rb, ra, rr = oracle_stats(wl)
    for got, ref in ((qbar, rb), (qabs, ra), (R, rr)):
        got = got.double().cpu().numpy()
        scale = np.abs(ref) + np.mean(np.abs(ref))
        assert np.all(np.abs(got - ref) <= 1e-5 * scale)
    assert np.all((rr > 0.3) & (rr <= 1.0))


def test_calibrate_degenerate_samples():
    q = torch.zeros(5, 1, 2, 128, device=DEV)
    q[:, 0, 1] = torch.randn(128, device=DEV)       # head 1: identical samples
    qbar = torch.empty(1, 2, 128, device=DEV)
    qabs = torch.empty(1, 2, 64, device=DEV)
    R = torch.empty(1, 2, device=DEV)
    tri.tri_calibrate_centers(q, qbar, qabs, R)
    torch.cuda.synchronize()
    assert R[0, 0].item() == 1.0                    # all-zero samples
    assert abs(R[0, 1].item() - 1.0) < 1e-6


# ------------------------------------------------------------- build query

@pytest.mark.parametrize("name", ["head1_t4096", "l2h8g8_ragged6", "hkv3"])
def test_build_query_matches_oracle(name):
    wl = _workload(name)
    stats = gpu_stats(wl)
    ref_stats = oracle_stats(wl)
    S, L, Hkv, G = wl.cfg.S, wl.cfg.L, wl.cfg.Hkv, wl.cfg.G
    qeff = torch.empty(S, L, Hkv, 128, device=DEV)
    w = torch.empty(S, L, Hkv, 64, device=DEV)
    tri.tri_build_query(cache_of(wl), *stats, wl.cfg.base, wl.deltas, qeff, w)
    qeff, w = qeff.double().cpu().numpy(), w.double().cpu().numpy()
    qb, qa, rr = ref_stats
    for s in range(S):
        for l in range(L):
            for h in range(Hkv):
                sl = slice(h * G, (h + 1) * G)
                rq, rw = oracle.group_query(qb[l, sl], qa[l, sl], rr[l, sl], int(wl.cur_pos[s]), wl.deltas,
                                            wl.cfg.base)
                sq = np.abs(rq).max() + 1e-30
                sw = np.abs(rw).max() + 1e-30
                assert np.abs(qeff[s, l, h] - rq).max() <= 2e-5 * sq
                assert np.abs(w[s, l, h] - rw).max() <= 2e-5 * sw + 1e-7


# ------------------------------------------------------------------ score

@pytest.mark.parametrize("name", list(SMALL))
def test_score_matches_oracle(name):
    wl = _workload(name)
    stats = gpu_stats(wl)
    ref_stats = oracle_stats(wl)
    cache = cache_of(wl)
    S, L, Hkv = wl.cfg.S, wl.cfg.L, wl.cfg.Hkv
    max_len = wl.max_blocks * 16
    sentinel = 12345.5
    scores = torch.full((S, L, Hkv, max_len), sentinel, device=DEV)
    ws = tri.alloc_workspace(cache, 1)
    tri.tri_score(cache, *stats, wl.cfg.base, wl.deltas, scores, ws)
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    sc = scores.cpu().numpy()
    table = wl.block_table.cpu().tolist()
    worst = 0.0
    for s in range(S):
        n = int(wl.seq_len[s])
        assert np.all(sc[s, :, :, n:] == sentinel), "score written past the sequence end"
        for l in range(L):
            for h in range(Hkv):
                keys = unit_rows(wl.k_pool, table[s], n, l, h)
                ref = oracle_unit_scores(wl, keys, ref_stats, s, l, h)
                worst = max(worst, check_scores(sc[s, l, h, :n], ref))
    print(f"{name}: worst score error / floor = {worst:.2e}")


# ----------------------------------------------------------------- select

def _score_fill(rng, n, kind):
    if kind == "normal":
        return rng.normal(size=n).astype(np.float32)
    if kind == "ties":
        return (np.round(rng.normal(size=n) * 4) / 4).astype(np.float32)
    if kind == "zeros":
        z = np.zeros(n, dtype=np.float32)
        z[rng.random(n) < 0.5] = -0.0
        return z
    if kind == "wide":
        return (rng.normal(size=n) * np.exp(rng.normal(size=n) * 20)).astype(np.float32)
    if kind == "dups":            # spread range, many exact duplicates near every value
        return (np.round(rng.normal(size=n) * 100) / 100).astype(np.float32)
    raise ValueError(kind)


@pytest.mark.parametrize("budget,window", [(64, 8), (1, 0), (1, 1), (64, 64), (64, 0), (2048, 128)])
def test_select_bit_exact_on_same_scores(budget, window):
    rng = np.random.default_rng(budget * 131 + window)
    # 140000 candidates exceed the shared-memory bitmaps: streaming path
    lens = [0, 1, budget, budget + 1, 3 * budget + 5, 40000, 777, 5000, 140000]
    kinds = ["normal", "ties", "zeros", "wide", "dups"]
    S, L, Hkv = len(lens), 1, len(kinds)
    max_blocks = -(-max(lens) // 16)
    k = torch.zeros(1, 1, Hkv, 16, 128, dtype=torch.bfloat16, device=DEV)
    table = torch.zeros(S, max_blocks, dtype=torch.int32, device=DEV)
    seq_len = torch.tensor(lens, dtype=torch.int32, device=DEV)
    pos = torch.zeros(S, dtype=torch.int64, device=DEV)
    cache = tri.KvCache(k, k.clone(), table, seq_len, pos, status_tensor(DEV), 1)
    sc = np.full((S, L, Hkv, max_blocks * 16), np.nan, dtype=np.float32)
    for s, n in enumerate(lens):
        for h in range(Hkv):
            sc[s, 0, h, :n] = _score_fill(rng, n, kinds[h])
    scores = torch.from_numpy(sc).to(DEV)
    idx = torch.full((S, L, Hkv, budget), -7, dtype=torch.int32, device=DEV)
    kept = torch.full((S,), -7, dtype=torch.int32, device=DEV)
    tri.tri_select_topk(cache, scores, budget, window, idx, kept)
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    idx, kept = idx.cpu().numpy(), kept.cpu().numpy()
    for s, n in enumerate(lens):
        assert kept[s] == min(n, budget)
        for h in range(Hkv):
            ref = oracle.select(sc[s, 0, h, :n].astype(np.float64), n, budget, window)
            assert np.array_equal(idx[s, 0, h, :kept[s]], ref), (s, h, n)
            assert np.all(idx[s, 0, h, kept[s]:] == -1)


def _spaced_runs(cand):
    """64 evenly spaced runs of 32 slots over candidates [0, cand)."""
    stride = (cand - 32) // 63
    return np.concatenate([c * stride + np.arange(32) for c in range(64)])


@pytest.mark.parametrize("budget,window", [(2048, 128), (256, 0), (4096, 256), (16384, 1024)])
def test_select_structured_score_patterns(budget, window):
    """Score patterns with structure along the slots - ramps, periodic
    scores, far outliers packed into evenly spaced runs, a low floor in them,
    and thousands of exact ties at the cut value - at lengths from one to
    several shared-memory bitmaps' worth of candidates.  Every result is the
    oracle's."""
    rng = np.random.default_rng(budget + window)
    lens = [8192 + window, 20000, 65536, 131000]
    kinds = ["normal", "ramp", "periodic", "spaced_high", "spaced_low", "crowded_cut"]
    S, L, Hkv = len(lens), 1, len(kinds)
    max_blocks = -(-max(lens) // 16)
    k = torch.zeros(1, 1, Hkv, 16, 128, dtype=torch.bfloat16, device=DEV)
    cache = tri.KvCache(k, k.clone(), torch.zeros(S, max_blocks, dtype=torch.int32, device=DEV),
                        torch.tensor(lens, dtype=torch.int32, device=DEV), torch.zeros(S, dtype=torch.int64, device=DEV),
                        status_tensor(DEV), 1)
    sc = np.full((S, L, Hkv, max_blocks * 16), np.nan, dtype=np.float32)
    for s, n in enumerate(lens):
        cand = n - window
        runs = _spaced_runs(cand)
        for h, kind in enumerate(kinds):
            x = rng.normal(size=n)
            if kind == "ramp":
                x = np.arange(n) * 1e-3 + 0.01 * x
            elif kind == "periodic":
                x = np.sin(np.arange(n) * 2 * np.pi / 512) + 0.05 * x
            elif kind == "spaced_high":       # half of every run far above everything else
                x[runs[::2]] = 50 + x[runs[::2]]
            elif kind == "spaced_low":        # the runs sit far below everything else
                x[runs] = -50 + x[runs]
            elif kind == "crowded_cut":       # thousands of exact ties at the cut value
                x = rng.normal(size=n) - 10
                hi = rng.choice(cand, budget // 2, replace=False)
                x[hi] = 10 + rng.random(budget // 2)
                rest = np.setdiff1d(np.arange(cand), hi)
                x[rng.choice(rest, min(3 * budget, rest.size), replace=False)] = 1.0
            sc[s, 0, h, :n] = x.astype(np.float32)
    idx = torch.full((S, L, Hkv, budget), -7, dtype=torch.int32, device=DEV)
    kept = torch.full((S,), -7, dtype=torch.int32, device=DEV)
    tri.tri_select_topk(cache, torch.from_numpy(sc).to(DEV), budget, window, idx, kept)
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    idx = idx.cpu().numpy()
    for s, n in enumerate(lens):
        k = min(n, budget)
        for h, kind in enumerate(kinds):
            ref = oracle.select(sc[s, 0, h, :n].astype(np.float64), n, budget, window)
            assert np.array_equal(idx[s, 0, h, :k], ref), (n, kind)
            assert np.all(idx[s, 0, h, k:] == -1)


def test_select_nan_ranks_lowest_and_is_flagged():
    n, budget, window = 300, 40, 5
    rng = np.random.default_rng(3)
    sc = rng.normal(size=(1, 1, 1, 304)).astype(np.float32)
    sc[0, 0, 0, rng.choice(n - window, 280, replace=False)] = np.nan
    k = torch.zeros(1, 1, 1, 16, 128, dtype=torch.bfloat16, device=DEV)
    cache = tri.KvCache(k, k.clone(), torch.zeros(1, 19, dtype=torch.int32, device=DEV),
                        torch.tensor([n], dtype=torch.int32, device=DEV), torch.zeros(1, dtype=torch.int64, device=DEV),
                        status_tensor(DEV), 1)
    idx = torch.empty(1, 1, 1, budget, dtype=torch.int32, device=DEV)
    kept = torch.empty(1, dtype=torch.int32, device=DEV)
    tri.tri_select_topk(cache, torch.from_numpy(sc).to(DEV), budget, window, idx, kept)
    assert tri.tri_sync_status(cache.status) == tri.TRI_ERR_NONFINITE
    ref = oracle.select(sc[0, 0, 0, :n].astype(np.float64), n, budget, window)
    assert np.array_equal(idx[0, 0, 0].cpu().numpy(), ref)


# ---------------------------------------------------------------- compact

@pytest.mark.parametrize("name", ["l2h8g8_ragged6", "hkv6", "head1_t4096"])
def test_compact_bit_exact_for_given_indices(name):
    wl = _workload(name, seed=5)
    budget, window = wl.cfg.budget, wl.cfg.window
    S, L, Hkv = wl.cfg.S, wl.cfg.L, wl.cfg.Hkv
    lens = wl.seq_len.cpu().tolist()
    rng = np.random.default_rng(9)
    idx = np.full((S, L, Hkv, budget), -1, dtype=np.int32)
    kept = [min(n, budget) for n in lens]
    for s, n in enumerate(lens):
        for l in range(L):
            for h in range(Hkv):
                if n <= budget:
                    idx[s, l, h, :n] = np.arange(n)
                else:
                    pick = np.sort(rng.choice(n - window, budget - window, replace=False))
                    if (s + l + h) % 3 == 0:       # a kept prefix that does not move
                        pick = np.arange(budget - window)
                    idx[s, l, h, :budget] = np.concatenate([pick, np.arange(n - window, n)])
    pk, pv = wl.k_pool.clone(), wl.v_pool.clone()
    cache = cache_of(wl)
    freed = torch.full((S * wl.max_blocks,), -7, dtype=torch.int32, device=DEV)
    count = torch.zeros(1, dtype=torch.int32, device=DEV)
    idx_t = torch.from_numpy(idx).to(DEV)
    tri.tri_compact_kv(cache, idx_t, torch.tensor(kept, dtype=torch.int32, device=DEV), budget, freed, count)
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    # the oracle moves the same rows on the bf16 bit patterns
    kb, vb = pk.view(torch.int16).cpu().numpy(), pv.view(torch.int16).cpu().numpy()
    nk, nv = kb.copy(), vb.copy()
    table = wl.block_table.cpu().numpy()
    for s, n in enumerate(lens):
        for l in range(L):
            for h in range(Hkv):
                rows_k = oracle.unit_rows(kb, table[s], n, l, h)
                rows_v = oracle.unit_rows(vb, table[s], n, l, h)
                oracle.tri_oracle.store_unit_rows(nk, table[s], oracle.compact_rows(rows_k, idx[s, l, h, :kept[s]]), l, h)
                oracle.tri_oracle.store_unit_rows(nv, table[s], oracle.compact_rows(rows_v, idx[s, l, h, :kept[s]]), l, h)
    assert np.array_equal(wl.k_pool.view(torch.int16).cpu().numpy(), nk)
    assert np.array_equal(wl.v_pool.view(torch.int16).cpu().numpy(), nv)
    assert wl.seq_len.cpu().tolist() == kept
    want = freed_expected(wl.block_table, lens, kept)
    assert int(count.item()) == len(want) and freed[:len(want)].cpu().tolist() == want


# ----------------------------------------------------------- compress step

@pytest.mark.parametrize("name", list(SMALL))
def test_compress_step_matches_oracle(name):
    wl = _workload(name, seed=1)
    budget, window = wl.cfg.budget, wl.cfg.window
    stats = gpu_stats(wl)
    ref_stats = oracle_stats(wl)
    S, L, Hkv = wl.cfg.S, wl.cfg.L, wl.cfg.Hkv
    lens = wl.seq_len.cpu().tolist()
    kept = [min(n, budget) for n in lens]
    table = wl.block_table.cpu().tolist()
    pk, pv = wl.k_pool.clone(), wl.v_pool.clone()
    out = run_step(wl, stats, budget, window)
    assert out["status"] == tri.TRI_OK
    assert wl.seq_len.cpu().tolist() == kept
    assert out["freed"] == freed_expected(wl.block_table, lens, kept)
    idx = out["idx"]
    differ = 0
    for s, n in enumerate(lens):
        for l in range(L):
            for h in range(Hkv):
                if n <= budget:
                    assert torch.all(idx[s, l, h] == -7), "idx written for an untouched sequence"
                    continue
                ref = oracle_unit_scores(wl, unit_rows(pk, table[s], n, l, h), ref_stats, s, l, h)
                differ += check_selection(idx[s, l, h].cpu().numpy(), ref, n, budget, window)
    ek, ev = expected_pools_after(pk, pv, wl.block_table, lens, idx, kept)
    assert torch.equal(wl.k_pool.view(torch.int16), ek.view(torch.int16))
    assert torch.equal(wl.v_pool.view(torch.int16), ev.view(torch.int16))
    print(f"{name}: {differ} kept slots differ from the oracle inside the cut band")


def test_compress_step_all_equal_scores_keeps_earliest():
    """Zero statistics make every score exactly 0: the step keeps the lowest
    slots plus the window, exactly as the oracle."""
    wl = _workload("l2h8g8_ragged6", seed=2)
    L, Hq = wl.cfg.L, wl.cfg.Hq
    zero = (torch.zeros(L, Hq, 128, device=DEV), torch.zeros(L, Hq, 64, device=DEV),
            torch.ones(L, Hq, device=DEV))
    lens = wl.seq_len.cpu().tolist()
    out = run_step(wl, zero, 512, 64)
    assert out["status"] == tri.TRI_OK
    for s, n in enumerate(lens):
        if n <= 512:
            continue
        want = np.concatenate([np.arange(448), np.arange(n - 64, n)])
        for l in range(L):
            for h in range(wl.cfg.Hkv):
                assert np.array_equal(out["idx"][s, l, h].cpu().numpy(), want)


def test_compress_step_budget_one_and_second_call_is_noop():
    wl = _workload("l2h8g4_t3001", seed=3)
    stats = gpu_stats(wl)
    out = run_step(wl, stats, 1, 1)
    assert out["status"] == tri.TRI_OK and wl.seq_len.tolist() == [1]
    k1 = wl.k_pool.clone()
    out2 = run_step(wl, stats, 1, 1)
    assert out2["freed"] == [] and torch.equal(k1, wl.k_pool)


def test_bad_block_id_is_flagged_not_followed():
    wl = _workload("l2h8g8_ragged6", seed=4)
    stats = gpu_stats(wl)
    wl.block_table[0, 3] = wl.num_blocks + 1000          # out of the pool
    wl.block_table[2, 0] = -5
    out = run_step(wl, stats, 512, 64)
    assert out["status"] == tri.TRI_ERR_DEVICE_BOUNDS
    # the context is intact: a clean call afterwards succeeds
    wl2 = _workload("l2h8g4_t3001", seed=4)
    assert run_step(wl2, gpu_stats(wl2), 512, 64)["status"] == tri.TRI_OK


def test_sequence_longer_than_its_table_is_flagged():
    wl = _workload("l2h8g4_t3001", seed=6)
    stats = gpu_stats(wl)
    wl.seq_len[0] = wl.max_blocks * 16 + 1
    k0 = wl.k_pool.clone()
    out = run_step(wl, stats, 512, 64)
    assert out["status"] == tri.TRI_ERR_DEVICE_BOUNDS
    assert torch.equal(k0, wl.k_pool)


def test_compress_step_prefix_heavy_units_mix_scratch_and_in_place():
    """Scores that fall with the slot make almost every kept source lie below
    the budget, so each unit's at-risk prefix is nearly B rows: the step's
    scratch (a quarter of the kept rows) fills up and later units compact
    their prefix in place.  Both paths must give the oracle's result."""
    cfg = CONFIGS["l32h8_t32k"].replace(L=1, Hkv=4, G=2, lens=[700, 650], budget=256, window=16, n_samples=64,
                                  table="shuffled")
    wl = make_workload(cfg, device=DEV, seed=7)
    L, Hkv, Hq = cfg.L, cfg.Hkv, cfg.Hq
    table = wl.block_table.cpu().tolist()
    gen = torch.Generator(device=DEV).manual_seed(3)
    for s, n in enumerate(cfg.lens):
        t = torch.arange(n, device=DEV, dtype=torch.float32)
        scale = 1.0 / (1.0 + t / 50.0)
        scale[0] = 1e-3                                  # slot 0 is evicted: every row moves
        for l in range(L):
            for h in range(Hkv):
                rows = torch.randn(n, 128, device=DEV, generator=gen) * scale[:, None]
                blocks = torch.tensor(table[s][: -(-n // 16)], device=DEV, dtype=torch.long)
                padded = torch.zeros(len(blocks) * 16, 128, device=DEV)
                padded[:n] = rows
                wl.k_pool[l, blocks, h] = padded.view(len(blocks), 16, 128).to(torch.bfloat16)
    # norm-only scoring: qbar = 0, E|q_i| = 1, R = 0
    stats = (torch.zeros(L, Hq, 128, device=DEV), torch.ones(L, Hq, 64, device=DEV), torch.zeros(L, Hq, device=DEV))
    ref_stats = tuple(x.double().cpu().numpy() for x in stats)
    lens = list(cfg.lens)
    kept = [min(n, cfg.budget) for n in lens]
    pk, pv = wl.k_pool.clone(), wl.v_pool.clone()
    out = run_step(wl, stats, cfg.budget, cfg.window)
    assert out["status"] == tri.TRI_OK
    idx = out["idx"]
    assert out["freed"] == freed_expected(wl.block_table, lens, kept)
    for s, n in enumerate(lens):
        for l in range(L):
            for h in range(Hkv):
                ref = oracle_unit_scores(wl, unit_rows(pk, table[s], n, l, h), ref_stats, s, l, h)
                check_selection(idx[s, l, h].cpu().numpy(), ref, n, cfg.budget, cfg.window)
                assert int((idx[s, l, h] < cfg.budget).sum()) > cfg.budget // 2     # prefix-heavy indeed
    ek, ev = expected_pools_after(pk, pv, wl.block_table, lens, idx, kept)
    assert torch.equal(wl.k_pool.view(torch.int16), ek.view(torch.int16))
    assert torch.equal(wl.v_pool.view(torch.int16), ev.view(torch.int16))


def test_bounded_device_wait_gives_up_and_context_stays_usable():
    """A device wait that nothing completes ends after the library's wait
    limit (2 s) with TRI_ERR_TIMEOUT; a flag that is already set ends it at
    once; and the context then runs a step as usual."""
    import time
    status = status_tensor(DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    tri.tri_selftest_bounded_wait(status)                      # barrier nobody arrives at
    assert tri.tri_sync_status(status) == tri.TRI_ERR_TIMEOUT
    waited = time.perf_counter() - t0
    assert 1.5 < waited < 30.0, waited
    unset = torch.zeros(1, dtype=torch.int32, device=DEV)
    tri.tri_selftest_bounded_wait(status, unset)               # flag nobody sets
    assert tri.tri_sync_status(status) == tri.TRI_ERR_TIMEOUT
    t0 = time.perf_counter()
    tri.tri_selftest_bounded_wait(status, torch.ones(1, dtype=torch.int32, device=DEV))
    assert tri.tri_sync_status(status) == tri.TRI_OK
    assert time.perf_counter() - t0 < 1.0
    wl = _workload("hkv4", seed=3)
    out = run_step(wl, gpu_stats(wl), wl.cfg.budget, wl.cfg.window)
    assert out["status"] == tri.TRI_OK


def test_compress_step_replays_from_a_cuda_graph():
    """One step captured in a CUDA graph (its launches with programmatic
    dependencies become graph edges) and replayed on a restored cache gives
    the same cache, lengths, freed blocks and kept slots as a direct call."""
    wl = _workload("l2h8g8_ragged6", seed=21)
    stats = gpu_stats(wl)
    budget, window = wl.cfg.budget, wl.cfg.window
    S, L, Hkv = wl.cfg.S, wl.cfg.L, wl.cfg.Hkv
    cache = cache_of(wl)
    ws = tri.alloc_workspace(cache, budget)
    freed = torch.zeros(S * wl.max_blocks, dtype=torch.int32, device=DEV)
    count = torch.zeros(1, dtype=torch.int32, device=DEV)
    idx = torch.full((S, L, Hkv, budget), -7, dtype=torch.int32, device=DEV)
    k0, v0, len0 = wl.k_pool.clone(), wl.v_pool.clone(), wl.seq_len.clone()

    def step():
        tri.tri_compress_step(cache, *stats, wl.cfg.base, wl.deltas, budget, window, freed, count, ws, idx_out=idx)

    step()
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    direct = (wl.k_pool.clone(), wl.v_pool.clone(), wl.seq_len.clone(), freed[:int(count.item())].clone(), idx.clone())
    wl.k_pool.copy_(k0)
    wl.v_pool.copy_(v0)
    wl.seq_len.copy_(len0)
    idx.fill_(-7)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    torch.cuda.synchronize()
    # capture records the work without running it: the cache is still the original
    assert torch.equal(wl.seq_len, len0)
    g.replay()
    torch.cuda.synchronize()
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    assert torch.equal(wl.k_pool.view(torch.int16), direct[0].view(torch.int16))
    assert torch.equal(wl.v_pool.view(torch.int16), direct[1].view(torch.int16))
    assert torch.equal(wl.seq_len, direct[2])
    assert torch.equal(freed[:int(count.item())], direct[3])
    assert torch.equal(idx, direct[4])
    del g
