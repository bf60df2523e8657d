"""Shared glue of the GPU parity tests: run the CUDA path through the C ABI,
run the float64 oracle on the same inputs, compare under the parity rules.

Parity rules (the tolerance of the score is the one the path is specified
with: relative 2e-3 for fp32 accumulation over bf16 keys):
  * score  : |s_gpu - s_ref| <= 2e-3 * max(|s_ref|, m_u), m_u = mean |s_ref|
             over the unit (floor so near-zero scores do not inflate the
             relative error);
  * indices: bit-exact for identical fp32 scores; against the oracle's own
             float64 scores the kept sets may differ only in keys whose oracle
             score lies within tau_u = 2e-3 * max(|s_cut|, m_u) of the cut;
  * compaction: bit-exact.
"""

from __future__ import annotations

from typing import Dict, List, Tuple

import numpy as np
import torch

import oracle
import rope_aware_kv_tri_b200 as tri

SCORE_TOL = 2e-3


def status_tensor(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def cache_of(wl, pools=None, seq_len=None) -> tri.KvCache:
    k, v = pools if pools is not None else (wl.k_pool, wl.v_pool)
    return tri.KvCache(k, v, wl.block_table, wl.seq_len if seq_len is None else seq_len, wl.cur_pos,
                       status_tensor(wl.device), wl.cfg.G)


def gpu_stats(wl):
    """Head statistics the CUDA path uses: the workload's own when given
    directly, else tri_calibrate_centers on the calibration samples."""
    if wl.qbar is not None:
        return wl.qbar, wl.qabs, wl.R
    L, Hq = wl.cfg.L, wl.cfg.Hq
    dev = wl.device
    qbar = torch.empty(L, Hq, 128, dtype=torch.float32, device=dev)
    qabs = torch.empty(L, Hq, 64, dtype=torch.float32, device=dev)
    R = torch.empty(L, Hq, dtype=torch.float32, device=dev)
    tri.tri_calibrate_centers(wl.q_samples, qbar, qabs, R)
    return qbar, qabs, R


def oracle_stats(wl, l=None, heads=None):
    """Head statistics the oracle uses, computed by the oracle (optionally for
    one layer and a slice of query heads only)."""
    if wl.qbar is not None:
        qb, qa, r = (t.double().cpu().numpy() for t in (wl.qbar, wl.qabs, wl.R))
        if l is not None:
            return qb[l, heads], qa[l, heads], r[l, heads]
        return qb, qa, r
    q = wl.q_samples
    if l is not None:
        q = q[:, l, heads]
    return oracle.calibrate(q.double().cpu().numpy())


def unit_rows(pool: torch.Tensor, table_row: List[int], length: int, l: int, h: int) -> torch.Tensor:
    """Rows [0, length) of (layer l, KV head h) of one sequence, [length, 128]."""
    nb = -(-length // 16)
    if nb == 0:
        return pool.new_empty((0, pool.shape[-1]))
    blocks = torch.tensor(table_row[:nb], dtype=torch.long, device=pool.device)
    return pool[l, blocks, h].reshape(nb * 16, pool.shape[-1])[:length]


def oracle_unit_scores(wl, keys: torch.Tensor, stats, s: int, l: int, h: int,
                       aggregate: str = "mean") -> np.ndarray:
    G = wl.cfg.G
    qb, qa, r = stats
    sl = slice(h * G, (h + 1) * G)
    return oracle.unit_scores(keys.double().cpu().numpy(), qb[l, sl], qa[l, sl], r[l, sl],
                              int(wl.cur_pos[s].item()), wl.deltas, wl.cfg.base, aggregate=aggregate)


def check_scores(s_gpu: np.ndarray, s_ref: np.ndarray, tol: float = SCORE_TOL) -> float:
    """Assert the score rule; return the worst error relative to the floor."""
    if s_ref.size == 0:
        return 0.0
    m_u = float(np.mean(np.abs(s_ref)))
    scale = np.maximum(np.abs(s_ref), m_u)
    err = np.abs(s_gpu.astype(np.float64) - s_ref)
    bad = err > tol * scale
    assert not bad.any(), (f"{int(bad.sum())} scores off: worst {float((err / scale).max()):.3e} "
                           f"at {int(np.argmax(err / scale))}")
    return float((err / scale).max())


def check_selection(idx_gpu: np.ndarray, s_ref: np.ndarray, length: int, budget: int, window: int,
                    tol: float = SCORE_TOL, sinks: int = 0) -> int:
    """Assert the index rule against the oracle's float64 scores; returns the
    number of kept slots that differ (all of them inside the cut band)."""
    ref = oracle.select(s_ref, length, budget, window, sinks)
    idx_gpu = np.asarray(idx_gpu, dtype=np.int64)
    assert idx_gpu.shape == ref.shape, (idx_gpu.shape, ref.shape)
    assert np.all(np.diff(idx_gpu) > 0), "kept slots not strictly ascending"
    if length <= budget:
        assert np.array_equal(idx_gpu, ref)
        return 0
    cand, take = length - window, budget - window
    assert np.array_equal(idx_gpu[take:], np.arange(cand, length)), "recent window not kept"
    assert np.array_equal(idx_gpu[:sinks], np.arange(sinks)), "sink slots not kept"
    take -= sinks
    if take == 0:
        return 0
    order = sorted(range(sinks, cand), key=lambda t: (-s_ref[t], t))
    s_cut = s_ref[order[take - 1]]
    m_u = float(np.mean(np.abs(s_ref)))
    tau = tol * max(abs(s_cut), m_u)
    diff = set(idx_gpu.tolist()) ^ set(ref.tolist())
    for t in diff:
        assert sinks <= t < cand and abs(s_ref[t] - s_cut) <= tau, (
            f"slot {t} differs with score {s_ref[t]} far from the cut {s_cut} (tau {tau})")
    return len(diff)


def expected_pools_after(pristine_k: torch.Tensor, pristine_v: torch.Tensor, table: torch.Tensor,
                         lens: List[int], idx: torch.Tensor, kept: List[int]) -> Tuple[torch.Tensor, torch.Tensor]:
    """Pools after moving, for every unit, pristine row idx[j] to row j
    (j < kept[s]); every other row unchanged.  Plain torch gathers."""
    ek, ev = pristine_k.clone(), pristine_v.clone()
    S, L, Hkv, B = idx.shape
    dev = pristine_k.device
    for s in range(S):
        n = kept[s]
        if n == 0 or lens[s] <= n:
            continue
        src = idx[s, :, :, :n].long()                          # [L, Hkv, n]
        assert int(src.min()) >= 0 and int(src.max()) < lens[s]
        trow = table[s].long()
        l_ix = torch.arange(L, device=dev)[:, None, None].expand(L, Hkv, n)
        h_ix = torch.arange(Hkv, device=dev)[None, :, None].expand(L, Hkv, n)
        j = torch.arange(n, device=dev)[None, None, :].expand(L, Hkv, n)
        sb, sr = trow[src // 16], src % 16
        db, dr = trow[j // 16], j % 16
        ek[l_ix, db, h_ix, dr] = pristine_k[l_ix, sb, h_ix, sr]
        ev[l_ix, db, h_ix, dr] = pristine_v[l_ix, sb, h_ix, sr]
    return ek, ev


def freed_expected(table: torch.Tensor, lens: List[int], kept: List[int]) -> List[int]:
    out: List[int] = []
    rows = table.cpu().tolist()
    for s, (n, k) in enumerate(zip(lens, kept)):
        out += oracle.freed_blocks(rows[s], n, k, 16)
    return out


def run_step(wl, stats, budget: int, window: int, events=None) -> Dict:
    """One tri_compress_step on the workload's own tensors (modified in place)."""
    cache = cache_of(wl)
    S, L, Hkv = wl.cfg.S, wl.cfg.L, wl.cfg.Hkv
    dev = wl.device
    ws = tri.alloc_workspace(cache, budget)
    freed = torch.full((S * wl.max_blocks,), -7, dtype=torch.int32, device=dev)
    count = torch.full((1,), -7, dtype=torch.int32, device=dev)
    idx = torch.full((S, L, Hkv, budget), -7, dtype=torch.int32, device=dev)
    qbar, qabs, R = stats
    tri.tri_compress_step(cache, qbar, qabs, R, wl.cfg.base, wl.deltas, budget, window, freed, count, ws,
                          idx_out=idx, events=events)
    code = tri.tri_sync_status(cache.status)
    n = int(count.item())
    return {"status": code, "freed": freed[:n].cpu().tolist(), "idx": idx, "ws": ws}
