"""The statistics sanity check on the GPU (tri_check_stats, and the step's
check_stats option).

Page: "TriAttention: trigonometric KV cache compression for long reasoning"
- "Calibration statistics are tied to a specific model": mismatched or
damaged statistics raise no error of their own, they only make the step keep
the wrong keys.  The check flags what no valid statistics can have (a NaN or
infinity, R outside [0, 1], a band whose mean magnitude is below the
magnitude of its mean, i.e. a negative norm weight) and reports an R that
differs from its definition.

Each case plants one defect in one head of otherwise calibrated statistics
and checks the per-head bits against the definitions evaluated here, the
status flag, and that a step run with check_stats changes nothing at all:
pools, lengths, free list, freed count and idx_out stay as they were.
Valid statistics pass, and a step with the check on equals one without it.
"""

import numpy as np
import pytest
import torch

import rope_aware_kv_tri_b200 as tri
from tests.gpu_helpers import cache_of, gpu_stats, status_tensor
from workload import CONFIGS, make_workload

pytestmark = pytest.mark.gpu
DEV = "cuda"

CFG = CONFIGS["l32h8_t32k"].replace(L=2, lens=[5000, 700, 3001], budget=512, window=64, n_samples=512)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rope_aware_kv_tri_b200 import build_lib
    build_lib.build()
    torch.cuda.init()


def _expected_bits(qbar, qabs, R):
    """The per-head bits written out from the definitions, in float64."""
    qb, qa, r = (t.double().cpu().numpy() for t in (qbar, qabs, R))
    L, Hq, D = qb.shape
    out = np.zeros((L, Hq), dtype=np.int32)
    for l in range(L):
        for h in range(Hq):
            bits = 0
            x, a, rr = qb[l, h], qa[l, h], r[l, h]
            mag = np.hypot(x[:64], x[64:])
            if not (np.isfinite(x).all() and np.isfinite(a).all() and np.isfinite(rr)):
                bits |= tri.TRI_STATS_NONFINITE
            else:
                if (a < mag * (1 - 1e-5)).any():
                    bits |= tri.TRI_STATS_NORM_WEIGHT
                if rr < 0 or rr > 1:
                    bits |= tri.TRI_STATS_R_RANGE
                ref = mag.sum() / a.sum() if a.sum() > 0 else 1.0
                if abs(rr - ref) > 1e-3 * ref + 1e-6:
                    bits |= tri.TRI_STATS_R_MISMATCH
            out[l, h] = bits
    return out


def _damage(kind, qbar, qabs, R):
    qbar, qabs, R = qbar.clone(), qabs.clone(), R.clone()
    if kind == "nan_centre":
        qbar[1, 5, 70] = float("nan")
    elif kind == "inf_abs":
        qabs[0, 3, 10] = float("inf")
    elif kind == "nan_R":
        R[1, 0] = float("nan")
    elif kind == "R_above_one":
        R[0, 7] = 1.25
    elif kind == "R_negative":
        R[1, 31] = -0.1
    elif kind == "abs_below_centre":
        # a band whose mean magnitude is below the centre's magnitude
        mag = torch.hypot(qbar[0, 9, 20], qbar[0, 9, 84])
        qabs[0, 9, 20] = 0.5 * mag
    elif kind == "other_models_R":
        R[1, 2] = 0.999 * R[1, 2] + 0.001 * 0.0 - 0.05     # valid range, not this head's concentration
    return qbar, qabs, R


KINDS = ["nan_centre", "inf_abs", "nan_R", "R_above_one", "R_negative", "abs_below_centre", "other_models_R"]


def test_valid_statistics_pass():
    wl = make_workload(CFG, device=DEV, seed=1)
    qbar, qabs, R = gpu_stats(wl)
    st = status_tensor(DEV)
    flags = torch.full(R.shape, -1, dtype=torch.int32, device=DEV)
    tri.tri_check_stats(qbar, qabs, R, st, flags)
    assert tri.tri_sync_status(st) == tri.TRI_OK
    assert (flags.cpu().numpy() == 0).all()
    assert np.array_equal(flags.cpu().numpy(), _expected_bits(qbar, qabs, R))


@pytest.mark.parametrize("kind", KINDS)
def test_each_defect_is_flagged_and_vetoes_the_step(kind):
    wl = make_workload(CFG, device=DEV, seed=2)
    qbar, qabs, R = _damage(kind, *gpu_stats(wl))
    want = _expected_bits(qbar, qabs, R)
    assert want.any(), kind
    fails = bool((want & (tri.TRI_STATS_NONFINITE | tri.TRI_STATS_R_RANGE | tri.TRI_STATS_NORM_WEIGHT)).any())

    st = status_tensor(DEV)
    flags = torch.full(R.shape, -1, dtype=torch.int32, device=DEV)
    tri.tri_check_stats(qbar, qabs, R, st, flags)
    assert np.array_equal(flags.cpu().numpy(), want)
    assert tri.tri_sync_status(st) == (tri.TRI_ERR_STATS if fails else tri.TRI_OK)

    cache = cache_of(wl)
    k0, v0, len0 = wl.k_pool.clone(), wl.v_pool.clone(), wl.seq_len.clone()
    opt = tri.step_options(CFG.budget, CFG.window, check_stats=True)
    ws = tri.alloc_workspace(cache, opt)
    fl = tri.FreeList.from_ids([900001, 900002], 4096, DEV)
    freed = torch.full((CFG.S * wl.max_blocks,), -7, dtype=torch.int32, device=DEV)
    count = torch.full((1,), -7, dtype=torch.int32, device=DEV)
    idx = torch.full((CFG.S, CFG.L, CFG.Hkv, CFG.budget), -7, dtype=torch.int32, device=DEV)
    tri.tri_compress_step_ex(cache, qbar, qabs, R, CFG.base, wl.deltas, opt, ws, free_list=fl, freed_ids=freed,
                             freed_count=count, idx_out=idx)
    code = tri.tri_sync_status(cache.status)
    if fails:
        assert code == tri.TRI_ERR_STATS
        assert torch.equal(wl.k_pool.view(torch.int16), k0.view(torch.int16))
        assert torch.equal(wl.v_pool.view(torch.int16), v0.view(torch.int16))
        assert torch.equal(wl.seq_len, len0)
        assert int(count.item()) == 0 and (freed == -7).all()
        assert (idx == -7).all()
        assert fl.contents() == [900001, 900002]
    else:
        # a mismatched R alone is reported per head but does not stop the step
        assert code == tri.TRI_OK
        assert int(count.item()) > 0 and len(fl.contents()) == 2 + int(count.item())


def test_check_on_valid_statistics_equals_the_plain_step():
    a = make_workload(CFG, device=DEV, seed=3)
    b = make_workload(CFG, device=DEV, seed=3)
    stats = gpu_stats(a)
    outs = []
    for wl, check in ((a, True), (b, False)):
        cache = cache_of(wl)
        opt = tri.step_options(CFG.budget, CFG.window, check_stats=check)
        ws = tri.alloc_workspace(cache, opt)
        freed = torch.empty(CFG.S * wl.max_blocks, dtype=torch.int32, device=DEV)
        count = torch.empty(1, dtype=torch.int32, device=DEV)
        idx = torch.full((CFG.S, CFG.L, CFG.Hkv, CFG.budget), -7, dtype=torch.int32, device=DEV)
        tri.tri_compress_step_ex(cache, *stats, CFG.base, wl.deltas, opt, ws, freed_ids=freed, freed_count=count,
                                 idx_out=idx)
        assert tri.tri_sync_status(cache.status) == tri.TRI_OK
        n = int(count.item())
        outs.append((idx, freed[:n].clone(), wl.seq_len.clone(), wl.k_pool.view(torch.int16),
                     wl.v_pool.view(torch.int16)))
    for x, y in zip(*outs):
        assert torch.equal(x, y)
