"""The no-allocation entry point, tri_compress_step_static_scratch (GPU).

Some callers cannot allocate device memory at all: a serving engine that
gives nearly all of HBM to its paged KV block pool at start-up and forbids
allocation while decoding, or a plain-C plugin loaded into such an engine
with no allocator of its own.  For them the library offers a variant of
tri_compress_step that takes no workspace and works in a fixed scratch array
built into the library.

These tests call that entry point through the C ABI and check that, on two
calls in a row with different caches (so the second call starts from the
scratch contents the first one left behind), it produces exactly what
tri_compress_step with a caller workspace produces: the same kept slots,
bit-identical K/V pools, the same freed blocks and lengths; that further
calls leave the device's free memory and torch's allocated bytes unchanged;
and that shapes beyond the array, an invalid descriptor and a budget above
the library's maximum are refused before anything is launched.  The file is
named so that pytest collects it last.
"""

import pytest
import torch

import rope_aware_kv_tri_b200 as tri
from tests.gpu_helpers import cache_of, gpu_stats
from workload import CONFIGS, make_workload

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    CONFIGS["head1_t4096"],
    CONFIGS["l64h8g8_4x64k"].replace(L=2, lens=[700, 33, 1001, 16, 0, 530], budget=512, window=64, n_samples=256),
]


def _run(wl, stats, static: bool):
    cfg = wl.cfg
    S, L, Hkv, B = cfg.S, cfg.L, cfg.Hkv, cfg.budget
    cache = cache_of(wl)
    freed = torch.full((S * wl.max_blocks,), -7, dtype=torch.int32, device=DEV)
    count = torch.full((1,), -7, dtype=torch.int32, device=DEV)
    idx = torch.full((S, L, Hkv, B), -7, dtype=torch.int32, device=DEV)
    if static:
        tri.tri_compress_step_static_scratch(cache, *stats, cfg.base, wl.deltas, B, cfg.window, freed, count,
                                             idx_out=idx)
    else:
        ws = tri.alloc_workspace(cache, B)
        tri.tri_compress_step(cache, *stats, cfg.base, wl.deltas, B, cfg.window, freed, count, ws, idx_out=idx)
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    n = int(count.item())
    return idx, freed[:n].clone(), wl.seq_len.clone(), wl.k_pool, wl.v_pool


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rope_aware_kv_tri_b200 import build_lib
    build_lib.build()
    torch.cuda.init()


def test_static_scratch_matches_workspace_entry_on_two_calls_in_a_row():
    for seed, cfg in enumerate(CASES):
        a = make_workload(cfg, device=DEV, seed=seed)        # for the static-scratch call
        b = make_workload(cfg, device=DEV, seed=seed)        # identical copy for the workspace call
        assert tri.tri_workspace_size(cache_of(a), cfg.budget) <= tri.tri_static_scratch_bytes()
        stats = gpu_stats(a)
        got = _run(a, stats, static=True)
        want = _run(b, stats, static=False)
        assert torch.equal(got[0], want[0]), "kept slots differ"
        assert torch.equal(got[1], want[1]), "freed blocks differ"
        assert torch.equal(got[2], want[2]), "new lengths differ"
        assert torch.equal(got[3].view(torch.int16), want[3].view(torch.int16)), "K pool differs"
        assert torch.equal(got[4].view(torch.int16), want[4].view(torch.int16)), "V pool differs"


def test_static_scratch_rejects_shapes_beyond_its_size():
    # 4 layers x 8 heads x 131072 slots of fp32 scores alone exceed the array
    L, Hkv, max_blocks = 4, 8, 8192
    k = torch.zeros(L, 1, Hkv, 16, 128, dtype=torch.bfloat16, device=DEV)
    table = torch.zeros(1, max_blocks, dtype=torch.int32, device=DEV)
    cache = tri.KvCache(k, k.clone(), table, torch.zeros(1, dtype=torch.int32, device=DEV),
                        torch.zeros(1, dtype=torch.int64, device=DEV), torch.zeros(1, dtype=torch.int32, device=DEV), 4)
    assert tri.tri_workspace_size(cache, 64) > tri.tri_static_scratch_bytes()
    st = (torch.zeros(L, Hkv * 4, 128, device=DEV), torch.zeros(L, Hkv * 4, 64, device=DEV),
          torch.ones(L, Hkv * 4, device=DEV))
    freed = torch.empty(max_blocks, dtype=torch.int32, device=DEV)
    count = torch.empty(1, dtype=torch.int32, device=DEV)
    with pytest.raises(tri.TriError) as e:
        tri.tri_compress_step_static_scratch(cache, *st, 1e4, [1], 64, 8, freed, count)
    assert e.value.code == tri.TRI_ERR_UNSUPPORTED


def _small_cache_and_outputs(seed):
    cfg = CASES[1]
    wl = make_workload(cfg, device=DEV, seed=seed)
    freed = torch.empty(cfg.S * wl.max_blocks, dtype=torch.int32, device=DEV)
    count = torch.empty(1, dtype=torch.int32, device=DEV)
    return wl, cache_of(wl), freed, count


def test_static_scratch_calls_allocate_nothing():
    wl, cache, freed, count = _small_cache_and_outputs(5)
    cfg = wl.cfg
    stats = gpu_stats(wl)
    save = (wl.k_pool.clone(), wl.v_pool.clone(), wl.seq_len.clone())

    def call():
        wl.k_pool.copy_(save[0])
        wl.v_pool.copy_(save[1])
        wl.seq_len.copy_(save[2])
        tri.tri_compress_step_static_scratch(cache, *stats, cfg.base, wl.deltas, cfg.budget, cfg.window,
                                             freed, count)

    call()                                   # warm-up: module load, symbol lookup
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(3):
        tri.tri_compress_step_static_scratch(cache, *stats, cfg.base, wl.deltas, cfg.budget, cfg.window,
                                             freed, count)
    torch.cuda.synchronize()
    assert tri.tri_sync_status(cache.status) == tri.TRI_OK
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes"


def test_static_scratch_refuses_invalid_descriptor_and_budget():
    wl, cache, freed, count = _small_cache_and_outputs(6)
    cfg = wl.cfg
    stats = gpu_stats(wl)
    before = (wl.k_pool.clone(), wl.seq_len.clone())
    bad = tri.KvCache(wl.k_pool, wl.v_pool, wl.block_table, wl.seq_len, wl.cur_pos, cache.status, cfg.G)
    bad.desc.L = 0                                           # no layers: invalid descriptor
    with pytest.raises(tri.TriError) as e:
        tri.tri_compress_step_static_scratch(bad, *stats, cfg.base, wl.deltas, cfg.budget, cfg.window, freed, count)
    assert e.value.code == tri.TRI_ERR_INVALID
    with pytest.raises(tri.TriError) as e:
        tri.tri_compress_step_static_scratch(cache, *stats, cfg.base, wl.deltas, tri.TRI_MAX_BUDGET + 1,
                                             cfg.window, freed, count)
    assert e.value.code == tri.TRI_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.equal(wl.k_pool.view(torch.int16), before[0].view(torch.int16))
    assert torch.equal(wl.seq_len, before[1])
