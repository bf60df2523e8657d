"""The C-ABI library on the host (CPU only, no CUDA call is made).

Checks that the in-tree shared library loads, exports every function that
include/tri_attention.h declares, and rejects bad arguments on the host with
the documented status before anything is launched.  The pointers passed are
never dereferenced: every case here fails validation first.
"""

import ctypes
import os
import re

import pytest

import rope_aware_kv_tri_b200 as tri
from rope_aware_kv_tri_b200 import build_lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "tri_attention.h")


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return tri.library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tri_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_function(lib):
    names = declared_functions()
    assert set(names) == set(tri.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_static_scratch_size_matches_header(lib):
    m = re.search(r"#define\s+TRI_STATIC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", open(HEADER).read())
    assert m, "TRI_STATIC_SCRATCH_BYTES not found in the header"
    assert tri.tri_static_scratch_bytes() == int(m.group(1)) << int(m.group(2))


def test_status_strings(lib):
    assert tri.tri_status_string(0) == "ok"
    for code in range(1, 9):
        assert tri.tri_status_string(code) not in ("ok", "unknown status")
    assert tri.tri_status_string(99) == "unknown status"


FAKE = 1 << 40           # 16-byte aligned, never dereferenced


def test_selftest_wait_rejects_bad_pointers(lib):
    assert lib.tri_selftest_bounded_wait(None, None, None) == tri.TRI_ERR_INVALID
    assert lib.tri_selftest_bounded_wait(FAKE + 2, None, None) == tri.TRI_ERR_INVALID
    assert lib.tri_selftest_bounded_wait(FAKE, FAKE + 1, None) == tri.TRI_ERR_INVALID


def _desc(**kw):
    d = dict(L=2, Hkv=8, G=4, D=128, block_size=16, k_pool=FAKE, v_pool=FAKE + 4096, num_blocks=100,
             block_table=FAKE, S=2, max_blocks=50, seq_len=FAKE, cur_pos=FAKE, status=FAKE)
    d.update(kw)
    return tri.TriKvDesc(**d)


def _step(lib, desc, budget=64, window=8, deltas=(1, 2, 4), ws_bytes=None, base=1e4, stats=FAKE,
          freed=FAKE, ws=FAKE):
    arr = (ctypes.c_int32 * max(len(deltas), 1))(*deltas)
    if ws_bytes is None:
        ws_bytes = lib.tri_workspace_size(ctypes.byref(desc), budget) if desc is not None else 0
    return lib.tri_compress_step(ctypes.byref(desc) if desc is not None else None, stats, FAKE, FAKE,
                                 base, arr, len(deltas), budget, window, freed, FAKE, None, ws, ws_bytes,
                                 None, None)


def test_workspace_size(lib):
    d = _desc()
    n = lib.tri_workspace_size(ctypes.byref(d), 64)
    U, max_len = 2 * 2 * 8, 50 * 16
    assert n >= U * max_len * 4 + U * 192 * 4
    assert n % 256 == 0
    assert lib.tri_workspace_size(ctypes.byref(_desc(S=4)), 64) > n
    assert lib.tri_workspace_size(ctypes.byref(_desc(D=64)), 64) == 0
    assert lib.tri_workspace_size(None, 64) == 0


@pytest.mark.parametrize("case,expect", [
    (dict(desc=None), tri.TRI_ERR_INVALID),
    (dict(D=64), tri.TRI_ERR_UNSUPPORTED),
    (dict(block_size=32), tri.TRI_ERR_UNSUPPORTED),
    (dict(L=0), tri.TRI_ERR_INVALID),
    (dict(Hkv=0), tri.TRI_ERR_INVALID),
    (dict(G=0), tri.TRI_ERR_INVALID),
    (dict(S=-1), tri.TRI_ERR_INVALID),
    (dict(num_blocks=0), tri.TRI_ERR_INVALID),
    (dict(max_blocks=0), tri.TRI_ERR_INVALID),
    (dict(k_pool=None), tri.TRI_ERR_INVALID),
    (dict(v_pool=FAKE + 8), tri.TRI_ERR_INVALID),          # not 16-byte aligned
    (dict(seq_len=None), tri.TRI_ERR_INVALID),
    (dict(cur_pos=FAKE + 4), tri.TRI_ERR_INVALID),         # int64 misaligned
    (dict(status=None), tri.TRI_ERR_INVALID),
    (dict(max_blocks=1 << 28), tri.TRI_ERR_INVALID),       # slot count overflows int32
    (dict(budget=0), tri.TRI_ERR_INVALID),
    (dict(window=65), tri.TRI_ERR_INVALID),                 # window > budget
    (dict(window=-1), tri.TRI_ERR_INVALID),
    (dict(budget=20000, window=0), tri.TRI_ERR_UNSUPPORTED),
    (dict(deltas=()), tri.TRI_ERR_INVALID),
    (dict(deltas=tuple(range(1, 66))), tri.TRI_ERR_INVALID),
    (dict(base=0.0), tri.TRI_ERR_INVALID),
    (dict(base=float("nan")), tri.TRI_ERR_INVALID),
    (dict(stats=None), tri.TRI_ERR_INVALID),
    (dict(freed=None), tri.TRI_ERR_INVALID),
    (dict(ws=None), tri.TRI_ERR_WORKSPACE),
    (dict(ws=FAKE + 16), tri.TRI_ERR_WORKSPACE),           # not 256-byte aligned
    (dict(ws_bytes=1024), tri.TRI_ERR_WORKSPACE),
])
def test_step_rejects_on_host(lib, case, expect):
    case = dict(case)
    desc_kw = {k: case.pop(k) for k in list(case) if k in tri.TriKvDesc.__dict__ or k in
               ("L", "Hkv", "G", "D", "block_size", "k_pool", "v_pool", "num_blocks", "block_table", "S",
                "max_blocks", "seq_len", "cur_pos", "status")}
    desc = case.pop("desc") if "desc" in case else _desc(**desc_kw)
    assert _step(lib, desc, **case) == expect


def test_other_entry_points_reject_on_host(lib):
    d = _desc()
    dp = ctypes.byref(d)
    arr = (ctypes.c_int32 * 1)(1)
    assert lib.tri_calibrate_centers(None, 4, 1, 1, 128, FAKE, FAKE, FAKE, None) == tri.TRI_ERR_INVALID
    assert lib.tri_calibrate_centers(FAKE, 0, 1, 1, 128, FAKE, FAKE, FAKE, None) == tri.TRI_ERR_INVALID
    assert lib.tri_calibrate_centers(FAKE, 4, 1, 1, 96, FAKE, FAKE, FAKE, None) == tri.TRI_ERR_UNSUPPORTED
    assert lib.tri_build_query(dp, FAKE, FAKE, FAKE, 1e4, arr, 1, None, FAKE, None) == tri.TRI_ERR_INVALID
    assert lib.tri_score(dp, FAKE, FAKE, FAKE, 1e4, arr, 1, FAKE, FAKE, 16, None) == tri.TRI_ERR_WORKSPACE
    assert lib.tri_select_topk(dp, FAKE, 8, 9, FAKE, FAKE, None) == tri.TRI_ERR_INVALID
    assert lib.tri_select_topk(dp, None, 8, 2, FAKE, FAKE, None) == tri.TRI_ERR_INVALID
    assert lib.tri_compact_kv(dp, FAKE, FAKE, 0, FAKE, FAKE, None) == tri.TRI_ERR_INVALID
    assert lib.tri_compact_kv(dp, FAKE, FAKE, 8, None, FAKE, None) == tri.TRI_ERR_INVALID
    assert lib.tri_sync_status(None, None) == tri.TRI_ERR_INVALID


def test_binding_refuses_cpu_tensors(lib):
    import torch
    with pytest.raises(ValueError):
        tri.tri_calibrate_centers(torch.zeros(2, 1, 1, 128), torch.zeros(1, 1, 128), torch.zeros(1, 1, 64),
                                  torch.zeros(1, 1))


def _opts(**kw):
    o = dict(budget=64, window=8, sinks=0, trigger=0, aggregate=tri.TRI_AGG_MEAN)
    o.update(kw)
    return tri.TriStepOptions(**o)


def _step_ex(lib, desc, opt, free_list=None, freed=FAKE, count=FAKE, ws_bytes=None):
    arr = (ctypes.c_int32 * 3)(1, 2, 4)
    if ws_bytes is None:
        ws_bytes = lib.tri_workspace_size_ex(ctypes.byref(desc), ctypes.byref(opt)) or (1 << 40)
    return lib.tri_compress_step_ex(ctypes.byref(desc), FAKE, FAKE, FAKE, 1e4, arr, 3,
                                    ctypes.byref(opt) if opt is not None else None,
                                    ctypes.byref(free_list) if free_list is not None else None,
                                    freed, count, None, FAKE, ws_bytes, None, None)


def test_workspace_size_ex(lib):
    d = _desc()
    mean = lib.tri_workspace_size_ex(ctypes.byref(d), ctypes.byref(_opts()))
    assert mean == lib.tri_workspace_size(ctypes.byref(d), 64)
    mx = lib.tri_workspace_size_ex(ctypes.byref(d), ctypes.byref(_opts(aggregate=tri.TRI_AGG_MAX)))
    U = 2 * 2 * 8
    assert mx >= mean + (4 - 1) * U * 192 * 4 - 512          # G = 4 coefficient sets per unit
    assert lib.tri_workspace_size_ex(ctypes.byref(_desc(G=3)), ctypes.byref(_opts(aggregate=1))) == 0
    assert lib.tri_workspace_size_ex(ctypes.byref(d), ctypes.byref(_opts(sinks=60))) == 0
    assert lib.tri_workspace_size_ex(ctypes.byref(d), None) == 0


@pytest.mark.parametrize("opt,expect", [
    (None, tri.TRI_ERR_INVALID),
    (dict(sinks=-1), tri.TRI_ERR_INVALID),
    (dict(sinks=57), tri.TRI_ERR_INVALID),                 # sinks + window > budget
    (dict(trigger=-5), tri.TRI_ERR_INVALID),
    (dict(aggregate=7), tri.TRI_ERR_INVALID),
    (dict(budget=0), tri.TRI_ERR_INVALID),
    (dict(budget=tri.TRI_MAX_BUDGET + 1, window=0), tri.TRI_ERR_UNSUPPORTED),
])
def test_step_ex_rejects_options(lib, opt, expect):
    o = None if opt is None else _opts(**opt)
    assert _step_ex(lib, _desc(), o, ws_bytes=1 << 40) == expect


def test_step_ex_rejects_max_for_odd_group(lib):
    assert _step_ex(lib, _desc(G=3), _opts(aggregate=tri.TRI_AGG_MAX), ws_bytes=1 << 40) == tri.TRI_ERR_UNSUPPORTED


def test_step_ex_output_rules(lib):
    d = _desc()
    # neither freed ids nor a free list
    assert _step_ex(lib, d, _opts(), freed=None, count=None) == tri.TRI_ERR_INVALID
    # freed ids without a count
    assert _step_ex(lib, d, _opts(), freed=FAKE, count=None) == tri.TRI_ERR_INVALID
    bad = tri.TriFreeList(ids=None, count=FAKE, capacity=10)
    assert _step_ex(lib, d, _opts(), free_list=bad) == tri.TRI_ERR_INVALID
    neg = tri.TriFreeList(ids=FAKE, count=FAKE, capacity=-1)
    assert _step_ex(lib, d, _opts(), free_list=neg) == tri.TRI_ERR_INVALID
    # the max workspace is larger than the mean one
    mean_bytes = lib.tri_workspace_size_ex(ctypes.byref(d), ctypes.byref(_opts()))
    assert _step_ex(lib, d, _opts(aggregate=tri.TRI_AGG_MAX), ws_bytes=mean_bytes) == tri.TRI_ERR_WORKSPACE


def test_select_ex_and_score_ex_reject(lib):
    d = _desc()
    assert lib.tri_select_topk_ex(ctypes.byref(d), FAKE, ctypes.byref(_opts(sinks=57)), FAKE, FAKE,
                                  None) == tri.TRI_ERR_INVALID
    assert lib.tri_select_topk_ex(ctypes.byref(d), FAKE + 4, ctypes.byref(_opts()), FAKE, FAKE,
                                  None) == tri.TRI_ERR_INVALID      # scores not 16-byte aligned
    arr = (ctypes.c_int32 * 1)(1)
    assert lib.tri_score_ex(ctypes.byref(d), FAKE, FAKE, FAKE, 1e4, arr, 1, 5, FAKE, FAKE, 1 << 40,
                            None) == tri.TRI_ERR_INVALID
    assert lib.tri_score_ex(ctypes.byref(_desc(G=6)), FAKE, FAKE, FAKE, 1e4, arr, 1, tri.TRI_AGG_MAX, FAKE,
                            FAKE, 1 << 40, None) == tri.TRI_ERR_UNSUPPORTED


def test_reserve_rejects(lib):
    d = _desc()
    fl = tri.TriFreeList(ids=FAKE, count=FAKE, capacity=10)
    assert lib.tri_reserve_blocks(ctypes.byref(d), FAKE + 64, FAKE, ctypes.byref(fl), None) == tri.TRI_ERR_INVALID
    assert lib.tri_reserve_blocks(ctypes.byref(d), FAKE, FAKE, None, None) == tri.TRI_ERR_INVALID
    assert lib.tri_reserve_blocks(ctypes.byref(d), FAKE, None, ctypes.byref(fl), None) == tri.TRI_ERR_INVALID
    assert lib.tri_reserve_blocks(ctypes.byref(_desc(D=64)), FAKE, FAKE, ctypes.byref(fl),
                                  None) == tri.TRI_ERR_UNSUPPORTED


def test_distance_entries_reject(lib):
    arr = (ctypes.c_int32 * 2)(1, 2)
    ok = dict(L=2, Hkv=8, G=4, D=128, qbar=FAKE, kbar=FAKE, base=1e4, deltas=arr, n=2, agg=0, max_dist=100, table=FAKE)

    def table(**kw):
        a = dict(ok)
        a.update(kw)
        return lib.tri_distance_table(a["L"], a["Hkv"], a["G"], a["D"], a["qbar"], a["kbar"], a["base"],
                                      a["deltas"], a["n"], a["agg"], a["max_dist"], a["table"], None)
    assert table(D=64) == tri.TRI_ERR_UNSUPPORTED
    assert table(L=0) == tri.TRI_ERR_INVALID
    assert table(kbar=None) == tri.TRI_ERR_INVALID
    assert table(max_dist=0) == tri.TRI_ERR_INVALID
    assert table(max_dist=1 << 24) == tri.TRI_ERR_INVALID
    assert table(agg=9) == tri.TRI_ERR_INVALID
    assert table(agg=tri.TRI_AGG_MAX, G=65) == tri.TRI_ERR_UNSUPPORTED
    assert table(n=0) == tri.TRI_ERR_INVALID
    d = _desc()
    assert lib.tri_score_distance(ctypes.byref(d), FAKE, 100, None, FAKE, None) == tri.TRI_ERR_INVALID
    assert lib.tri_score_distance(ctypes.byref(d), FAKE, 0, FAKE, FAKE, None) == tri.TRI_ERR_INVALID
    o = _opts()
    step = lambda **kw: lib.tri_compress_step_distance(  # noqa: E731
        ctypes.byref(d), kw.get("table", FAKE), kw.get("max_dist", 100), kw.get("pos", FAKE), ctypes.byref(kw.get("o", o)),
        None, kw.get("freed", FAKE), kw.get("count", FAKE), None, FAKE, kw.get("ws", 1 << 40), None, None)
    assert step(pos=None) == tri.TRI_ERR_INVALID
    assert step(o=_opts(sinks=60)) == tri.TRI_ERR_INVALID
    assert step(freed=None, count=None) == tri.TRI_ERR_INVALID
    assert step(ws=64) == tri.TRI_ERR_WORKSPACE


def test_distance_alignment_rules(lib):
    d = _desc()
    assert lib.tri_score_distance(ctypes.byref(d), FAKE, 100, FAKE + 4, FAKE, None) == tri.TRI_ERR_INVALID
    assert lib.tri_score_distance(ctypes.byref(d), FAKE, 100, FAKE, FAKE + 8, None) == tri.TRI_ERR_INVALID


def test_check_stats_rejects(lib):
    assert lib.tri_check_stats(None, FAKE, FAKE, 2, 4, 128, None, FAKE, None) == tri.TRI_ERR_INVALID
    assert lib.tri_check_stats(FAKE, FAKE, FAKE, 0, 4, 128, None, FAKE, None) == tri.TRI_ERR_INVALID
    assert lib.tri_check_stats(FAKE, FAKE, FAKE, 2, 0, 128, None, FAKE, None) == tri.TRI_ERR_INVALID
    assert lib.tri_check_stats(FAKE, FAKE, FAKE, 2, 4, 64, None, FAKE, None) == tri.TRI_ERR_UNSUPPORTED
    assert lib.tri_check_stats(FAKE, FAKE, FAKE, 2, 4, 128, None, None, None) == tri.TRI_ERR_INVALID
    assert lib.tri_check_stats(FAKE, FAKE, FAKE, 2, 4, 128, FAKE + 2, FAKE, None) == tri.TRI_ERR_INVALID
    assert lib.tri_check_stats(FAKE + 1, FAKE, FAKE, 2, 4, 128, None, FAKE, None) == tri.TRI_ERR_INVALID
    assert lib.tri_check_stats(FAKE, FAKE, FAKE, 1 << 16, 1 << 16, 128, None, FAKE, None) == tri.TRI_ERR_INVALID
    assert tri.tri_status_string(tri.TRI_ERR_STATS) == "head statistics failed the sanity check"


def test_step_options_mirror_has_check_stats(lib):
    o = tri.step_options(64, 8, check_stats=True)
    assert o.check_stats == 1 and ctypes.sizeof(o) == 6 * ctypes.sizeof(ctypes.c_int)
    assert tri.step_options(64, 8).check_stats == 0
