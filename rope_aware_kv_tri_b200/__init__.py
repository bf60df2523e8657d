"""Python binding of the B200 TriAttention key-importance + eviction library.

Argument marshalling only: every function here takes torch tensors, checks
that they are CUDA tensors of the dtype and layout the C ABI documents
(``include/tri_attention.h``), and forwards their device pointers and the
current CUDA stream to the function of the same name in ``libtriattn.so``.
No step of the path runs in Python, and there is no fallback: if the shared
library is missing, every call raises.

Build the library with ``python -m rope_aware_kv_tri_b200.build_lib``.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libtriattn.so")

TRI_OK = 0
TRI_ERR_INVALID = 1
TRI_ERR_UNSUPPORTED = 2
TRI_ERR_CUDA = 3
TRI_ERR_DEVICE_BOUNDS = 4
TRI_ERR_TIMEOUT = 5
TRI_ERR_NONFINITE = 6
TRI_ERR_WORKSPACE = 7
TRI_ERR_FREELIST = 8
TRI_ERR_STATS = 9

TRI_DEVFLAG_STATS = 16
TRI_STATS_NONFINITE = 1
TRI_STATS_R_RANGE = 2
TRI_STATS_NORM_WEIGHT = 4
TRI_STATS_R_MISMATCH = 8

TRI_AGG_MEAN = 0
TRI_AGG_MAX = 1

TRI_HEAD_DIM = 128
TRI_BLOCK_SIZE = 16
TRI_MAX_DELTAS = 64
TRI_MAX_BUDGET = 16384

# Every symbol include/tri_attention.h declares.
EXPORTS = (
    "tri_calibrate_centers", "tri_build_query", "tri_workspace_size", "tri_score",
    "tri_select_topk", "tri_compact_kv", "tri_compress_step", "tri_compress_step_static_scratch",
    "tri_sync_status", "tri_status_string", "tri_workspace_size_ex", "tri_score_ex", "tri_select_topk_ex",
    "tri_compress_step_ex", "tri_reserve_blocks", "tri_distance_table", "tri_score_distance",
    "tri_compress_step_distance", "tri_selftest_bounded_wait", "tri_static_scratch_bytes",
    "tri_check_stats", "tri_step_is_fused",
)


class TriError(RuntimeError):
    """A non-OK tri_status from the library."""

    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {tri_status_string(code)} (status {code})")


class TriKvDesc(ctypes.Structure):
    """Mirror of ``tri_kv_desc``."""

    _fields_ = [
        ("L", ctypes.c_int), ("Hkv", ctypes.c_int), ("G", ctypes.c_int), ("D", ctypes.c_int),
        ("block_size", ctypes.c_int),
        ("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p), ("num_blocks", ctypes.c_int),
        ("block_table", ctypes.c_void_p), ("S", ctypes.c_int), ("max_blocks", ctypes.c_int),
        ("seq_len", ctypes.c_void_p), ("cur_pos", ctypes.c_void_p), ("status", ctypes.c_void_p),
    ]


class TriPhaseEvents(ctypes.Structure):
    """Mirror of ``tri_phase_events`` (cudaEvent_t handles or NULL)."""

    _fields_ = [("start", ctypes.c_void_p), ("after_query", ctypes.c_void_p),
                ("after_score", ctypes.c_void_p), ("after_evict", ctypes.c_void_p)]


class TriStepOptions(ctypes.Structure):
    """Mirror of ``tri_step_options``."""

    _fields_ = [("budget", ctypes.c_int), ("window", ctypes.c_int), ("sinks", ctypes.c_int),
                ("trigger", ctypes.c_int), ("aggregate", ctypes.c_int), ("check_stats", ctypes.c_int)]


class TriFreeList(ctypes.Structure):
    """Mirror of ``tri_free_list``."""

    _fields_ = [("ids", ctypes.c_void_p), ("count", ctypes.c_void_p), ("capacity", ctypes.c_int)]


class FreeList:
    """A device-resident stack of free block ids (int32 ``ids`` of length
    capacity, int32 ``count`` of one element), kept alive with its mirror."""

    def __init__(self, ids: torch.Tensor, count: torch.Tensor):
        if ids.dim() != 1 or count.numel() != 1:
            raise ValueError("ids must be 1-D and count a single element")
        self.ids, self.count = ids, count
        self.c = TriFreeList(ids=_ptr(ids, torch.int32, "ids"), count=_ptr(count, torch.int32, "count"),
                             capacity=ids.numel())

    @classmethod
    def from_ids(cls, free_ids, capacity: int, device) -> "FreeList":
        ids = torch.full((capacity,), -1, dtype=torch.int32, device=device)
        free = torch.as_tensor(list(free_ids), dtype=torch.int32)
        if free.numel() > capacity:
            raise ValueError("more free ids than capacity")
        ids[:free.numel()] = free.to(device)
        return cls(ids, torch.tensor([free.numel()], dtype=torch.int32, device=device))

    def contents(self):
        n = int(self.count.item())
        return [int(x) for x in self.ids[:n].tolist()]

    @property
    def ref(self):
        return ctypes.byref(self.c)


def step_options(budget: int, window: int, sinks: int = 0, trigger: int = 0,
                 aggregate: int = TRI_AGG_MEAN, check_stats: bool = False) -> TriStepOptions:
    return TriStepOptions(int(budget), int(window), int(sinks), int(trigger), int(aggregate), int(bool(check_stats)))


_lib: Optional[ctypes.CDLL] = None


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"TriAttention CUDA library not built ({LIB_PATH} missing); "
            "run `python -m rope_aware_kv_tri_b200.build_lib`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, D, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_size_t
    desc_p = ctypes.POINTER(TriKvDesc)
    sig = {
        "tri_calibrate_centers": (I, [P, I, I, I, I, P, P, P, P]),
        "tri_build_query": (I, [desc_p, P, P, P, D, P, I, P, P, P]),
        "tri_workspace_size": (S, [desc_p, I]),
        "tri_score": (I, [desc_p, P, P, P, D, P, I, P, P, S, P]),
        "tri_select_topk": (I, [desc_p, P, I, I, P, P, P]),
        "tri_compact_kv": (I, [desc_p, P, P, I, P, P, P]),
        "tri_compress_step": (I, [desc_p, P, P, P, D, P, I, I, I, P, P, P, P, S,
                                  ctypes.POINTER(TriPhaseEvents), P]),
        "tri_compress_step_static_scratch": (I, [desc_p, P, P, P, D, P, I, I, I, P, P, P, P]),
        "tri_sync_status": (I, [P, P]),
        "tri_workspace_size_ex": (S, [desc_p, ctypes.POINTER(TriStepOptions)]),
        "tri_score_ex": (I, [desc_p, P, P, P, D, P, I, I, P, P, S, P]),
        "tri_select_topk_ex": (I, [desc_p, P, ctypes.POINTER(TriStepOptions), P, P, P]),
        "tri_compress_step_ex": (I, [desc_p, P, P, P, D, P, I, ctypes.POINTER(TriStepOptions),
                                     ctypes.POINTER(TriFreeList), P, P, P, P, S,
                                     ctypes.POINTER(TriPhaseEvents), P]),
        "tri_reserve_blocks": (I, [desc_p, P, P, ctypes.POINTER(TriFreeList), P]),
        "tri_distance_table": (I, [I, I, I, I, P, P, D, P, I, I, I, P, P]),
        "tri_score_distance": (I, [desc_p, P, I, P, P, P]),
        "tri_compress_step_distance": (I, [desc_p, P, I, P, ctypes.POINTER(TriStepOptions),
                                           ctypes.POINTER(TriFreeList), P, P, P, P, S,
                                           ctypes.POINTER(TriPhaseEvents), P]),
        "tri_status_string": (ctypes.c_char_p, [I]),
        "tri_selftest_bounded_wait": (I, [P, P, P]),
        "tri_static_scratch_bytes": (S, []),
        "tri_check_stats": (I, [P, P, P, I, I, I, P, P, P]),
        "tri_step_is_fused": (I, [desc_p, ctypes.POINTER(TriStepOptions)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def library() -> ctypes.CDLL:
    """The loaded shared library (loads it on first use; raises if missing)."""
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


# ----------------------------------------------------------------- helpers

def _ptr(t: Optional[torch.Tensor], dtype: torch.dtype, name: str, allow_none: bool = False):
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _deltas(deltas: Sequence[int]):
    arr = (ctypes.c_int32 * max(len(deltas), 1))(*[int(d) for d in deltas])
    return arr, len(deltas)


def _check(code: int, where: str) -> None:
    if code != TRI_OK:
        raise TriError(code, where)


class KvCache:
    """Keeps the tensors of one paged cache alive together with its descriptor.

    k_pool, v_pool : bf16 [L][num_blocks][Hkv][16][128]
    block_table    : int32 [S][max_blocks]
    seq_len        : int32 [S]      cur_pos : int64 [S]
    status         : int32 [1]      (device status word)
    """

    def __init__(self, k_pool, v_pool, block_table, seq_len, cur_pos, status, G: int):
        L, NB, Hkv, bs, D = k_pool.shape
        self.tensors = (k_pool, v_pool, block_table, seq_len, cur_pos, status)
        self.desc = TriKvDesc(
            L=L, Hkv=Hkv, G=G, D=D, block_size=bs,
            k_pool=_ptr(k_pool, torch.bfloat16, "k_pool"), v_pool=_ptr(v_pool, torch.bfloat16, "v_pool"),
            num_blocks=NB, block_table=_ptr(block_table, torch.int32, "block_table"),
            S=block_table.shape[0], max_blocks=block_table.shape[1],
            seq_len=_ptr(seq_len, torch.int32, "seq_len"), cur_pos=_ptr(cur_pos, torch.int64, "cur_pos"),
            status=_ptr(status, torch.int32, "status"))
        if tuple(v_pool.shape) != tuple(k_pool.shape):
            raise ValueError("k_pool and v_pool shapes differ")

    @property
    def ref(self):
        return ctypes.byref(self.desc)

    @property
    def status(self) -> torch.Tensor:
        return self.tensors[5]


# ------------------------------------------------------------ entry points

def tri_status_string(code: int) -> str:
    return library().tri_status_string(int(code)).decode()


def tri_calibrate_centers(q_pre, qbar, qabs, R, stream=None) -> None:
    N, L, Hq, D = q_pre.shape
    code = library().tri_calibrate_centers(
        _ptr(q_pre, torch.float32, "q_pre"), N, L, Hq, D, _ptr(qbar, torch.float32, "qbar"),
        _ptr(qabs, torch.float32, "qabs"), _ptr(R, torch.float32, "R"), _stream(stream))
    _check(code, "tri_calibrate_centers")


def tri_build_query(cache: KvCache, qbar, qabs, R, rope_base: float, deltas, qeff, w, stream=None) -> None:
    arr, n = _deltas(deltas)
    code = library().tri_build_query(
        cache.ref, _ptr(qbar, torch.float32, "qbar"), _ptr(qabs, torch.float32, "qabs"),
        _ptr(R, torch.float32, "R"), float(rope_base), arr, n, _ptr(qeff, torch.float32, "qeff"),
        _ptr(w, torch.float32, "w"), _stream(stream))
    _check(code, "tri_build_query")


def tri_workspace_size(cache: KvCache, budget: int) -> int:
    return int(library().tri_workspace_size(cache.ref, int(budget)))


def tri_score(cache: KvCache, qbar, qabs, R, rope_base: float, deltas, scores, workspace, stream=None) -> None:
    arr, n = _deltas(deltas)
    code = library().tri_score(
        cache.ref, _ptr(qbar, torch.float32, "qbar"), _ptr(qabs, torch.float32, "qabs"),
        _ptr(R, torch.float32, "R"), float(rope_base), arr, n, _ptr(scores, torch.float32, "scores"),
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream))
    _check(code, "tri_score")


def tri_select_topk(cache: KvCache, scores, budget: int, window: int, idx, kept, stream=None) -> None:
    code = library().tri_select_topk(
        cache.ref, _ptr(scores, torch.float32, "scores"), int(budget), int(window),
        _ptr(idx, torch.int32, "idx"), _ptr(kept, torch.int32, "kept"), _stream(stream))
    _check(code, "tri_select_topk")


def tri_compact_kv(cache: KvCache, idx, kept, budget: int, freed_ids, freed_count, stream=None) -> None:
    code = library().tri_compact_kv(
        cache.ref, _ptr(idx, torch.int32, "idx"), _ptr(kept, torch.int32, "kept"), int(budget),
        _ptr(freed_ids, torch.int32, "freed_ids"), _ptr(freed_count, torch.int32, "freed_count"),
        _stream(stream))
    _check(code, "tri_compact_kv")


def _events(events):
    if events is None:
        return None
    handles = []
    for e in events:
        if e is None:
            handles.append(None)
            continue
        if e.cuda_event == 0:          # torch creates the CUDA event lazily
            e.record()
        handles.append(ctypes.c_void_p(e.cuda_event))
    return ctypes.byref(TriPhaseEvents(*handles))


def tri_compress_step(cache: KvCache, qbar, qabs, R, rope_base: float, deltas, budget: int, window: int,
                      freed_ids, freed_count, workspace, idx_out=None, events=None, stream=None) -> None:
    """``events``: optional sequence of four recorded-or-fresh torch.cuda.Event
    (start, after_query, after_score, after_evict), each with enable_timing."""
    arr, n = _deltas(deltas)
    ev = _events(events)
    code = library().tri_compress_step(
        cache.ref, _ptr(qbar, torch.float32, "qbar"), _ptr(qabs, torch.float32, "qabs"),
        _ptr(R, torch.float32, "R"), float(rope_base), arr, n, int(budget), int(window),
        _ptr(freed_ids, torch.int32, "freed_ids"), _ptr(freed_count, torch.int32, "freed_count"),
        _ptr(idx_out, torch.int32, "idx_out", allow_none=True),
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), ev, _stream(stream))
    _check(code, "tri_compress_step")


def tri_static_scratch_bytes() -> int:
    """Bytes of the fixed device scratch built into the library (the
    largest workspace tri_compress_step_static_scratch can serve)."""
    return int(library().tri_static_scratch_bytes())


def tri_compress_step_static_scratch(cache: KvCache, qbar, qabs, R, rope_base: float, deltas, budget: int,
                                     window: int, freed_ids, freed_count, idx_out=None, stream=None) -> None:
    """tri_compress_step without a workspace argument: the library's own
    fixed device scratch (TRI_STATIC_SCRATCH_BYTES) is used instead, for
    callers that cannot allocate device memory.  Calls must not overlap on
    the GPU; the first call on a device should precede any graph capture."""
    arr, n = _deltas(deltas)
    code = library().tri_compress_step_static_scratch(
        cache.ref, _ptr(qbar, torch.float32, "qbar"), _ptr(qabs, torch.float32, "qabs"),
        _ptr(R, torch.float32, "R"), float(rope_base), arr, n, int(budget), int(window),
        _ptr(freed_ids, torch.int32, "freed_ids"), _ptr(freed_count, torch.int32, "freed_count"),
        _ptr(idx_out, torch.int32, "idx_out", allow_none=True), _stream(stream))
    _check(code, "tri_compress_step_static_scratch")


def tri_workspace_size_ex(cache: KvCache, opt: TriStepOptions) -> int:
    return int(library().tri_workspace_size_ex(cache.ref, ctypes.byref(opt)))


def tri_score_ex(cache: KvCache, qbar, qabs, R, rope_base: float, deltas, aggregate: int, scores, workspace,
                 stream=None) -> None:
    arr, n = _deltas(deltas)
    code = library().tri_score_ex(
        cache.ref, _ptr(qbar, torch.float32, "qbar"), _ptr(qabs, torch.float32, "qabs"),
        _ptr(R, torch.float32, "R"), float(rope_base), arr, n, int(aggregate),
        _ptr(scores, torch.float32, "scores"), _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
        _stream(stream))
    _check(code, "tri_score_ex")


def tri_select_topk_ex(cache: KvCache, scores, opt: TriStepOptions, idx, kept, stream=None) -> None:
    code = library().tri_select_topk_ex(
        cache.ref, _ptr(scores, torch.float32, "scores"), ctypes.byref(opt), _ptr(idx, torch.int32, "idx"),
        _ptr(kept, torch.int32, "kept"), _stream(stream))
    _check(code, "tri_select_topk_ex")


def tri_compress_step_ex(cache: KvCache, qbar, qabs, R, rope_base: float, deltas, opt: TriStepOptions,
                         workspace, free_list: Optional[FreeList] = None, freed_ids=None, freed_count=None,
                         idx_out=None, events=None, stream=None) -> None:
    arr, n = _deltas(deltas)
    code = library().tri_compress_step_ex(
        cache.ref, _ptr(qbar, torch.float32, "qbar"), _ptr(qabs, torch.float32, "qabs"),
        _ptr(R, torch.float32, "R"), float(rope_base), arr, n, ctypes.byref(opt),
        free_list.ref if free_list is not None else None,
        _ptr(freed_ids, torch.int32, "freed_ids", allow_none=True),
        _ptr(freed_count, torch.int32, "freed_count", allow_none=True),
        _ptr(idx_out, torch.int32, "idx_out", allow_none=True),
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _events(events), _stream(stream))
    _check(code, "tri_compress_step_ex")


def tri_reserve_blocks(cache: KvCache, n_new, free_list: FreeList, stream=None) -> None:
    """Pop the blocks that n_new[s] more slots per sequence need from the
    free list into the cache's block table (seq_len is not changed)."""
    code = library().tri_reserve_blocks(
        cache.ref, _ptr(cache.tensors[2], torch.int32, "block_table"), _ptr(n_new, torch.int32, "n_new"),
        free_list.ref, _stream(stream))
    _check(code, "tri_reserve_blocks")


def tri_distance_table(qbar, kbar, rope_base: float, deltas, aggregate: int, table, stream=None) -> None:
    """qbar f32 [L][Hq][D], kbar f32 [L][Hkv][D] -> table f32 [L][Hkv][max_dist + 1]."""
    L, Hq, D = qbar.shape
    Hkv = kbar.shape[1]
    if Hq % Hkv or tuple(kbar.shape) != (L, Hkv, D) or table.dim() != 3 or tuple(table.shape[:2]) != (L, Hkv):
        raise ValueError("inconsistent shapes")
    arr, n = _deltas(deltas)
    code = library().tri_distance_table(
        L, Hkv, Hq // Hkv, D, _ptr(qbar, torch.float32, "qbar"), _ptr(kbar, torch.float32, "kbar"),
        float(rope_base), arr, n, int(aggregate), table.shape[2] - 1, _ptr(table, torch.float32, "table"),
        _stream(stream))
    _check(code, "tri_distance_table")


def tri_score_distance(cache: KvCache, table, slot_pos, scores, stream=None) -> None:
    code = library().tri_score_distance(
        cache.ref, _ptr(table, torch.float32, "table"), table.shape[-1] - 1, _ptr(slot_pos, torch.int32, "slot_pos"),
        _ptr(scores, torch.float32, "scores"), _stream(stream))
    _check(code, "tri_score_distance")


def tri_compress_step_distance(cache: KvCache, table, slot_pos, opt: TriStepOptions, workspace,
                               free_list: Optional[FreeList] = None, freed_ids=None, freed_count=None,
                               idx_out=None, events=None, stream=None) -> None:
    code = library().tri_compress_step_distance(
        cache.ref, _ptr(table, torch.float32, "table"), table.shape[-1] - 1, _ptr(slot_pos, torch.int32, "slot_pos"),
        ctypes.byref(opt), free_list.ref if free_list is not None else None,
        _ptr(freed_ids, torch.int32, "freed_ids", allow_none=True),
        _ptr(freed_count, torch.int32, "freed_count", allow_none=True),
        _ptr(idx_out, torch.int32, "idx_out", allow_none=True),
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _events(events), _stream(stream))
    _check(code, "tri_compress_step_distance")


def tri_step_is_fused(cache: KvCache, opt: TriStepOptions) -> bool:
    """Whether the step with these options runs as the one fused kernel."""
    r = int(library().tri_step_is_fused(cache.ref, ctypes.byref(opt)))
    if r < 0:
        raise TriError(TRI_ERR_INVALID, "tri_step_is_fused")
    return r == 1


def tri_check_stats(qbar, qabs, R, status, head_flags=None, stream=None) -> None:
    """Check head statistics qbar f32 [L][Hq][D], qabs f32 [L][Hq][D/2],
    R f32 [L][Hq]; per-head TRI_STATS_* bits go to head_flags (int32
    [L][Hq], optional) and TRI_DEVFLAG_STATS to the status word on a failure."""
    L, Hq, D = qbar.shape
    if tuple(qabs.shape) != (L, Hq, D // 2) or tuple(R.shape) != (L, Hq):
        raise ValueError("inconsistent statistics shapes")
    if head_flags is not None and tuple(head_flags.shape) != (L, Hq):
        raise ValueError("head_flags must be [L][Hq]")
    code = library().tri_check_stats(
        _ptr(qbar, torch.float32, "qbar"), _ptr(qabs, torch.float32, "qabs"), _ptr(R, torch.float32, "R"),
        L, Hq, D, _ptr(head_flags, torch.int32, "head_flags", allow_none=True),
        _ptr(status, torch.int32, "status"), _stream(stream))
    _check(code, "tri_check_stats")


def tri_sync_status(status, stream=None) -> int:
    """Wait for the stream, read and clear the device status word; returns the code."""
    return int(library().tri_sync_status(_ptr(status, torch.int32, "status"), _stream(stream)))


def tri_selftest_bounded_wait(status, flag=None, stream=None) -> None:
    """Launch the self-test wait (see the C header): it gives up after the
    library's wait limit unless ``flag`` (device int32) is non-zero."""
    fp = None if flag is None else _ptr(flag, torch.int32, "flag")
    _check(library().tri_selftest_bounded_wait(_ptr(status, torch.int32, "status"), fp, _stream(stream)),
           "tri_selftest_bounded_wait")


def alloc_workspace(cache: KvCache, budget, device=None) -> torch.Tensor:
    """A uint8 workspace of tri_workspace_size bytes, or of
    tri_workspace_size_ex bytes when ``budget`` is a TriStepOptions (torch
    allocations are 256-byte aligned)."""
    if isinstance(budget, TriStepOptions):
        n = tri_workspace_size_ex(cache, budget)
    else:
        n = tri_workspace_size(cache, budget)
    if n == 0:
        raise TriError(TRI_ERR_INVALID, "tri_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device or cache.tensors[0].device)
    if ws.data_ptr() % 256:
        raise RuntimeError("workspace is not 256-byte aligned")
    return ws
