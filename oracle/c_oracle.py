"""ctypes wrapper of the plain C oracle (tri_oracle_c.c).

TEST INFRASTRUCTURE: used by the tests and by the CPU legs of ``bench.py``
(the CPU baseline and the reference arm) to time the oracle on every host
core.  Built in-tree with gcc into ``oracle/_lib/libtrioracle.so``.
"""

from __future__ import annotations

import ctypes
import os
import shutil
import subprocess
import threading
from typing import Sequence, Tuple

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "tri_oracle_c.c")
LIB = os.path.join(HERE, "_lib", "libtrioracle.so")

_lib = None
_lock = threading.RLock()


def build(force: bool = False) -> str:
    """Compile the C oracle (plain -O2, no fast-math) if missing or stale.
    Safe to call from several threads or processes at once: each compiles
    to its own temporary file and renames it into place."""
    with _lock:
        if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
            return LIB
        cc = shutil.which("gcc") or shutil.which("cc")
        if cc is None:
            raise RuntimeError("no C compiler for the C oracle")
        os.makedirs(os.path.dirname(LIB), exist_ok=True)
        tmp = f"{LIB}.{os.getpid()}.tmp"
        subprocess.run([cc, "-O2", "-fPIC", "-shared", "-o", tmp, SRC, "-lm"], check=True, capture_output=True)
        os.replace(tmp, LIB)
        return LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P, I = ctypes.c_void_p, ctypes.c_int
        lib.tri_oracle_unit.restype = I
        lib.tri_oracle_unit.argtypes = [P, P, I, I, P, P, P, I, ctypes.c_int64, P, I, ctypes.c_double, I, I,
                                        I, I, P, P, P, P]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    return ctypes.c_void_p(a.ctypes.data)


def compress_unit_c(k_bits: np.ndarray, v_bits: np.ndarray, qbar: np.ndarray, qabs: np.ndarray, R: np.ndarray,
                    p: int, deltas: Sequence[int], base: float, budget: int, window: int, sinks: int = 0,
                    aggregate: str = "mean") -> Tuple[np.ndarray, np.ndarray, np.ndarray, np.ndarray]:
    """One unit: k_bits / v_bits are bf16 bit patterns [T, D] (int16 or uint16),
    statistics of its G query heads; ``sinks`` leading slots always kept and
    the group ``aggregate`` ("mean" or "max") as in the numpy oracle.
    Returns (scores, idx, new K rows, new V rows)."""
    if aggregate not in ("mean", "max"):
        raise ValueError("aggregate must be 'mean' or 'max'")
    lib = _load()
    k = np.ascontiguousarray(k_bits).view(np.uint16)
    v = np.ascontiguousarray(v_bits).view(np.uint16)
    T, D = k.shape
    qb = np.ascontiguousarray(qbar, dtype=np.float64)
    qa = np.ascontiguousarray(qabs, dtype=np.float64)
    r = np.ascontiguousarray(R, dtype=np.float64)
    d = np.ascontiguousarray(np.asarray(deltas, dtype=np.int32))
    scores = np.empty(T, dtype=np.float64)
    idx = np.empty(max(min(T, budget), 1), dtype=np.int32)
    ko, vo = np.empty_like(k), np.empty_like(v)
    kept = lib.tri_oracle_unit(_ptr(k), _ptr(v), T, D, _ptr(qb), _ptr(qa), _ptr(r), qb.shape[0], int(p), _ptr(d),
                               d.shape[0], float(base), int(budget), int(window), int(sinks),
                               1 if aggregate == "max" else 0, _ptr(scores), _ptr(idx), _ptr(ko), _ptr(vo))
    if kept < 0:
        raise ValueError("C oracle rejected its arguments")
    return scores, idx[:kept].astype(np.int64), ko.view(k_bits.dtype), vo.view(v_bits.dtype)
