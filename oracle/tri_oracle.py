"""Float64 CPU oracle of the TriAttention key-importance + eviction path.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The CUDA library
never calls it, and it shares no code, table or constant with that library.

It is written to be read against the pages, step by step, not to be fast:
every quantity is formed in float64 from its definition, one (sequence,
layer, KV head) unit at a time, with no blocking, folding or reordering
beyond what the definitions state.  bf16 inputs are widened to float64
exactly before any arithmetic.

Pages cited (title, then section):
  [Digest]   "TriAttention: Trigonometric KV Compression for Efficient Long
              Reasoning" - "Core Mechanism" (three stages and the data-flow
              figure), "Key Concepts" (Q/K Concentration, Trigonometric
              Distance Preference, Norm as Importance Signal)
  [Abstract] "TriAttention: Efficient Long Reasoning with Trigonometric KV
              Compression" - "English" (centres, trigonometric series,
              Q/K norms as an additional signal)
  [GeoTrick] "TriAttention: How a Geometric Trick Cuts LLM Memory Use by 10x
              Without Losing Accuracy" - "The Core Idea: Q/K Concentration in
              Pre-RoPE Space" (norm signal blended in, weighted by a measured
              concentration), "Solving the Memory Fragmentation Problem"
              (Forward-Packing Compaction)

Notation.  D = head dimension, n = D/2 bands.  Band i pairs dimensions
(i, i + n) (rotate-half) and is the complex number z_i = x_i + j x_{i+n}.
Rotary embedding turns band i by theta_i * position, theta_i = base^(-2i/D).
A unit is one (sequence s, layer l, KV head h); its G query heads are
h*G .. h*G + G - 1.  A cached slot t holds the post-rotation key k^_t.

Where the pages leave a step open, the reading taken is stated beside the
code that takes it:
  * concentration R of a head = sum_i |qbar_i| / sum_i E|q_i| (R = 1 when
    the samples are all zero);
  * future query positions are p + delta for the listed offsets, averaged
    uniformly;
  * per-head scores are averaged over the GQA group;
  * the recent window counts inside the budget; ties in score go to the
    lower slot; -0 and +0 are equal; a NaN score ranks below every number.
"""

from __future__ import annotations

import math
from typing import Dict, List, Sequence, Tuple

import numpy as np


# ----------------------------------------------------------------------------
# Bands and rotary frequencies
# ----------------------------------------------------------------------------

def rope_frequencies(D: int, base: float) -> np.ndarray:
    """theta_i = base^(-2i/D) for i = 0 .. D/2 - 1 (rotary embedding)."""
    i = np.arange(D // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / D)


def as_bands(x: np.ndarray) -> np.ndarray:
    """Complex band view z_i = x_i + j x_{i+n} of real vectors x[..., D]."""
    n = x.shape[-1] // 2
    return x[..., :n].astype(np.float64) + 1j * x[..., n:].astype(np.float64)


def from_bands(z: np.ndarray) -> np.ndarray:
    """Inverse of ``as_bands``: real vectors [..., D] from bands [..., D/2]."""
    return np.concatenate([z.real, z.imag], axis=-1)


# ----------------------------------------------------------------------------
# Stage 1: centres and concentration (one-time calibration)
# [Digest] "Core Mechanism" data-flow figure, centre calibration; "Key
# Concepts", Q/K Concentration (the centre is the mean pre-rotation query);
# [GeoTrick] "The Core Idea" (a measured concentration per head).
# ----------------------------------------------------------------------------

def calibrate(q_samples: np.ndarray) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Reduce pre-rotation query samples [N, ..., D] to head statistics.

    Returns (qbar [..., D], qabs [..., D/2], R [...]):
      qbar : the centre, the mean sample (as real dims, bands (i, i+n));
      qabs : A_i = E|q_i|, the mean band magnitude;
      R    : sum_i |qbar_i| / sum_i A_i, in [0, 1] (1 if sum_i A_i = 0).
    """
    z = as_bands(np.asarray(q_samples, dtype=np.float64))
    zbar = z.mean(axis=0)
    A = np.abs(z).mean(axis=0)
    num = np.abs(zbar).sum(axis=-1)
    den = A.sum(axis=-1)
    with np.errstate(invalid="ignore", divide="ignore"):
        R = np.where(den > 0.0, num / np.where(den > 0.0, den, 1.0), 1.0)
    return from_bands(zbar), A, R


# ----------------------------------------------------------------------------
# Stage 2: the score
# [Digest] "Key Concepts", Trigonometric Distance Preference (the centre dot
# product after rotation is a cosine series in the distance); [Abstract]
# "English"; [GeoTrick] "The Core Idea" (norm signal weighted by measured
# concentration).
# ----------------------------------------------------------------------------

def future_phase_mean(p: int, deltas: Sequence[int], D: int, base: float) -> np.ndarray:
    """m_i = (1/|deltas|) sum_delta exp(j theta_i (p + delta)), i < D/2."""
    theta = rope_frequencies(D, base)
    acc = np.zeros(D // 2, dtype=np.complex128)
    for d in deltas:
        acc += np.exp(1j * theta * float(int(p) + int(d)))
    return acc / len(deltas)


def effective_query(qbar_g: np.ndarray, p: int, deltas: Sequence[int], base: float) -> np.ndarray:
    """Bands c_i = qbar_i * m_i of one query head's effective query."""
    D = qbar_g.shape[-1]
    return as_bands(qbar_g) * future_phase_mean(p, deltas, D, base)


def head_score(keys: np.ndarray, qbar_g: np.ndarray, qabs_g: np.ndarray, R_g: float,
               p: int, deltas: Sequence[int], base: float) -> np.ndarray:
    """Score of every cached post-rotation key [T, D] for one query head.

      trig(t) = sum_i Re( c_i * conj(k^_{t,i}) )
              = mean_delta sum_i |qbar_i||k_i| cos(theta_i (p+delta-t) + phi_i)
      norm(t) = sum_i (A_i - |qbar_i|) |k^_{t,i}|
      s(t)    = trig(t) + (1 - R) norm(t)
    """
    khat = as_bands(np.asarray(keys, dtype=np.float64))
    c = effective_query(np.asarray(qbar_g, dtype=np.float64), p, deltas, base)
    trig = (c[None, :] * np.conj(khat)).real.sum(axis=-1)
    weight = np.asarray(qabs_g, dtype=np.float64) - np.abs(as_bands(np.asarray(qbar_g, dtype=np.float64)))
    norm = (weight[None, :] * np.abs(khat)).sum(axis=-1)
    return trig + (1.0 - float(R_g)) * norm


def unit_scores(keys: np.ndarray, qbar: np.ndarray, qabs: np.ndarray, R: np.ndarray,
                p: int, deltas: Sequence[int], base: float, aggregate: str = "mean") -> np.ndarray:
    """The G query heads' ``head_score`` combined per key (qbar [G, D], ...):
    their mean (the method's reading), or their maximum (a variant)."""
    G = qbar.shape[0]
    per_head = [head_score(keys, qbar[g], qabs[g], R[g], p, deltas, base) for g in range(G)]
    if aggregate == "mean":
        total = np.zeros(keys.shape[0], dtype=np.float64)
        for sg in per_head:
            total += sg
        return total / G
    if aggregate == "max":
        best = per_head[0].copy()
        for sg in per_head[1:]:
            best = np.maximum(best, sg)
        return best
    raise ValueError("aggregate must be 'mean' or 'max'")


def group_query(qbar: np.ndarray, qabs: np.ndarray, R: np.ndarray, p: int,
                deltas: Sequence[int], base: float) -> Tuple[np.ndarray, np.ndarray]:
    """The group's score as one real dot product plus one weighted band norm.

    The trig term is linear in the effective query and the norm term linear
    in its weights, so the mean over the G heads equals
      s(t) = sum_d qeff_d K_{t,d} + sum_i w_i |k^_{t,i}|
    with qeff = the real dims of mean_g c_g and w_i = mean_g (1 - R_g)(A_{g,i}
    - |qbar_{g,i}|).  Returns (qeff [D], w [D/2]).
    """
    G = qbar.shape[0]
    c = np.zeros(qbar.shape[-1] // 2, dtype=np.complex128)
    w = np.zeros(qbar.shape[-1] // 2, dtype=np.float64)
    for g in range(G):
        c += effective_query(qbar[g], p, deltas, base)
        w += (1.0 - float(R[g])) * (np.asarray(qabs[g], np.float64) - np.abs(as_bands(np.asarray(qbar[g], np.float64))))
    return from_bands(c / G), w / G


# ----------------------------------------------------------------------------
# Stage 3: keep the top-scoring keys, always with a recent window
# [Digest] "Core Mechanism" (keep only the top-scoring subset; data-flow
# figure, top-K selection).
# ----------------------------------------------------------------------------

def select(scores: Sequence[float], length: int, budget: int, window: int, sinks: int = 0) -> np.ndarray:
    """Ascending slot indices kept for one unit.

    If length <= budget every slot is kept.  Otherwise the first ``sinks``
    slots and the last ``window`` slots are kept, plus the
    (budget - window - sinks) best of the slots between them, ordered by
    score (higher first) and then by slot (lower first).  Sinks are the
    optional attention-sink variant; the method itself keeps none.
    """
    if not (budget >= 1 and 0 <= window and 0 <= sinks and window + sinks <= budget):
        raise ValueError("need budget >= 1 and 0 <= window, sinks with window + sinks <= budget")
    if length <= budget:
        return np.arange(length, dtype=np.int64)
    cand = length - window
    take = budget - window - sinks

    def rank_key(t: int):
        v = float(scores[t])
        if math.isnan(v):
            v = -math.inf
        return (-v, t)

    best = sorted(range(sinks, cand), key=rank_key)[:take]
    kept = list(range(sinks)) + sorted(best) + list(range(cand, length))
    return np.asarray(kept, dtype=np.int64)


# ----------------------------------------------------------------------------
# Stage 4: Forward-Packing Compaction
# [GeoTrick] "Solving the Memory Fragmentation Problem" (survivors move
# forward, tail blocks empty out and return to the paged allocator).
# ----------------------------------------------------------------------------

def compact_rows(rows: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """New rows of one unit: row j <- old row idx[j] for j < len(idx).

    Rows from len(idx) on keep their old contents.
    """
    out = rows.copy()
    for j, src in enumerate(idx):
        out[j] = rows[int(src)]
    return out


def freed_blocks(table_row: Sequence[int], old_len: int, kept: int, block_size: int) -> List[int]:
    """Blocks of a sequence that hold no row once ``kept`` rows remain."""
    keep = -(-kept // block_size)
    had = -(-old_len // block_size)
    return [int(b) for b in table_row[keep:had]]


# ----------------------------------------------------------------------------
# Paged cache plumbing (layout [L][num_blocks][Hkv][block_size][D])
# [GeoTrick] "Solving the Memory Fragmentation Problem" and "Why Existing KV
# Cache Compression Breaks in Production": a sequence's cache is a chain of
# fixed-size pages; its block table names the page of every run of
# block_size slots, so slot t sits in row t mod block_size of page
# table[t div block_size].
# ----------------------------------------------------------------------------

def unit_rows(pool: np.ndarray, table_row: Sequence[int], length: int, l: int, h: int) -> np.ndarray:
    """The ``length`` cached rows of (layer l, KV head h) of one sequence:
    row t is pool[l, table_row[t // bs], h, t % bs]."""
    bs = pool.shape[3]
    out = np.empty((length, pool.shape[4]), dtype=pool.dtype)
    for t in range(length):
        out[t] = pool[l, int(table_row[t // bs]), h, t % bs]
    return out


def store_unit_rows(pool: np.ndarray, table_row: Sequence[int], rows: np.ndarray, l: int, h: int) -> None:
    """Write rows[t] to pool[l, table_row[t // bs], h, t % bs] for every t."""
    bs = pool.shape[3]
    for t in range(rows.shape[0]):
        pool[l, int(table_row[t // bs]), h, t % bs] = rows[t]


def compress_unit(keys_f64: np.ndarray, k_rows: np.ndarray, v_rows: np.ndarray,
                  qbar: np.ndarray, qabs: np.ndarray, R: np.ndarray, p: int,
                  deltas: Sequence[int], base: float, budget: int, window: int,
                  sinks: int = 0, aggregate: str = "mean"):
    """Score, select and compact one unit.

    ``keys_f64`` are the unit's keys widened to float64; ``k_rows`` /
    ``v_rows`` are the same rows in any representation (e.g. bf16 bit
    patterns) and are moved, never computed on.  Returns (scores, idx,
    new_k_rows, new_v_rows).
    """
    length = keys_f64.shape[0]
    s = unit_scores(keys_f64, qbar, qabs, R, p, deltas, base, aggregate)
    idx = select(s, length, budget, window, sinks)
    return s, idx, compact_rows(k_rows, idx), compact_rows(v_rows, idx)


# ----------------------------------------------------------------------------
# Variant: scores from the centres alone, as a table over the distance
# [Digest] "Core Mechanism" (the trigonometric series of the distance,
# evaluated as lookups indexed by relative position) and "Key Concepts",
# Trigonometric Distance Preference (after rotation the centres' dot product
# depends on the query-key distance only).
#
# Reading: the table is the trigonometric term with the key's own rotated
# band replaced by its head's rotated key centre kbar (calibrated from
# pre-rotation keys like the query centre).  The norm term of the centres,
# (1 - R) sum_i (A_i - |qbar_i|) |kbar_i|, is the same for every key of a unit
# and cannot change its ranking, so the table leaves it out.  A key's score
# is f(p - pos_t), pos_t the position the key was cached at; after a
# compaction slots no longer equal positions, so positions travel with the
# rows.
# ----------------------------------------------------------------------------

def distance_series(qbar_g: np.ndarray, kbar: np.ndarray, deltas: Sequence[int], base: float,
                    max_dist: int) -> np.ndarray:
    """f_g(dist) for dist = 0 .. max_dist, one query head g against a key
    centre:
      logit(p + delta, t) = sum_i Re( qbar_i e^{j theta_i (p+delta)} conj(kbar_i e^{j theta_i t}) )
                          = sum_i Re( qbar_i conj(kbar_i) e^{j theta_i (dist + delta)} ),  dist = p - t,
    averaged uniformly over the offsets delta."""
    qb = as_bands(np.asarray(qbar_g, dtype=np.float64))
    kb = as_bands(np.asarray(kbar, dtype=np.float64))
    theta = rope_frequencies(qbar_g.shape[-1], base)
    a = qb * np.conj(kb)
    dist = np.arange(int(max_dist) + 1, dtype=np.float64)
    out = np.zeros(dist.shape[0], dtype=np.float64)
    for d in deltas:
        phase = np.exp(1j * theta[None, :] * (dist[:, None] + float(int(d))))
        out += (a[None, :] * phase).real.sum(axis=-1)
    return out / len(deltas)


def distance_table(qbar: np.ndarray, kbar: np.ndarray, deltas: Sequence[int], base: float,
                   max_dist: int, aggregate: str = "mean") -> np.ndarray:
    """The table of one (layer, KV head): its G query heads' series
    (qbar [G, D], kbar [D]) combined per distance by mean (the method's
    reading) or max (the variant)."""
    G = qbar.shape[0]
    per_head = [distance_series(qbar[g], kbar, deltas, base, max_dist) for g in range(G)]
    if aggregate == "mean":
        total = np.zeros_like(per_head[0])
        for f in per_head:
            total += f
        return total / G
    if aggregate == "max":
        best = per_head[0].copy()
        for f in per_head[1:]:
            best = np.maximum(best, f)
        return best
    raise ValueError("aggregate must be 'mean' or 'max'")


def distance_scores(table: np.ndarray, p: int, positions: Sequence[int]) -> np.ndarray:
    """Score of keys cached at ``positions`` for the query at p: f(p - pos)."""
    out = np.empty(len(positions), dtype=np.float64)
    for t, pos in enumerate(positions):
        dist = int(p) - int(pos)
        if dist < 0 or dist >= table.shape[0]:
            raise ValueError(f"distance {dist} outside the table")
        out[t] = table[dist]
    return out


def compress_step_distance(k_bits: np.ndarray, v_bits: np.ndarray, block_table: np.ndarray,
                           seq_len: Sequence[int], cur_pos: Sequence[int], positions: np.ndarray,
                           tables: np.ndarray, budget: int, window: int, sinks: int = 0,
                           trigger: int = 0) -> Dict:
    """``compress_step`` with distance-table scores.  positions [S][L][Hkv][>= len]
    holds each slot's cached position; tables [L][Hkv][max_dist + 1].  The
    returned positions are compacted with the rows."""
    L, _, Hkv, bs, _ = k_bits.shape
    trigger = max(int(trigger), int(budget))
    new_k, new_v, new_pos = k_bits.copy(), v_bits.copy(), positions.copy()
    new_len, freed = [], []
    scores, kept_idx = {}, {}
    for s, length in enumerate(seq_len):
        length = int(length)
        table_row = block_table[s]
        if length <= trigger:
            new_len.append(length)
            continue
        for l in range(L):
            for h in range(Hkv):
                sc = distance_scores(tables[l, h], int(cur_pos[s]), positions[s, l, h, :length])
                idx = select(sc, length, budget, window, sinks)
                kr = unit_rows(k_bits, table_row, length, l, h)
                vr = unit_rows(v_bits, table_row, length, l, h)
                store_unit_rows(new_k, table_row, compact_rows(kr, idx), l, h)
                store_unit_rows(new_v, table_row, compact_rows(vr, idx), l, h)
                new_pos[s, l, h, :length] = compact_rows(positions[s, l, h, :length], idx)
                scores[(s, l, h)] = sc
                kept_idx[(s, l, h)] = idx
        new_len.append(budget)
        freed += freed_blocks(table_row, length, budget, bs)
    return {"k_pool": new_k, "v_pool": new_v, "seq_len": new_len, "freed_ids": freed,
            "positions": new_pos, "scores": scores, "idx": kept_idx}


def compress_step(k_vals: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray,
                  block_table: np.ndarray, seq_len: Sequence[int], cur_pos: Sequence[int],
                  qbar: np.ndarray, qabs: np.ndarray, R: np.ndarray, G: int,
                  deltas: Sequence[int], base: float, budget: int, window: int,
                  sinks: int = 0, trigger: int = 0, aggregate: str = "mean") -> Dict:
    """One compression step over every unit of every sequence.

    k_vals : float64 [L][NB][Hkv][bs][D], the cached keys' values
    k_bits, v_bits : the pools in any representation; copies are returned
    qbar [L][Hq][D], qabs [L][Hq][D/2], R [L][Hq] : head statistics

    A sequence is compressed only when its length exceeds ``trigger`` (which
    defaults to the budget and is never below it); shorter sequences are left
    as they are.

    Returns a dict with the new pools, new lengths, the freed block ids (in
    sequence order, each sequence's blocks in table order), and per unit
    (s, l, h) its scores and kept indices.
    """
    L, _, Hkv, bs, _ = k_vals.shape
    trigger = max(int(trigger), int(budget))
    new_k, new_v = k_bits.copy(), v_bits.copy()
    new_len, freed = [], []
    scores, kept_idx = {}, {}
    for s, length in enumerate(seq_len):
        length = int(length)
        table_row = block_table[s]
        if length <= trigger:
            for l in range(L):
                for h in range(Hkv):
                    kept_idx[(s, l, h)] = np.arange(length, dtype=np.int64)
            new_len.append(length)
            continue
        kept = min(length, budget)
        for l in range(L):
            for h in range(Hkv):
                g0 = h * G
                keys = unit_rows(k_vals, table_row, length, l, h)
                sc = unit_scores(keys, qbar[l, g0:g0 + G], qabs[l, g0:g0 + G], R[l, g0:g0 + G],
                                 int(cur_pos[s]), deltas, base, aggregate)
                idx = select(sc, length, budget, window, sinks)
                assert idx.shape[0] == kept
                kr = unit_rows(k_bits, table_row, length, l, h)
                vr = unit_rows(v_bits, table_row, length, l, h)
                store_unit_rows(new_k, table_row, compact_rows(kr, idx), l, h)
                store_unit_rows(new_v, table_row, compact_rows(vr, idx), l, h)
                scores[(s, l, h)] = sc
                kept_idx[(s, l, h)] = idx
        new_len.append(kept)
        freed += freed_blocks(table_row, length, kept, bs)
    return {"k_pool": new_k, "v_pool": new_v, "seq_len": new_len, "freed_ids": freed,
            "scores": scores, "idx": kept_idx}
