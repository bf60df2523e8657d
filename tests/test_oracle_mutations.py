"""Planted mistakes in the oracle must each fail at least one pin (CPU only).

Each mutation replaces one oracle function with a plausible wrong variant
(a flipped sign, the other band pairing, a dropped factor, a wrong index...)
and runs the pins of ``test_oracle_pins``.  The mutation is caught if any pin
raises.  Nothing here touches a GPU.
"""

import inspect
import math

import numpy as np
import pytest

import oracle
from oracle import tri_oracle as T
import tests.test_oracle_pins as pins


def _all_pins():
    out = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        params = inspect.signature(fn).parameters
        if name == "test_trig_term_is_mean_attention_logit_under_hf_rotary":
            out += [(name, lambda fn=fn, a=a: fn(*a)) for a in [(8, 1e4, 37), (128, 5e5, 32768)]]
        elif name == "test_select_brute_force_dominance":
            out += [(name, lambda fn=fn, s=s: fn(s)) for s in range(30)]
        elif name == "test_select_with_sinks_brute_force":
            out += [(name, lambda fn=fn, s=s: fn(s)) for s in range(20)]
        elif len(params) == 0:
            out.append((name, fn))
    return out


def _caught(monkeypatch, attr, replacement):
    monkeypatch.setattr(T, attr, replacement)
    monkeypatch.setattr(oracle, attr, replacement, raising=False)
    failed = []
    for name, fn in _all_pins():
        try:
            fn()
        except (Exception, pytest.fail.Exception):   # a pin's pytest.raises failing counts
            failed.append(name)
    return failed


def _phase_sign_flipped(p, deltas, D, base):
    theta = T.rope_frequencies(D, base)
    return np.mean([np.exp(-1j * theta * (p + d)) for d in deltas], axis=0)


def _phase_summed(p, deltas, D, base):
    theta = T.rope_frequencies(D, base)
    return np.sum([np.exp(1j * theta * (p + d)) for d in deltas], axis=0)


def _theta_half_exponent(D, base):
    return np.power(float(base), -1.0 * np.arange(D // 2) / D)


def _interleaved_bands(x):
    return x[..., 0::2].astype(np.float64) + 1j * x[..., 1::2].astype(np.float64)


def _head_score_no_concentration_weight(keys, qbar_g, qabs_g, R_g, p, deltas, base):
    kh = T.as_bands(np.asarray(keys, np.float64))
    c = T.effective_query(qbar_g, p, deltas, base)
    trig = (c[None] * np.conj(kh)).real.sum(-1)
    norm = ((qabs_g - np.abs(T.as_bands(qbar_g)))[None] * np.abs(kh)).sum(-1)
    return trig + norm


def _head_score_norm_weight_A(keys, qbar_g, qabs_g, R_g, p, deltas, base):
    kh = T.as_bands(np.asarray(keys, np.float64))
    c = T.effective_query(qbar_g, p, deltas, base)
    trig = (c[None] * np.conj(kh)).real.sum(-1)
    norm = (np.asarray(qabs_g)[None] * np.abs(kh)).sum(-1)
    return trig + (1 - R_g) * norm


def _head_score_conj_swapped(keys, qbar_g, qabs_g, R_g, p, deltas, base):
    kh = T.as_bands(np.asarray(keys, np.float64))
    c = T.effective_query(qbar_g, p, deltas, base)
    trig = (c[None] * kh).real.sum(-1)            # conjugate on neither operand
    norm = ((qabs_g - np.abs(T.as_bands(qbar_g)))[None] * np.abs(kh)).sum(-1)
    return trig + (1 - R_g) * norm


def _head_score_squared_norm(keys, qbar_g, qabs_g, R_g, p, deltas, base):
    kh = T.as_bands(np.asarray(keys, np.float64))
    c = T.effective_query(qbar_g, p, deltas, base)
    trig = (c[None] * np.conj(kh)).real.sum(-1)
    norm = ((qabs_g - np.abs(T.as_bands(qbar_g)))[None] * np.abs(kh) ** 2).sum(-1)
    return trig + (1 - R_g) * norm


def _unit_scores_sum(keys, qbar, qabs, R, p, deltas, base, aggregate="mean"):
    return sum(T.head_score(keys, qbar[g], qabs[g], R[g], p, deltas, base) for g in range(qbar.shape[0]))


def _select_ties_high(scores, length, budget, window, sinks=0):
    if length <= budget:
        return np.arange(length)
    cand, take = length - window, budget - window
    key = lambda t: (-(-math.inf if math.isnan(scores[t]) else scores[t]), -t)  # noqa: E731
    return np.asarray(sorted(sorted(range(cand), key=key)[:take]) + list(range(cand, length)))


def _select_window_outside(scores, length, budget, window, sinks=0):
    if length <= budget:
        return np.arange(length)
    cand = length - window
    key = lambda t: (-(-math.inf if math.isnan(scores[t]) else scores[t]), t)  # noqa: E731
    best = sorted(range(cand), key=key)[:min(budget, cand)]
    return np.asarray(sorted(best) + list(range(cand, length)))


def _select_nan_high(scores, length, budget, window, sinks=0):
    if length <= budget:
        return np.arange(length)
    cand, take = length - window, budget - window
    key = lambda t: (-(math.inf if math.isnan(scores[t]) else scores[t]), t)  # noqa: E731
    return np.asarray(sorted(sorted(range(cand), key=key)[:take]) + list(range(cand, length)))


def _select_sinks_outside(scores, length, budget, window, sinks=0):
    # sinks added on top of the budget instead of inside it
    if length <= budget:
        return np.arange(length)
    cand, take = length - window, budget - window
    key = lambda t: (-(-math.inf if math.isnan(scores[t]) else scores[t]), t)  # noqa: E731
    best = sorted(range(sinks, cand), key=key)[:take]
    return np.asarray(list(range(sinks)) + sorted(best) + list(range(cand, length)))


def _unit_scores_max_is_mean(keys, qbar, qabs, R, p, deltas, base, aggregate="mean"):
    G = qbar.shape[0]
    return sum(T.head_score(keys, qbar[g], qabs[g], R[g], p, deltas, base) for g in range(G)) / G


_compress_step = T.compress_step


def _compress_step_trigger_ignored(*args, **kw):
    kw["trigger"] = 0
    return _compress_step(*args, **kw)


def _distance_series_no_conj(qbar_g, kbar, deltas, base, max_dist):
    qb, kb = T.as_bands(np.asarray(qbar_g, np.float64)), T.as_bands(np.asarray(kbar, np.float64))
    theta = T.rope_frequencies(qbar_g.shape[-1], base)
    dist = np.arange(max_dist + 1, dtype=np.float64)
    out = sum(((qb * kb)[None] * np.exp(1j * theta[None] * (dist[:, None] + d))).real.sum(-1) for d in deltas)
    return out / len(deltas)


def _distance_series_reversed(qbar_g, kbar, deltas, base, max_dist):
    qb, kb = T.as_bands(np.asarray(qbar_g, np.float64)), T.as_bands(np.asarray(kbar, np.float64))
    theta = T.rope_frequencies(qbar_g.shape[-1], base)
    dist = np.arange(max_dist + 1, dtype=np.float64)
    out = sum(((qb * np.conj(kb))[None] * np.exp(1j * theta[None] * (-dist[:, None] + d))).real.sum(-1)
              for d in deltas)
    return out / len(deltas)


def _distance_scores_slot_not_position(table, p, positions):
    return np.array([table[int(p) - t] for t in range(len(positions))], dtype=np.float64)


def _compact_off_by_one(rows, idx):
    out = rows.copy()
    for j, src in enumerate(idx):
        out[j] = rows[min(int(src) + 1, rows.shape[0] - 1)]
    return out


def _freed_floor(table_row, old_len, kept, bs):
    return [int(b) for b in table_row[kept // bs:-(-old_len // bs)]]


def _calibrate_vector_norms(q):
    q = np.asarray(q, np.float64)
    z = T.as_bands(q)
    zbar = z.mean(0)
    A = np.abs(z).mean(0)
    R = np.linalg.norm(q.mean(0), axis=-1) / np.linalg.norm(q, axis=-1).mean(0)
    return T.from_bands(zbar), A, R


def _calibrate_rms(q):
    z = T.as_bands(np.asarray(q, np.float64))
    zbar = z.mean(0)
    A = np.sqrt((np.abs(z) ** 2).mean(0))
    num, den = np.abs(zbar).sum(-1), A.sum(-1)
    return T.from_bands(zbar), A, np.where(den > 0, num / np.where(den > 0, den, 1), 1.0)


def _unit_rows_table_ignored(pool, table_row, length, l, h):
    bs = pool.shape[3]
    return np.stack([pool[l, t // bs, h, t % bs] for t in range(length)]) if length else \
        np.empty((0, pool.shape[4]), pool.dtype)


def _unit_rows_div_mod_swapped(pool, table_row, length, l, h):
    bs = pool.shape[3]
    out = np.empty((length, pool.shape[4]), dtype=pool.dtype)
    for t in range(length):
        out[t] = pool[l, int(table_row[t % bs]), h, t // bs]
    return out


def _store_unit_rows_div_mod_swapped(pool, table_row, rows, l, h):
    bs = pool.shape[3]
    for t in range(rows.shape[0]):
        pool[l, int(table_row[t % bs]), h, t // bs] = rows[t]


MUTATIONS = [
    ("future_phase_mean", _phase_sign_flipped),
    ("future_phase_mean", _phase_summed),
    ("rope_frequencies", _theta_half_exponent),
    ("as_bands", _interleaved_bands),
    ("head_score", _head_score_no_concentration_weight),
    ("head_score", _head_score_norm_weight_A),
    ("head_score", _head_score_conj_swapped),
    ("head_score", _head_score_squared_norm),
    ("unit_scores", _unit_scores_sum),
    ("select", _select_ties_high),
    ("select", _select_window_outside),
    ("select", _select_nan_high),
    ("select", _select_sinks_outside),
    ("unit_scores", _unit_scores_max_is_mean),
    ("compress_step", _compress_step_trigger_ignored),
    ("distance_series", _distance_series_no_conj),
    ("distance_series", _distance_series_reversed),
    ("distance_scores", _distance_scores_slot_not_position),
    ("compact_rows", _compact_off_by_one),
    ("freed_blocks", _freed_floor),
    ("calibrate", _calibrate_vector_norms),
    ("calibrate", _calibrate_rms),
    ("unit_rows", _unit_rows_table_ignored),
    ("unit_rows", _unit_rows_div_mod_swapped),
    ("store_unit_rows", _store_unit_rows_div_mod_swapped),
]


def test_unmutated_oracle_passes_every_pin():
    for name, fn in _all_pins():
        fn()


@pytest.mark.parametrize("attr,mutant", MUTATIONS, ids=[f"{a}:{m.__name__}" for a, m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, attr, mutant):
    failed = _caught(monkeypatch, attr, mutant)
    assert failed, f"mutation {mutant.__name__} of {attr} passed every pin"
