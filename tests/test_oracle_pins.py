"""Pins of the float64 oracle to facts outside itself (CPU only).

Each test ties one part of the oracle to something it does not compute
itself: the HuggingFace rotary embedding, explicit rotation matrices, closed
forms, textbook distributions, numpy / library routines, brute force on tiny
inputs, or figures printed on the pages.  A dropped term, a wrong sign,
pairing or index, or a transposed operand in the oracle fails at least one.

Pages cited (title, then section):
  [Digest]   "TriAttention: Trigonometric KV Compression for Efficient Long Reasoning"
  [GeoTrick] "TriAttention: How a Geometric Trick Cuts LLM Memory Use by 10x
              Without Losing Accuracy"
  [Abstract] "TriAttention: Efficient Long Reasoning with Trigonometric KV Compression"
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workload import rope_rotate_half, noise_scale_for_target_concentration

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rot2(angle):
    c, s = math.cos(angle), math.sin(angle)
    return np.array([[c, -s], [s, c]])


def _rotate_explicit(x, pos, base):
    """Rotary embedding with an explicit 2x2 matrix per band (pairs i, i+D/2)."""
    D = x.shape[-1]
    n = D // 2
    out = np.empty(D)
    for i in range(n):
        theta = float(base) ** (-2.0 * i / D)
        v = _rot2(theta * pos) @ np.array([x[i], x[i + n]])
        out[i], out[i + n] = v
    return out


# ---------------------------------------------------------------------------
# Rotary convention and the trigonometric term
# ---------------------------------------------------------------------------

def test_theta_matches_huggingface_inv_freq():
    """theta_i = base^(-2i/D) is the HF Llama rotary frequency table."""
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding
    for base in (1e4, 5e5, 1e6):
        cfg = LlamaConfig(hidden_size=256, num_attention_heads=2, head_dim=128, rope_theta=base)
        hf = LlamaRotaryEmbedding(cfg).inv_freq.double().numpy()
        np.testing.assert_allclose(oracle.rope_frequencies(128, base), hf, rtol=2e-7, atol=0)


@pytest.mark.parametrize("D,base,p", [(8, 1e4, 37), (128, 1e4, 4096), (128, 5e5, 32768)])
def test_trig_term_is_mean_attention_logit_under_hf_rotary(D, base, p):
    """With R = 1 the score is the mean over future offsets of the HF-rotated
    centre dotted with the HF-rotated key ([Digest] "Key Concepts",
    Trigonometric Distance Preference)."""
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    rng = np.random.default_rng(1)
    T = 40
    qbar = rng.normal(size=D)
    k_pre = rng.normal(size=(T, D))
    pos_k = rng.integers(0, p, size=T)
    deltas = [1, 2, 4, 8, 16, 1000]
    theta = oracle.rope_frequencies(D, base)

    def cos_sin(pos):
        f = np.outer(np.asarray(pos, dtype=np.float64), theta)
        emb = np.concatenate([f, f], axis=-1)
        return torch.from_numpy(np.cos(emb))[None], torch.from_numpy(np.sin(emb))[None]

    kt = torch.from_numpy(k_pre)[None, None]           # [1, 1, T, D]
    cos_k, sin_k = cos_sin(pos_k)
    _, k_post = apply_rotary_pos_emb(kt, kt, cos_k, sin_k)
    k_post = k_post[0, 0].numpy()

    logits = np.zeros(T)
    for d in deltas:
        qt = torch.from_numpy(qbar)[None, None, None]   # [1, 1, 1, D]
        cq, sq = cos_sin([p + d])
        q_post, _ = apply_rotary_pos_emb(qt, qt, cq, sq)
        logits += k_post @ q_post[0, 0, 0].numpy()
    logits /= len(deltas)

    got = oracle.head_score(k_post, qbar, np.abs(oracle.as_bands(qbar)), 1.0, p, deltas, base)
    np.testing.assert_allclose(got, logits, rtol=1e-10, atol=1e-10 * np.abs(logits).max())


def test_trig_term_explicit_rotation_matrices_large_positions():
    """Same identity with hand-built rotation matrices at positions ~1.3e5."""
    rng = np.random.default_rng(2)
    D, base, p = 8, 1e6, 131072
    qbar = rng.normal(size=D)
    deltas = [1, 64, 4096, 8192]
    pos = [0, 5, 70000, 131071]
    k_pre = rng.normal(size=(len(pos), D))
    k_post = np.stack([_rotate_explicit(k_pre[t], pos[t], base) for t in range(len(pos))])
    want = np.array([np.mean([_rotate_explicit(qbar, p + d, base) @ k_post[t] for d in deltas])
                     for t in range(len(pos))])
    got = oracle.head_score(k_post, qbar, np.abs(oracle.as_bands(qbar)), 1.0, p, deltas, base)
    np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-9)


def test_d2_closed_form():
    """D = 2: theta_0 = 1 for every base, so the score is
    |qbar||k| mean_delta cos(p + delta - t + arg qbar - arg k_pre)."""
    cases = [((1.0, 0.0), (1.0, 0.0), 0, 0, [1]),
             ((0.3, -1.2), (2.0, 0.5), 17, 40, [1, 2, 4]),
             ((-0.7, 0.1), (0.0, 1.0), 1000, 1003, [3, 9, 27, 81])]
    for q, k, t, p, deltas in cases:
        q, k = np.array(q), np.array(k)
        k_post = np.array([k[0] * math.cos(t) - k[1] * math.sin(t), k[1] * math.cos(t) + k[0] * math.sin(t)])
        phi = math.atan2(q[1], q[0]) - math.atan2(k[1], k[0])
        want = math.hypot(*q) * math.hypot(*k) * np.mean([math.cos(p + d - t + phi) for d in deltas])
        got = oracle.head_score(k_post[None], q, np.array([math.hypot(*q)]), 1.0, p, deltas, 12345.0)
        assert abs(got[0] - want) < 1e-12
    # The simplest case evaluates to cos(1).
    got = oracle.head_score(np.array([[1.0, 0.0]]), np.array([1.0, 0.0]), np.array([1.0]), 1.0, 0, [1], 1e4)
    assert abs(got[0] - math.cos(1.0)) < 1e-15


def test_trig_series_polar_form():
    """The trig term equals sum_i |qbar_i||k_i| mean_delta cos(theta_i (p+delta-t)
    + phi_i) written with magnitudes and angles ([Abstract] "English")."""
    rng = np.random.default_rng(3)
    D, base, p = 128, 5e5, 32768
    deltas = [1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096]
    qbar = rng.normal(size=D)
    T = 16
    pos = rng.integers(0, p, size=T)
    k_pre = rng.normal(size=(T, D))
    k_post = np.stack([_rotate_explicit(k_pre[t], pos[t], base) for t in range(T)])
    n = D // 2
    qz = qbar[:n] + 1j * qbar[n:]
    want = np.zeros(T)
    for t in range(T):
        kz = k_pre[t, :n] + 1j * k_pre[t, n:]
        for i in range(n):
            th = base ** (-2.0 * i / D)
            phi = np.angle(qz[i]) - np.angle(kz[i])
            want[t] += abs(qz[i]) * abs(kz[i]) * np.mean([math.cos(th * (p + d - pos[t]) + phi) for d in deltas])
    got = oracle.head_score(k_post, qbar, np.abs(qz), 1.0, p, deltas, base)
    np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-9 * np.abs(want).max())


# ---------------------------------------------------------------------------
# The norm term and its concentration weight
# ---------------------------------------------------------------------------

def _single_band_keys(rng, T, D):
    n = D // 2
    k = np.zeros((T, D))
    band = rng.integers(0, n, size=T)
    for t in range(T):
        k[t, band[t]] = rng.normal()
        k[t, band[t] + n] = rng.normal()
    return k, band


def test_norm_term_single_band_keys():
    """A key with one non-zero band i*: score - trig = (1 - R)(A_i* - |qbar_i*|)||k||
    ([GeoTrick] "The Core Idea", norm signal weighted by concentration)."""
    rng = np.random.default_rng(4)
    D, p, base, R = 16, 100, 1e4, 0.3
    deltas = [1, 2, 4]
    k, band = _single_band_keys(rng, 12, D)
    qbar = rng.normal(size=D)
    qmag = np.abs(oracle.as_bands(qbar))
    A = qmag + rng.uniform(0.1, 2.0, size=D // 2)
    full = oracle.head_score(k, qbar, A, R, p, deltas, base)
    trig = oracle.head_score(k, qbar, qmag, 1.0, p, deltas, base)
    want = (1 - R) * (A[band] - qmag[band]) * np.linalg.norm(k, axis=1)
    np.testing.assert_allclose(full - trig, want, rtol=1e-12, atol=1e-13)


def test_zero_centre_ranks_by_norm():
    """qbar = 0 (R = 0): the trig term vanishes and a constant A gives a*||k||
    for single-band keys."""
    rng = np.random.default_rng(5)
    D = 32
    k, _ = _single_band_keys(rng, 20, D)
    got = oracle.head_score(k, np.zeros(D), np.full(D // 2, 0.7), 0.0, 500, [1, 3], 1e4)
    np.testing.assert_allclose(got, 0.7 * np.linalg.norm(k, axis=1), rtol=1e-13)


def test_full_concentration_drops_norm_term():
    """R = 1 or A = |qbar| leaves only the trig term."""
    rng = np.random.default_rng(6)
    D = 16
    k = rng.normal(size=(10, D))
    qbar = rng.normal(size=D)
    qmag = np.abs(oracle.as_bands(qbar))
    A = qmag + 1.0
    a = oracle.head_score(k, qbar, A, 1.0, 7, [1], 1e4)
    b = oracle.head_score(k, qbar, qmag, 0.2, 7, [1], 1e4)
    c = oracle.head_score(k, qbar, qmag, 1.0, 7, [1], 1e4)
    np.testing.assert_allclose(a, c, rtol=0, atol=1e-13)
    np.testing.assert_allclose(b, c, rtol=0, atol=1e-13)


def test_norm_term_is_rotation_invariant():
    """Band magnitudes do not change under rotary embedding: with qbar = 0 the
    score of a key is the same at every position."""
    rng = np.random.default_rng(7)
    D, base = 128, 1e6
    k_pre = rng.normal(size=D)
    A = rng.uniform(0.5, 1.5, size=D // 2)
    posts = np.stack([_rotate_explicit(k_pre, t, base) for t in (0, 1, 999, 123456)])
    s = oracle.head_score(posts, np.zeros(D), A, 0.0, 10, [1], base)
    assert np.ptp(s) < 1e-12 * abs(s[0])
    want = float((A * np.linalg.norm(np.stack([k_pre[:64], k_pre[64:]]), axis=0)).sum())
    assert abs(s[0] - want) < 1e-12 * abs(want)


def test_relative_position_shift_invariance():
    """Shifting every key position and the query position by the same amount
    leaves every score unchanged ([Digest] "Framework Shift")."""
    rng = np.random.default_rng(8)
    D, base, G = 128, 5e5, 4
    T, p = 64, 5000
    deltas = [1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096]
    k_pre = torch.from_numpy(rng.normal(size=(T, D)))
    pos = torch.from_numpy(rng.integers(0, p, size=T))
    qbar = rng.normal(size=(G, D))
    qabs = np.abs(oracle.as_bands(qbar)) + rng.uniform(0, 1, size=(G, D // 2))
    R = rng.uniform(0.3, 0.95, size=G)
    s0 = oracle.unit_scores(rope_rotate_half(k_pre, pos, base).numpy(), qbar, qabs, R, p, deltas, base)
    for shift in (1, 977, 100000):
        s1 = oracle.unit_scores(rope_rotate_half(k_pre, pos + shift, base).numpy(), qbar, qabs, R,
                                p + shift, deltas, base)
        np.testing.assert_allclose(s1, s0, rtol=1e-9, atol=1e-9 * np.abs(s0).max())


# ---------------------------------------------------------------------------
# GQA aggregation
# ---------------------------------------------------------------------------

def test_group_fold_equals_mean_of_head_scores():
    rng = np.random.default_rng(9)
    D, G, base, p = 128, 4, 5e5, 32768
    deltas = [1, 2, 4, 8, 4096]
    keys = rng.normal(size=(50, D))
    qbar = rng.normal(size=(G, D))
    qabs = np.abs(oracle.as_bands(qbar)) + rng.uniform(0, 1, size=(G, D // 2))
    R = rng.uniform(0.3, 0.95, size=G)
    per_head = np.mean([oracle.head_score(keys, qbar[g], qabs[g], R[g], p, deltas, base) for g in range(G)], axis=0)
    np.testing.assert_allclose(oracle.unit_scores(keys, qbar, qabs, R, p, deltas, base), per_head, rtol=1e-13)
    qeff, w = oracle.group_query(qbar, qabs, R, p, deltas, base)
    kb = oracle.as_bands(keys)
    folded = keys @ qeff + np.abs(kb) @ w
    np.testing.assert_allclose(folded, per_head, rtol=1e-11, atol=1e-11 * np.abs(per_head).max())


def test_group_of_identical_heads_and_opposite_centres():
    rng = np.random.default_rng(10)
    D = 16
    keys = rng.normal(size=(9, D))
    q = rng.normal(size=D)
    A = np.abs(oracle.as_bands(q)) + 0.5
    one = oracle.unit_scores(keys, q[None], A[None], np.array([0.4]), 33, [1, 2], 1e4)
    two = oracle.unit_scores(keys, np.stack([q, q]), np.stack([A, A]), np.array([0.4, 0.4]), 33, [1, 2], 1e4)
    np.testing.assert_allclose(two, one, rtol=1e-14)
    # Opposite centres: the trig terms cancel, the norm terms remain.
    opp = oracle.unit_scores(keys, np.stack([q, -q]), np.stack([A, A]), np.array([0.4, 0.4]), 33, [1, 2], 1e4)
    norm_only = 0.6 * (np.abs(oracle.as_bands(keys)) @ (A - np.abs(oracle.as_bands(q))))
    np.testing.assert_allclose(opp, norm_only, rtol=1e-12)


# ---------------------------------------------------------------------------
# Calibration
# ---------------------------------------------------------------------------

def test_calibrate_centre_is_numpy_mean():
    rng = np.random.default_rng(11)
    q = rng.normal(size=(300, 3, 5, 16))
    qbar, qabs, R = oracle.calibrate(q)
    np.testing.assert_allclose(qbar, q.mean(axis=0), rtol=1e-14, atol=1e-15)
    mags = np.hypot(q[..., :8], q[..., 8:])
    np.testing.assert_allclose(qabs, mags.mean(axis=0), rtol=1e-14)
    assert np.all((R >= 0) & (R <= 1))


def test_calibrate_noise_free_gives_full_concentration():
    c = np.random.default_rng(12).normal(size=(2, 32))
    q = np.repeat(c[None], 17, axis=0)
    qbar, qabs, R = oracle.calibrate(q)
    np.testing.assert_allclose(R, 1.0, rtol=1e-14)
    np.testing.assert_allclose(qabs, np.abs(oracle.as_bands(c)), rtol=1e-14)


def test_calibrate_symmetric_samples_give_zero_concentration():
    z = np.random.default_rng(13).normal(size=(50, 1, 8))
    q = np.concatenate([z, -z], axis=0)
    _, _, R = oracle.calibrate(q)
    assert abs(R[0]) < 1e-15
    _, _, R0 = oracle.calibrate(np.zeros((4, 1, 8)))
    assert R0[0] == 1.0


def test_calibrate_rayleigh_mean():
    """Zero-mean isotropic Gaussian bands: E|z| = sigma sqrt(pi/2) (Rayleigh)."""
    rng = np.random.default_rng(14)
    sigma, N = 0.8, 200000
    q = sigma * rng.normal(size=(N, 1, 8))
    _, qabs, _ = oracle.calibrate(q)
    want = sigma * math.sqrt(math.pi / 2)
    se = sigma * math.sqrt((4 - math.pi) / 2) / math.sqrt(N)
    assert np.all(np.abs(qabs - want) < 5 * se)


def test_calibrate_hits_generator_concentration_target():
    """Samples drawn for a target concentration calibrate back to it."""
    rng = np.random.default_rng(15)
    D, N = 128, 20000
    c = rng.normal(size=D)
    cmag = np.abs(oracle.as_bands(c))
    for target in (0.3, 0.6, 0.98):
        sigma = noise_scale_for_target_concentration(cmag, target)
        q = c[None, None] + sigma * rng.normal(size=(N, 1, D))
        _, _, R = oracle.calibrate(q)
        assert abs(R[0] - target) < 0.01


# ---------------------------------------------------------------------------
# Selection
# ---------------------------------------------------------------------------

def _dominates(s, a, b):
    """a ranks before b: higher score, then lower slot (NaN lowest)."""
    va = -math.inf if math.isnan(s[a]) else s[a]
    vb = -math.inf if math.isnan(s[b]) else s[b]
    return va > vb or (va == vb and a < b)


@pytest.mark.parametrize("seed", range(30))
def test_select_brute_force_dominance(seed):
    rng = np.random.default_rng(100 + seed)
    length = int(rng.integers(1, 14))
    budget = int(rng.integers(1, 10))
    window = int(rng.integers(0, budget + 1))
    s = rng.integers(-3, 4, size=length).astype(np.float64)   # many ties
    if seed % 3 == 0:
        s[rng.integers(0, length)] = -0.0
    idx = oracle.select(s, length, budget, window)
    if length <= budget:
        assert list(idx) == list(range(length))
        return
    cand, take = length - window, budget - window
    kept = set(int(i) for i in idx)
    assert len(kept) == budget and list(idx) == sorted(kept)
    assert set(range(cand, length)) <= kept
    chosen = kept - set(range(cand, length))
    # brute force: the chosen set is the unique size-`take` subset of the
    # candidates that ranks every member ahead of every non-member
    winners = [set(c) for c in itertools.combinations(range(cand), take)
               if all(_dominates(s, a, b) for a in c for b in range(cand) if b not in c)]
    assert winners == [chosen]


def test_select_special_cases():
    s = np.arange(20, dtype=np.float64)[::-1].copy()       # strictly decreasing
    assert list(oracle.select(s, 20, 8, 3)) == [0, 1, 2, 3, 4, 17, 18, 19]
    s = np.arange(20, dtype=np.float64)                    # strictly increasing
    assert list(oracle.select(s, 20, 8, 3)) == [12, 13, 14, 15, 16, 17, 18, 19]
    s = np.zeros(20)                                       # all equal
    assert list(oracle.select(s, 20, 8, 3)) == [0, 1, 2, 3, 4, 17, 18, 19]
    assert list(oracle.select(s, 20, 8, 8)) == list(range(12, 20))    # window fills B
    assert list(oracle.select(s, 20, 8, 0)) == list(range(8))
    assert list(oracle.select(s, 8, 8, 3)) == list(range(8))          # B >= T keeps all
    assert list(oracle.select(s, 0, 8, 3)) == []
    z = np.array([0.0, -0.0, 0.0, -0.0, -1.0])                         # -0 == +0
    assert list(oracle.select(z, 5, 2, 0)) == [0, 1]
    nan = np.array([np.nan, -5.0, np.nan, -7.0, 1.0])                  # NaN lowest
    assert list(oracle.select(nan, 5, 3, 1)) == [1, 3, 4]
    with pytest.raises(ValueError):
        oracle.select(s, 20, 4, 5)


# ---------------------------------------------------------------------------
# Compaction
# ---------------------------------------------------------------------------

def test_compact_matches_fancy_indexing_and_preserves_order():
    rng = np.random.default_rng(16)
    rows = rng.integers(0, 2 ** 16, size=(100, 8)).astype(np.uint16)
    idx = np.sort(rng.choice(100, size=37, replace=False))
    out = oracle.compact_rows(rows, idx)
    np.testing.assert_array_equal(out[:37], rows[idx])
    np.testing.assert_array_equal(out[37:], rows[37:])
    # surviving rows appear in their original relative order
    pos = [int(np.where((rows == out[j]).all(axis=1))[0][0]) for j in range(37)]
    assert pos == sorted(pos)
    # keeping everything changes nothing
    np.testing.assert_array_equal(oracle.compact_rows(rows, np.arange(100)), rows)


def test_freed_blocks_are_the_emptied_tail():
    table = [7, 3, 9, 1, 4, 8]
    assert oracle.freed_blocks(table, 90, 33, 16) == [1, 4, 8]     # 6 blocks -> 3
    assert oracle.freed_blocks(table, 90, 90, 16) == []
    assert oracle.freed_blocks(table, 96, 32, 16) == [9, 1, 4, 8]
    assert oracle.freed_blocks(table, 0, 0, 16) == []
    for length in range(0, 97):
        for kept in range(0, length + 1):
            f = oracle.freed_blocks(table, length, kept, 16)
            assert len(f) == -(-length // 16) - (-(-kept // 16))


def _identity_pool(L, NB, Hkv, bs):
    """A pool whose row [l, b, h, r] holds its own address (l, b, h, r)."""
    pool = np.zeros((L, NB, Hkv, bs, 4), dtype=np.int64)
    for l, b, h, r in itertools.product(range(L), range(NB), range(Hkv), range(bs)):
        pool[l, b, h, r] = (l, b, h, r)
    return pool


def test_unit_rows_follow_the_block_table():
    """Slot t of a unit lives in row t mod 16 of the table's block t div 16
    ([GeoTrick] "Solving the Memory Fragmentation Problem": a sequence's
    cache is a chain of fixed-size pages named by its block table).  Block
    size 4 here; every expected address is written out by hand."""
    pool = _identity_pool(L=2, NB=8, Hkv=3, bs=4)
    table_row = [5, 2, 7, 0]                       # a permuted table
    rows = oracle.unit_rows(pool, table_row, 14, 1, 2)
    assert rows.shape == (14, 4)
    expected = {
        0: (1, 5, 2, 0), 1: (1, 5, 2, 1), 3: (1, 5, 2, 3),     # block table_row[0] = 5
        4: (1, 2, 2, 0), 6: (1, 2, 2, 2),                      # block table_row[1] = 2
        8: (1, 7, 2, 0), 9: (1, 7, 2, 1), 11: (1, 7, 2, 3),    # block table_row[2] = 7
        12: (1, 0, 2, 0), 13: (1, 0, 2, 1),                    # block table_row[3] = 0
    }
    for t, addr in expected.items():
        assert tuple(rows[t]) == addr, t
    # another layer and head through the same table
    rows0 = oracle.unit_rows(pool, table_row, 6, 0, 0)
    assert [tuple(r) for r in rows0] == [(0, 5, 0, 0), (0, 5, 0, 1), (0, 5, 0, 2), (0, 5, 0, 3),
                                         (0, 2, 0, 0), (0, 2, 0, 1)]
    assert oracle.unit_rows(pool, table_row, 0, 1, 1).shape == (0, 4)


def test_store_unit_rows_writes_exactly_the_table_addresses():
    """Storing a unit's rows touches rows (l, table[t div 16], h, t mod 16)
    for t < len and nothing else (block size 4 here, addresses by hand)."""
    L, NB, Hkv, bs = 2, 8, 3, 4
    pool = _identity_pool(L, NB, Hkv, bs)
    before = pool.copy()
    table_row = [6, 1, 4]
    marks = np.full((10, 4), -1, dtype=np.int64)
    marks[:, 0] = np.arange(10)
    oracle.tri_oracle.store_unit_rows(pool, table_row, marks, 0, 1)
    written = {(0, 6, 1, 0): 0, (0, 6, 1, 1): 1, (0, 6, 1, 2): 2, (0, 6, 1, 3): 3,
               (0, 1, 1, 0): 4, (0, 1, 1, 1): 5, (0, 1, 1, 2): 6, (0, 1, 1, 3): 7,
               (0, 4, 1, 0): 8, (0, 4, 1, 1): 9}
    for addr in itertools.product(range(L), range(NB), range(Hkv), range(bs)):
        if addr in written:
            assert pool[addr][0] == written[addr] and pool[addr][1] == -1, addr
        else:
            np.testing.assert_array_equal(pool[addr], before[addr])
    # reading back through the table returns what was stored
    np.testing.assert_array_equal(oracle.unit_rows(pool, table_row, 10, 0, 1), marks)


def test_paged_step_equals_unit_by_unit():
    """The paged compress_step moves exactly what compress_unit says, per unit,
    and leaves other rows alone."""
    rng = np.random.default_rng(17)
    L, Hkv, G, D, bs = 2, 2, 2, 8, 4
    lens, budget, window = [13, 5, 9], 6, 2
    NB = 12
    table = rng.permutation(NB)[:12].reshape(3, 4)
    k = rng.normal(size=(L, NB, Hkv, bs, D))
    kb = np.arange(k.size, dtype=np.int64).reshape(k.shape)      # row identities
    vb = -kb
    qbar = rng.normal(size=(L, Hkv * G, D))
    qabs = np.abs(oracle.as_bands(qbar)) + 0.3
    R = rng.uniform(0.2, 0.9, size=(L, Hkv * G))
    out = oracle.compress_step(k, kb, vb, table, lens, [20, 30, 40], qbar, qabs, R, G,
                               [1, 2], 1e4, budget, window)
    assert out["seq_len"] == [6, 5, 6]
    assert out["freed_ids"] == [int(table[0, 2]), int(table[0, 3]), int(table[2, 2])]
    for s in range(3):
        for l in range(L):
            for h in range(Hkv):
                keys = oracle.unit_rows(k, table[s], lens[s], l, h)
                sc, idx, nk, nv = oracle.compress_unit(
                    keys, oracle.unit_rows(kb, table[s], lens[s], l, h),
                    oracle.unit_rows(vb, table[s], lens[s], l, h),
                    qbar[l, h * G:(h + 1) * G], qabs[l, h * G:(h + 1) * G], R[l, h * G:(h + 1) * G],
                    [20, 30, 40][s], [1, 2], 1e4, budget, window)
                np.testing.assert_array_equal(out["idx"][(s, l, h)], idx)
                np.testing.assert_array_equal(oracle.unit_rows(out["k_pool"], table[s], lens[s], l, h), nk)
                np.testing.assert_array_equal(oracle.unit_rows(out["v_pool"], table[s], lens[s], l, h), nv)


# ---------------------------------------------------------------------------
# Figures printed on the pages
# ---------------------------------------------------------------------------

def test_page_memory_ratios():
    """Keeping B of T = 32768 cached keys reproduces the KV-memory figures the
    pages print (fixture cites them); the window counts inside the budget."""
    with open(os.path.join(GOLDEN, "page_memory_ratios.json")) as f:
        cases = json.load(f)["cases"]
    rng = np.random.default_rng(18)
    for c in cases:
        T, B, W = c["cached_tokens"], c["budget"], c["window"]
        s = rng.normal(size=T)
        idx = oracle.select(s, T, B, W)
        ratio = len(idx) / T
        if "memory_ratio_printed" in c:
            assert round(math.floor(ratio * 1000) / 1000, 3) == c["memory_ratio_printed"]
        assert round(T / len(idx), c["reduction_decimals"]) == c["reduction_printed"]
        freed = oracle.freed_blocks(list(range(T // 16)), T, len(idx), 16)
        assert len(freed) == (T - B) // 16


# ---------------------------------------------------------------------------
# Variants: attention sinks, compression trigger, max over the GQA group
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(20))
def test_select_with_sinks_brute_force(seed):
    """With s sinks: slots [0, s) and the last W slots are kept, plus the
    best (B - W - s) of the slots between, by (score desc, slot asc)."""
    rng = np.random.default_rng(300 + seed)
    length = int(rng.integers(1, 14))
    budget = int(rng.integers(1, 10))
    window = int(rng.integers(0, budget + 1))
    sinks = int(rng.integers(0, budget - window + 1))
    s = rng.integers(-3, 4, size=length).astype(np.float64)
    idx = oracle.select(s, length, budget, window, sinks)
    if length <= budget:
        assert list(idx) == list(range(length))
        return
    cand, take = length - window, budget - window - sinks
    kept = set(int(i) for i in idx)
    assert len(kept) == budget and list(idx) == sorted(kept)
    assert set(range(sinks)) <= kept and set(range(cand, length)) <= kept
    chosen = kept - set(range(sinks)) - set(range(cand, length))
    pool = range(sinks, cand)
    winners = [set(c) for c in itertools.combinations(pool, take)
               if all(_dominates(s, a, b) for a in c for b in pool if b not in c)]
    assert winners == [chosen]


def test_select_sinks_special_cases():
    inc = np.arange(20, dtype=np.float64)                 # later slots score higher
    assert list(oracle.select(inc, 20, 8, 3, 2)) == [0, 1, 14, 15, 16, 17, 18, 19]
    assert list(oracle.select(inc, 20, 8, 3, 0)) == [12, 13, 14, 15, 16, 17, 18, 19]
    assert list(oracle.select(inc, 20, 8, 0, 8)) == list(range(8))
    with pytest.raises(ValueError):
        oracle.select(inc, 20, 8, 5, 4)


def test_trigger_leaves_short_sequences_alone():
    rng = np.random.default_rng(19)
    L, Hkv, G, D, bs = 1, 1, 1, 8, 4
    k = rng.normal(size=(L, 12, Hkv, bs, D))
    kb = np.arange(k.size, dtype=np.int64).reshape(k.shape)
    table = np.arange(12).reshape(3, 4)
    qbar = rng.normal(size=(L, 1, D))
    qabs = np.abs(oracle.as_bands(qbar)) + 0.2
    R = np.array([[0.5]])
    lens = [10, 14, 16]
    out = oracle.compress_step(k, kb, -kb, table, lens, [20, 20, 20], qbar, qabs, R, G, [1], 1e4,
                               budget=8, window=2, trigger=12)
    assert out["seq_len"] == [10, 8, 8]                  # 10 <= trigger untouched
    np.testing.assert_array_equal(out["k_pool"][0, 0:3], kb[0, 0:3])
    assert out["freed_ids"] == [int(table[1, 2]), int(table[1, 3]), int(table[2, 2]), int(table[2, 3])]
    low = oracle.compress_step(k, kb, -kb, table, lens, [20, 20, 20], qbar, qabs, R, G, [1], 1e4,
                               budget=8, window=2, trigger=3)   # below the budget: the budget
    assert low["seq_len"] == [8, 8, 8]


def test_max_over_group_matches_per_head_brute_force():
    """aggregate='max' is the largest of the G per-head scores, each from the
    mean rotated-centre logit (explicit rotation matrices) plus its norm term."""
    rng = np.random.default_rng(20)
    D, G, base, p = 8, 3, 1e4, 50
    deltas = [1, 3, 9]
    T = 12
    pos = rng.integers(0, p, size=T)
    k_pre = rng.normal(size=(T, D))
    k_post = np.stack([_rotate_explicit(k_pre[t], pos[t], base) for t in range(T)])
    qbar = rng.normal(size=(G, D))
    qmag = np.abs(oracle.as_bands(qbar))
    A = qmag + rng.uniform(0.1, 1.0, size=(G, D // 2))
    R = rng.uniform(0.2, 0.9, size=G)
    per_head = np.zeros((G, T))
    for g in range(G):
        for t in range(T):
            trig = np.mean([_rotate_explicit(qbar[g], p + d, base) @ k_post[t] for d in deltas])
            bands = np.hypot(k_pre[t, :D // 2], k_pre[t, D // 2:])
            per_head[g, t] = trig + (1 - R[g]) * float(((A[g] - qmag[g]) * bands).sum())
    got = oracle.unit_scores(k_post, qbar, A, R, p, deltas, base, aggregate="max")
    np.testing.assert_allclose(got, per_head.max(axis=0), rtol=1e-10, atol=1e-12)
    one = oracle.unit_scores(k_post, qbar[:1], A[:1], R[:1], p, deltas, base, aggregate="max")
    np.testing.assert_allclose(one, oracle.unit_scores(k_post, qbar[:1], A[:1], R[:1], p, deltas, base), rtol=1e-14)


# ---------------------------------------------------------------------------
# Variant: the distance-only table of the centres
# ---------------------------------------------------------------------------

def test_distance_table_is_rotated_centre_logit():
    """f(p - t) = mean_g mean_delta RoPE(qbar_g, p + delta) . RoPE(kbar, t) with
    explicit rotation matrices, for many (p, t) with the same distance."""
    rng = np.random.default_rng(30)
    D, G, base = 8, 3, 1e4
    deltas = [1, 2, 4, 9]
    qbar = rng.normal(size=(G, D))
    kbar = rng.normal(size=D)
    table = oracle.distance_table(qbar, kbar, deltas, base, 60)
    for p, t in [(50, 10), (60, 20), (45, 5), (33, 33), (60, 0), (7, 0)]:
        want = np.mean([np.mean([_rotate_explicit(qbar[g], p + d, base) @ _rotate_explicit(kbar, t, base)
                                 for d in deltas]) for g in range(G)])
        assert table[p - t] == pytest.approx(want, rel=1e-11, abs=1e-12)
    mx = oracle.distance_table(qbar, kbar, deltas, base, 60, aggregate="max")
    per = [oracle.distance_table(qbar[g:g + 1], kbar, deltas, base, 60) for g in range(G)]
    np.testing.assert_allclose(mx, np.max(per, axis=0), rtol=1e-14)


def test_distance_table_equals_trig_term_of_keys_on_their_centre():
    """Keys exactly at the key centre (k_t = RoPE(kbar, t)) with R = 1 (no
    norm term): the method's own unit score is the table at p - t."""
    rng = np.random.default_rng(31)
    D, G, base, p = 16, 2, 5e5, 300
    deltas = [1, 2, 4, 8, 16]
    qbar = rng.normal(size=(G, D))
    kbar = rng.normal(size=D)
    ts = np.array([0, 1, 5, 77, 150, 299])
    keys = np.stack([_rotate_explicit(kbar, int(t), base) for t in ts])
    qabs = np.abs(oracle.as_bands(qbar)) + 0.5
    got = oracle.unit_scores(keys, qbar, qabs, np.ones(G), p, deltas, base)
    table = oracle.distance_table(qbar, kbar, deltas, base, p)
    np.testing.assert_allclose(got, table[p - ts], rtol=1e-10, atol=1e-10)


def test_distance_table_closed_form_two_dims():
    """D = 2: f(dist) = |qbar||kbar| mean_delta cos(theta_0 (dist + delta) + phi)."""
    qbar = np.array([[0.6, -1.1]])
    kbar = np.array([1.3, 0.4])
    deltas, base = [1, 3, 10], 1e4
    table = oracle.distance_table(qbar, kbar, deltas, base, 40)
    zq, zk = complex(0.6, -1.1), complex(1.3, 0.4)
    phi = np.angle(zq) - np.angle(zk)
    for dist in (0, 1, 17, 40):
        want = abs(zq) * abs(zk) * np.mean([np.cos(1.0 * (dist + d) + phi) for d in deltas])
        assert table[dist] == pytest.approx(want, rel=1e-12, abs=1e-13)


def test_distance_step_moves_positions_with_rows():
    """After a distance-table step the kept rows carry their positions: the
    scores recomputed from the new positions are the kept keys' old scores,
    and the selection is the plain selection of f(p - pos)."""
    rng = np.random.default_rng(32)
    L, Hkv, bs, D, S = 1, 2, 4, 8, 2
    NB = 12
    kb = rng.integers(-30000, 30000, size=(L, NB, Hkv, bs, D)).astype(np.int16)
    vb = rng.integers(-30000, 30000, size=(L, NB, Hkv, bs, D)).astype(np.int16)
    table_ids = np.array([[3, 0, 7, 5, 9, 1], [2, 4, 6, 8, 10, 11]])
    lens, p = [21, 14], [40, 30]
    pos = np.zeros((S, L, Hkv, 24), dtype=np.int64)
    for s in range(S):
        for h in range(Hkv):
            pos[s, 0, h, :lens[s]] = np.sort(rng.choice(p[s], lens[s], replace=False))
    tables = rng.normal(size=(L, Hkv, 41))
    out = oracle.compress_step_distance(kb, vb, table_ids, lens, p, pos, tables, budget=8, window=2, sinks=1,
                                        trigger=15)
    assert out["seq_len"] == [8, 14]
    for h in range(Hkv):
        sc = tables[0, h, p[0] - pos[0, 0, h, :21]]
        idx = oracle.select(sc, 21, 8, 2, 1)
        assert np.array_equal(out["idx"][(0, 0, h)], idx)
        assert np.array_equal(out["positions"][0, 0, h, :8], pos[0, 0, h, idx])
        again = oracle.distance_scores(tables[0, h], p[0], out["positions"][0, 0, h, :8])
        np.testing.assert_array_equal(again, sc[idx])
        rows = oracle.unit_rows(out["k_pool"], table_ids[0], 8, 0, h)
        np.testing.assert_array_equal(rows, oracle.unit_rows(kb, table_ids[0], 21, 0, h)[idx])
    np.testing.assert_array_equal(out["positions"][1], pos[1])                 # untouched (14 <= 15)
    assert out["freed_ids"] == [int(table_ids[0, 2]), int(table_ids[0, 3]), int(table_ids[0, 4]),
                                int(table_ids[0, 5])]
    with pytest.raises(ValueError):
        oracle.distance_scores(tables[0, 0], 5, [6])                            # key after the query
