"""The plain C oracle (used to time the CPU baseline on every host core)
against the numpy oracle: same scores to rounding, same kept slots, same
compacted rows.  CPU only."""

import numpy as np
import pytest
import torch

import oracle
from oracle.c_oracle import compress_unit_c


def _bf16_bits(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy()


def _unit(rng, T, D, G, dup=False):
    keys = rng.normal(size=(T, D))
    if dup and T > 4:
        keys[T // 2] = keys[1]                      # an exact tie in score
    kb = _bf16_bits(keys)
    vb = _bf16_bits(rng.normal(size=(T, D)))
    qbar = rng.normal(size=(G, D))
    qabs = np.abs(oracle.as_bands(qbar)) + rng.uniform(0.0, 1.0, size=(G, D // 2))
    R = rng.uniform(0.2, 1.0, size=G)
    return kb, vb, qbar, qabs, R


@pytest.mark.parametrize("T,G,budget,window", [(0, 1, 4, 1), (1, 2, 4, 1), (5, 1, 8, 2), (40, 4, 16, 4),
                                               (200, 3, 64, 0), (200, 2, 64, 64), (300, 8, 1, 1), (123, 1, 122, 5)])
def test_c_oracle_matches_numpy_oracle(T, G, budget, window):
    rng = np.random.default_rng(T * 31 + G * 7 + budget)
    D, p, base = 128, T + 17, 5e5
    deltas = [1, 2, 4, 8, 16, 4096]
    kb, vb, qbar, qabs, R = _unit(rng, T, D, G, dup=True)
    s_c, idx_c, k_c, v_c = compress_unit_c(kb, vb, qbar, qabs, R, p, deltas, base, budget, window)
    kf = torch.from_numpy(kb).view(torch.bfloat16).double().numpy()
    s_py, idx_py, k_py, v_py = oracle.compress_unit(kf, kb, vb, qbar, qabs, R, p, deltas, base, budget, window)
    scale = max(1.0, float(np.max(np.abs(s_py)))) if T else 1.0
    np.testing.assert_allclose(s_c, s_py, rtol=1e-12, atol=1e-12 * scale)
    assert np.array_equal(idx_c, idx_py)
    assert np.array_equal(k_c, k_py) and np.array_equal(v_c, v_py)


@pytest.mark.parametrize("T,G,budget,window,sinks,agg", [(40, 4, 16, 4, 3, "mean"), (200, 2, 64, 8, 5, "max"),
                                                          (200, 8, 64, 0, 0, "max"), (100, 1, 30, 10, 20, "mean"),
                                                          (64, 4, 64, 4, 4, "max"), (65, 3, 9, 0, 9, "mean")])
def test_c_oracle_variants_match_numpy_oracle(T, G, budget, window, sinks, agg):
    """Attention sinks and the max over the group, as the numpy oracle
    defines them."""
    rng = np.random.default_rng(T * 13 + G + sinks)
    D, p, base = 128, T + 5, 1e6
    deltas = [1, 2, 4, 8, 1024]
    kb, vb, qbar, qabs, R = _unit(rng, T, D, G, dup=True)
    s_c, idx_c, k_c, v_c = compress_unit_c(kb, vb, qbar, qabs, R, p, deltas, base, budget, window, sinks, agg)
    kf = torch.from_numpy(kb).view(torch.bfloat16).double().numpy()
    s_py, idx_py, k_py, v_py = oracle.compress_unit(kf, kb, vb, qbar, qabs, R, p, deltas, base, budget, window,
                                                    sinks=sinks, aggregate=agg)
    scale = max(1.0, float(np.max(np.abs(s_py))))
    np.testing.assert_allclose(s_c, s_py, rtol=1e-12, atol=1e-12 * scale)
    assert np.array_equal(idx_c, idx_py)
    if T > budget:
        assert np.array_equal(idx_c[:sinks], np.arange(sinks))
    assert np.array_equal(k_c, k_py) and np.array_equal(v_c, v_py)


def test_c_oracle_rejects_bad_arguments():
    rng = np.random.default_rng(0)
    kb, vb, qbar, qabs, R = _unit(rng, 10, 128, 1)
    with pytest.raises(ValueError):
        compress_unit_c(kb, vb, qbar, qabs, R, 10, [1], 1e4, 4, 5)        # window > budget
    with pytest.raises(ValueError):
        compress_unit_c(kb, vb, qbar, qabs, R, 10, [1], 1e4, 4, 2, 3)     # sinks + window > budget
    with pytest.raises(ValueError):
        compress_unit_c(kb, vb, qbar, qabs, R, 10, [1], 1e4, 4, 2, 0, "median")
