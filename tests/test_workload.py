"""The seeded generator and the decode-loop bookkeeping (CPU only)."""

import numpy as np
import pytest
import torch

from workload import CONFIGS, make_workload, rope_rotate_half
from workload.decode import PoolExhausted, append_tokens, recycle_freed


def _small(name, **kw):
    return CONFIGS[name].replace(**kw)


def test_generator_is_deterministic():
    cfg = _small("l32h8_t32k", L=2, lens=[300], n_samples=64)
    a, b = make_workload(cfg), make_workload(cfg)
    assert torch.equal(a.k_pool, b.k_pool) and torch.equal(a.v_pool, b.v_pool)
    assert torch.equal(a.q_samples, b.q_samples)
    c = make_workload(cfg, seed=1)
    assert not torch.equal(a.k_pool, c.k_pool)


def test_shapes_and_tables():
    cfg = _small("l64h8g8_4x64k", L=2, lens=[70, 33, 1, 16], n_samples=8)
    wl = make_workload(cfg)
    L, NB, Hkv, bs, D = wl.k_pool.shape
    assert (L, Hkv, bs, D) == (2, 8, 16, 128) and wl.k_pool.dtype == torch.bfloat16
    assert wl.q_samples.shape == (8, 2, 64, 128)
    tab = wl.block_table.tolist()
    used = []
    for s, n in enumerate([70, 33, 1, 16]):
        nb = -(-n // 16)
        assert all(0 <= b < NB for b in tab[s][:nb]) and all(b == -1 for b in tab[s][nb:])
        used += tab[s][:nb]
    assert len(set(used)) == len(used)
    assert set(used).isdisjoint(wl.free_blocks)
    assert wl.seq_len.tolist() == [70, 33, 1, 16] and wl.cur_pos.tolist() == [70, 33, 1, 16]


def test_cached_keys_are_rotated_centred_draws():
    """Each cached key, rotated back by its position, lies near its head's centre."""
    cfg = _small("head1_t4096", lens=[64])
    wl = make_workload(cfg)
    keys = wl.k_pool[0, 0:4, 0].reshape(64, 128).double()
    back = rope_rotate_half(keys, -torch.arange(64, dtype=torch.float64), cfg.base)
    resid = back - wl.key_centres[0, 0][None]
    # noise 0.3 per dimension plus bf16 rounding of O(1) values
    assert resid.std().item() == pytest.approx(0.3, rel=0.1)


def test_direct_statistics():
    wl = make_workload(CONFIGS["head1_t4096"])
    mag = torch.sqrt(wl.qbar[..., :64].double() ** 2 + wl.qbar[..., 64:].double() ** 2)
    torch.testing.assert_close(wl.qabs.double(), 1.2 * mag, rtol=1e-6, atol=0)
    assert abs(wl.R.item() - 1 / 1.2) < 1e-7


def test_decode_append_and_recycle():
    cfg = _small("decode16", L=1, lens=[0, 0], lens_range=(40, 60), budget=32, window=8,
                 decode_append=20, n_samples=8)
    wl = make_workload(cfg)
    old = wl.seq_len.tolist()
    free0 = len(wl.free_blocks)
    append_tokens(wl, 0, 20)
    assert wl.seq_len[0].item() == old[0] + 20 and wl.cur_pos[0].item() == old[0] + 20
    nb = -(-(old[0] + 20) // 16)
    assert (wl.block_table[0, :nb] >= 0).all()
    assert len(wl.free_blocks) == free0 - (nb - (-(-old[0] // 16)))
    # pretend a step kept 32 rows of each sequence
    lens = wl.seq_len.tolist()
    expect = []
    for s in range(2):
        expect += wl.block_table[s, 2:-(-lens[s] // 16)].tolist()
    wl.seq_len[:] = 32
    freed = torch.tensor(expect + [999], dtype=torch.int32)
    ids = recycle_freed(wl, lens, freed, len(expect))
    assert ids == expect and (wl.block_table[:, 2:] == -1).all()
    with pytest.raises(AssertionError):
        recycle_freed(wl, [32, 32], torch.tensor([5], dtype=torch.int32), 1)
    with pytest.raises(PoolExhausted):
        append_tokens(wl, 0, 10 ** 6)
