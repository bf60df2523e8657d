"""Seeded synthetic KV caches and query calibration samples.

Pages cited (title, then section):
  [Digest]   "TriAttention: Trigonometric KV Compression for Efficient Long Reasoning"
  [GeoTrick] "TriAttention: How a Geometric Trick Cuts LLM Memory Use by 10x
              Without Losing Accuracy"
  [Abstract] "TriAttention: Efficient Long Reasoning with Trigonometric KV Compression"

What is drawn, and why it looks like this:

* Pre-RoPE keys of a KV head cluster around a fixed non-zero centre
  ([Abstract] "English"; [Digest] "Key Concepts", Q/K Concentration):
  k_t = c_k + key_noise * N(0, I) with c_k ~ N(0, I) per (layer, KV head).
* The cache stores keys after rotary embedding ([Digest] "The Gap"); keys are
  rotated in float64 at their own position t and only then rounded to bf16.
* Values are N(0, I) in bf16 (the pages never describe V).
* Query statistics: per query head a centre c_q ~ N(0, I) and calibration
  samples q = c_q + sigma * N(0, I), sigma chosen so that the large-sample
  concentration of the head hits a drawn target; or, where a workload states
  E|q_i| directly, the statistics themselves.
* The cache is paged: [layer][block][KV head][16 rows][128] bf16 with a
  per-sequence block table ([GeoTrick] "Why Existing KV Cache Compression
  Breaks in Production", the paged allocator).

Everything is drawn from one ``torch.Generator`` seeded by the workload seed,
on the device the tensors are built on.  Rows of the pool that hold no token
are filled with random garbage so that a kernel reading past a sequence's end
produces visibly wrong results.

Rotary embedding here is the model's positional encoding, used only to
synthesise the cached keys; the CUDA path never applies it.  It uses the
rotate-half pairing (dimension i with i + D/2) and frequencies
base^(-2i/D), the convention of the HuggingFace models the pages list.
"""

from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch

from .configs import WorkloadConfig


def rope_rotate_half(x: torch.Tensor, pos: torch.Tensor, base: float) -> torch.Tensor:
    """Rotate float64 vectors ``x[..., D]`` to positions ``pos[...]``.

    Pairs dimension i with i + D/2 and turns the pair by pos * base^(-2i/D).
    """
    D = x.shape[-1]
    n = D // 2
    i = torch.arange(n, dtype=torch.float64, device=x.device)
    inv_freq = torch.pow(torch.tensor(base, dtype=torch.float64, device=x.device), -2.0 * i / D)
    ang = pos.to(torch.float64)[..., None] * inv_freq
    c, s = torch.cos(ang), torch.sin(ang)
    x1, x2 = x[..., :n], x[..., n:]
    return torch.cat([x1 * c - x2 * s, x2 * c + x1 * s], dim=-1)


def _rice_mean(nu: np.ndarray, sigma: float) -> np.ndarray:
    """Mean of |c + sigma (x + j y)|, x, y ~ N(0, 1), |c| = nu (Rice law)."""
    from scipy.special import i0e, i1e
    if sigma == 0.0:
        return nu.copy()
    a = nu * nu / (2.0 * sigma * sigma)
    lag = (1.0 + a) * i0e(a / 2.0) + a * i1e(a / 2.0)
    return sigma * math.sqrt(math.pi / 2.0) * lag


def noise_scale_for_target_concentration(centre_band_mag: np.ndarray, target: float) -> float:
    """Noise scale sigma for which sum_i |c_i| / sum_i E|c_i + noise_i| = target.

    ``centre_band_mag`` holds the D/2 band magnitudes |c_i| of one head's
    centre.  This shapes inputs only: the concentration the method uses is
    measured from the drawn samples by each implementation on its own.
    """
    if not (0.0 < target <= 1.0):
        raise ValueError("target concentration must lie in (0, 1]")
    num = float(centre_band_mag.sum())
    if target >= 1.0:
        return 0.0
    lo, hi = 0.0, 1.0
    while num / float(_rice_mean(centre_band_mag, hi).sum()) > target:
        hi *= 2.0
    for _ in range(80):
        mid = 0.5 * (lo + hi)
        if num / float(_rice_mean(centre_band_mag, mid).sum()) > target:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def _noise_scales(mags: np.ndarray, targets: np.ndarray) -> np.ndarray:
    """``noise_scale_for_target_concentration`` for many heads at once."""
    from scipy.special import i0e, i1e

    def conc(sig):
        a = mags * mags / (2.0 * sig[:, None] ** 2)
        mean = sig[:, None] * math.sqrt(math.pi / 2.0) * ((1.0 + a) * i0e(a / 2.0) + a * i1e(a / 2.0))
        return mags.sum(1) / mean.sum(1)

    if np.any(targets <= 0.0) or np.any(targets > 1.0):
        raise ValueError("target concentration must lie in (0, 1]")
    lo = np.zeros(len(targets))
    hi = np.ones(len(targets))
    while True:
        grow = conc(hi) > targets
        if not grow.any():
            break
        hi[grow] *= 2.0
    for _ in range(80):
        mid = 0.5 * (lo + hi)
        above = conc(np.maximum(mid, 1e-300)) > targets
        lo = np.where(above, mid, lo)
        hi = np.where(above, hi, mid)
    out = 0.5 * (lo + hi)
    out[targets >= 1.0] = 0.0
    return out


@dataclasses.dataclass
class Workload:
    """Device tensors of one synthetic workload, laid out as the C ABI wants."""

    cfg: WorkloadConfig
    k_pool: torch.Tensor          # bf16 [L][NB][Hkv][bs][D]
    v_pool: torch.Tensor          # bf16 [L][NB][Hkv][bs][D]
    block_table: torch.Tensor     # int32 [S][max_blocks]
    seq_len: torch.Tensor         # int32 [S]
    cur_pos: torch.Tensor         # int64 [S]
    deltas: List[int]
    q_samples: Optional[torch.Tensor]   # float32 [N][L][Hq][D]
    qbar: Optional[torch.Tensor]        # float32 [L][Hq][D]   (direct stats)
    qabs: Optional[torch.Tensor]        # float32 [L][Hq][D/2] (direct stats)
    R: Optional[torch.Tensor]           # float32 [L][Hq]      (direct stats)
    key_centres: torch.Tensor           # float64 [L][Hkv][D]
    free_blocks: List[int]              # pool blocks owned by no sequence
    gen: torch.Generator

    @property
    def num_blocks(self) -> int:
        return self.k_pool.shape[1]

    @property
    def max_blocks(self) -> int:
        return self.block_table.shape[1]

    @property
    def device(self) -> torch.device:
        return self.k_pool.device


def _draw_lengths(cfg: WorkloadConfig, rng: np.random.Generator) -> List[int]:
    if cfg.lens_range is None:
        return list(cfg.lens)
    lo, hi = cfg.lens_range
    return [int(x) for x in rng.integers(lo, hi + 1, size=len(cfg.lens))]


def write_tokens(wl: Workload, s: int, start: int, count: int) -> None:
    """Draw ``count`` new tokens for sequence ``s`` at slots start..start+count-1.

    The tokens sit at positions cur_pos[s] .. cur_pos[s]+count-1 (the slot
    index and the position differ once a sequence has been compacted).  The
    block table must already map those slots.  Used both for the initial
    cache (start = 0, positions 0..) and for decode-loop appends.
    """
    cfg = wl.cfg
    dev = wl.device
    bs, D, Hkv = cfg.block_size, cfg.D, cfg.Hkv
    if count <= 0:
        return
    pos0 = int(wl.cur_pos[s].item())
    pos = torch.arange(pos0, pos0 + count, device=dev, dtype=torch.float64)
    slots = torch.arange(start, start + count, device=dev, dtype=torch.int64)
    blk = wl.block_table[s].to(torch.int64)[slots // bs]
    row = slots % bs
    for l in range(cfg.L):
        noise = torch.randn(count, Hkv, D, dtype=torch.float64, device=dev, generator=wl.gen)
        pre = wl.key_centres[l][None] + cfg.key_noise * noise
        post = rope_rotate_half(pre, pos[:, None].expand(count, Hkv), cfg.base)
        val = torch.randn(count, Hkv, D, dtype=torch.float32, device=dev, generator=wl.gen)
        # pool[l, blk, h, row, :] <- post[t, h, :]
        kl = wl.k_pool[l]
        vl = wl.v_pool[l]
        kl[blk[:, None], torch.arange(Hkv, device=dev)[None, :], row[:, None]] = post.to(torch.bfloat16)
        vl[blk[:, None], torch.arange(Hkv, device=dev)[None, :], row[:, None]] = val.to(torch.bfloat16)


def _query_statistics(cfg: WorkloadConfig, dev, gen: torch.Generator, rng: np.random.Generator,
                      with_samples: bool):
    """Draw query centres and either calibration samples or direct statistics."""
    L, Hq, D = cfg.L, cfg.Hq, cfg.D
    n = D // 2
    centres = torch.randn(L, Hq, D, dtype=torch.float64, device=dev, generator=gen)
    if cfg.stats == "direct":
        # E|q_i| is stated as qabs_ratio * |c_i|; under the concentration
        # R = sum|qbar_i| / sum E|q_i| this gives R = 1 / qabs_ratio exactly.
        mag = torch.sqrt(centres[..., :n] ** 2 + centres[..., n:] ** 2)
        qbar = centres.to(torch.float32)
        qabs = (cfg.qabs_ratio * mag).to(torch.float32)
        R = torch.full((L, Hq), 1.0 / cfg.qabs_ratio, dtype=torch.float32, device=dev)
        return None, qbar, qabs, R
    if not with_samples:
        return None, None, None, None
    lo, hi = cfg.r_range
    targets = rng.uniform(lo, hi, size=(L, Hq))
    if cfg.low_r_fraction > 0.0:
        n_low = int(round(cfg.low_r_fraction * L * Hq))
        pick = rng.permutation(L * Hq)[:n_low]
        targets.reshape(-1)[pick] = cfg.low_r_value
    cmag = torch.sqrt(centres[..., :n] ** 2 + centres[..., n:] ** 2).cpu().numpy()
    sigma = _noise_scales(cmag.reshape(L * Hq, n), targets.reshape(-1)).reshape(L, Hq)
    sig = torch.tensor(sigma, dtype=torch.float64, device=dev)
    N = cfg.n_samples
    q = torch.empty(N, L, Hq, D, dtype=torch.float32, device=dev)
    for l in range(L):
        noise = torch.randn(N, Hq, D, dtype=torch.float64, device=dev, generator=gen)
        q[:, l] = (centres[l][None] + sig[l][None, :, None] * noise).to(torch.float32)
    return q, None, None, None


def make_workload(cfg: WorkloadConfig, device="cpu", seed: Optional[int] = None,
                  with_samples: bool = True) -> Workload:
    """Build the seeded workload ``cfg`` on ``device``.

    The same (cfg, seed, device) always yields the same tensors.  Different
    devices use different random streams, so CPU and GPU workloads differ;
    both sides of every comparison are always given the same tensors.
    """
    seed = cfg.seed if seed is None else seed
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    rng = np.random.default_rng(seed)

    lens = _draw_lengths(cfg, rng)
    S, L, Hkv, D, bs = len(lens), cfg.L, cfg.Hkv, cfg.D, cfg.block_size
    need = [(t + bs - 1) // bs for t in lens]
    extra = cfg.extra_blocks_per_seq
    if cfg.decode_rounds > 0:
        extra = max(extra, (cfg.decode_append + bs - 1) // bs + 1)
    max_blocks = max(max(need), (cfg.budget + bs - 1) // bs) + extra
    max_blocks = max(max_blocks, 1)

    if cfg.table == "identity":
        NB = S * max_blocks
        table = torch.arange(NB, dtype=torch.int32).view(S, max_blocks).clone()
        free: List[int] = []
        for s in range(S):
            table[s, need[s]:] = -1
            free += list(range(s * max_blocks + need[s], (s + 1) * max_blocks))
    else:
        total = sum(need)
        NB = max(int(math.ceil(total * (1.0 + cfg.pool_headroom))), total) + extra * S
        perm = rng.permutation(NB)
        table = torch.full((S, max_blocks), -1, dtype=torch.int32)
        off = 0
        for s in range(S):
            blocks = perm[off:off + need[s]]
            off += need[s]
            table[s, :need[s]] = torch.tensor(blocks, dtype=torch.int32)
        free = [int(b) for b in perm[off:]]

    k_pool = torch.empty(L, NB, Hkv, bs, D, dtype=torch.bfloat16, device=dev)
    v_pool = torch.empty(L, NB, Hkv, bs, D, dtype=torch.bfloat16, device=dev)
    for pool in (k_pool, v_pool):            # garbage in rows no token uses
        for l in range(L):
            pool[l].copy_(torch.randn(NB, Hkv, bs, D, device=dev, generator=gen) * 2.0)
    key_centres = torch.randn(L, Hkv, D, dtype=torch.float64, device=dev, generator=gen)

    q_samples, qbar, qabs, R = _query_statistics(cfg, dev, gen, rng, with_samples)

    wl = Workload(
        cfg=cfg, k_pool=k_pool, v_pool=v_pool,
        block_table=table.to(dev), seq_len=torch.tensor(lens, dtype=torch.int32, device=dev),
        cur_pos=torch.zeros(S, dtype=torch.int64, device=dev), deltas=list(cfg.deltas),
        q_samples=q_samples, qbar=qbar, qabs=qabs, R=R, key_centres=key_centres,
        free_blocks=free, gen=gen)
    for s in range(S):
        write_tokens(wl, s, 0, lens[s])
        wl.cur_pos[s] = lens[s]
    return wl
