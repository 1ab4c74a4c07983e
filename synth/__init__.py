"""Seeded synthetic inputs for the hybrid KV-cache decode path.

This module is shared by the CPU oracle side and the CUDA side *as input
only*: it draws random fp16 tensors and holds none of the method's
arithmetic (no quantization, attention or selection).

Recipe (the pages' models and datasets are not available; only their shapes
are used -- Llama-3.1-8B / Qwen3-8B attention: 32 query heads, 8 KV heads,
head_dim 128):
  * Q, K, V entries ~ N(0, 1) drawn in fp32, rounded to fp16 (RNE).
  * K outliers: per (batch, kv head) unit, 4 distinct channels are multiplied
    by 8 at every position.
  * Vertical-line planting: per unit, u = mean of the unit's selection-query
    rows (64 queries x G heads), normalised; planted positions get
    K += 4 * sqrt(128) * u (a boost of 4 in logit units for a query aligned
    with u).  Planted positions are distinct and drawn uniformly from
    [0, T - W); the very-long-context workload always plants position 0
    (attention sink) and draws the rest from [1, T - W).
  * Seeds: 0x4859510000 + workload id; every tensor uses its own stream keyed
    by (seed, tag, batch, head, step) so any unit can be drawn alone.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

D = 128
W = 128
N_Q = 64
BASE_SEED = 0x4859510000

_TAG_QSEL, _TAG_Q, _TAG_K, _TAG_V, _TAG_OUT, _TAG_PLANT, _TAG_KNEW, _TAG_VNEW = range(1, 9)


@dataclasses.dataclass(frozen=True)
class Config:
    cid: int
    name: str
    B: int
    Hq: int
    Hkv: int
    T: int            # positions in the cache at the first decode step
    k: int            # vertical-line count
    W: int = W
    n_q: int = N_Q
    steps: int = 0    # streaming steps (workload 5)
    reselect: int = 64
    sink: bool = False
    seed: int = 0

    @property
    def G(self):
        return self.Hq // self.Hkv

    @property
    def units(self):
        return self.B * self.Hkv

    @property
    def capacity(self):
        t = self.T + self.steps
        return ((t + 63) // 64) * 64

    def rng(self, *key):
        return np.random.Generator(np.random.PCG64(np.random.SeedSequence([self.seed & 0xFFFFFFFF, self.seed >> 32, *key])))


def config(cid: int) -> Config:
    """The five workloads: tiny, Llama-3.1-8B 32K, batched 32K, 128K, streaming."""
    s = BASE_SEED + cid
    if cid == 1:
        return Config(1, "tiny-4k-b1-gqa8/2", 1, 8, 2, 4096, 64, seed=s)
    if cid == 2:
        return Config(2, "llama3.1-8b-32k-b1", 1, 32, 8, 32768, int(0.03 * 32768), seed=s)
    if cid == 3:
        return Config(3, "batched-32k-b16", 16, 32, 8, 32768, int(0.03 * 32768), seed=s)
    if cid == 4:
        return Config(4, "long-128k-b4-sink", 4, 32, 8, 131072, int(0.02 * 131072) + 1, sink=True, seed=s)
    if cid == 5:
        return Config(5, "qwen3-8b-stream-16k-b8", 8, 32, 8, 16384, int(0.04 * 16384), steps=512, seed=s)
    raise ValueError(cid)


def custom(B, Hq, Hkv, T, k, seed=12345, steps=0, sink=False, W_=W, n_q=N_Q) -> Config:
    return Config(0, f"custom-B{B}-{Hq}/{Hkv}-T{T}-k{k}", B, Hq, Hkv, T, k, W=W_, n_q=n_q,
                  steps=steps, sink=sink, seed=seed)


def _normal16(rng, shape):
    return rng.standard_normal(shape, dtype=np.float32).astype(np.float16)


def qsel(cfg: Config, b: int) -> np.ndarray:
    """Selection queries of batch b: [Hq][n_q][128] fp16."""
    return _normal16(cfg.rng(_TAG_QSEL, b), (cfg.Hq, cfg.n_q, D))


def q(cfg: Config, step: int = 0) -> np.ndarray:
    """Decode queries of one step: [B][Hq][128] fp16."""
    return _normal16(cfg.rng(_TAG_Q, step), (cfg.B, cfg.Hq, D))


def outlier_channels(cfg: Config, b: int, h: int) -> np.ndarray:
    return np.sort(cfg.rng(_TAG_OUT, b, h).choice(D, 4, replace=False))


def planted_positions(cfg: Config, b: int, h: int) -> np.ndarray:
    n_old = cfg.T - cfg.W
    k = min(cfg.k, max(n_old, 0))
    r = cfg.rng(_TAG_PLANT, b, h)
    if k == 0:
        return np.zeros(0, np.int32)
    if cfg.sink:
        rest = r.choice(np.arange(1, n_old), k - 1, replace=False)
        pos = np.concatenate([[0], rest])
    else:
        pos = r.choice(n_old, k, replace=False)
    return np.sort(pos).astype(np.int32)


def unit_kv(cfg: Config, b: int, h: int, T: int | None = None, qs: np.ndarray | None = None):
    """Prompt K, V of unit (b, h): ([T][128] fp16, [T][128] fp16, planted)."""
    T = cfg.T if T is None else T
    k32 = cfg.rng(_TAG_K, b, h).standard_normal((T, D), dtype=np.float32)
    k32[:, outlier_channels(cfg, b, h)] *= 8.0
    K = k32.astype(np.float16)
    V = _normal16(cfg.rng(_TAG_V, b, h), (T, D))
    planted = planted_positions(cfg, b, h)
    if len(planted):
        if qs is None:
            qs = qsel(cfg, b)
        rows = qs[h * cfg.G:(h + 1) * cfg.G].reshape(-1, D).astype(np.float64)
        m = rows.mean(axis=0)
        u = m / np.linalg.norm(m)
        boost = 4.0 * math.sqrt(D) * u
        K[planted] = (K[planted].astype(np.float64) + boost).astype(np.float16)
    return K, V, planted


def kv_full(cfg: Config, cap: int | None = None):
    """All units: K, V [B][Hkv][cap][128] fp16 (zero beyond T) and the planted
    positions [B][Hkv][k'] (k' = min(k, T - W))."""
    cap = cfg.T if cap is None else cap
    K = np.zeros((cfg.B, cfg.Hkv, cap, D), np.float16)
    V = np.zeros((cfg.B, cfg.Hkv, cap, D), np.float16)
    plist = []
    for b in range(cfg.B):
        qs = qsel(cfg, b)
        row = []
        for h in range(cfg.Hkv):
            k_, v_, p_ = unit_kv(cfg, b, h, qs=qs)
            K[b, h, :cfg.T] = k_
            V[b, h, :cfg.T] = v_
            row.append(p_)
        plist.append(row)
    planted = np.array(plist, dtype=np.int32).reshape(cfg.B, cfg.Hkv, -1)
    return K, V, planted


def step_kv(cfg: Config, step: int):
    """New K, V of one decode step: [B][Hkv][128] fp16 each (N(0,1), the
    unit's outlier channels x8, never planted)."""
    kn = np.zeros((cfg.B, cfg.Hkv, D), np.float16)
    vn = np.zeros((cfg.B, cfg.Hkv, D), np.float16)
    for b in range(cfg.B):
        for h in range(cfg.Hkv):
            k32 = cfg.rng(_TAG_KNEW, b, h, step).standard_normal(D, dtype=np.float32)
            k32[outlier_channels(cfg, b, h)] *= 8.0
            kn[b, h] = k32.astype(np.float16)
            vn[b, h] = _normal16(cfg.rng(_TAG_VNEW, b, h, step), D)
    return kn, vn
