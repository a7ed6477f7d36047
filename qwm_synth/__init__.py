"""Seeded synthetic inputs for the QuantWM KV-cache path (test and benchmark data).

This module only draws random numbers and rounds them to bf16. It holds none of
the quantizer's arithmetic, so both the CUDA path and the CPU oracle can take
their inputs from here without sharing any method code.

Workload recipe (one attention layer of a video world model, frames appended one
at a time):

* Keys, per head: a fixed set of outlier channels (chosen by a seeded
  permutation) is scaled by a constant factor, ``K = (Z + mu_f) * w`` with
  ``Z ~ N(0, 1)``.  The per-frame channel mean ``mu_f`` is 0 (tiny), i.i.d.
  ``N(0, 0.3^2)`` per channel per frame (small / 480p / 720p), or a random walk
  ``mu_f = mu_{f-1} + 0.05 N(0, 1)`` (1-minute streaming).
* Values: ``N(0, 1)``.
* Queries: tiny uses ``F G + 0.1 Z`` with a rank-4 factor; the others use
  ``alpha F W^T + beta Z`` with ``W`` a fixed orthonormal ``d x 8`` basis,
  ``alpha^2 = 10.88`` and ``beta^2 = 0.32``, so ``E|q|^2 = d`` and the top-8
  principal directions hold exactly 70 % of the Query energy.  That matches the
  concentration the QuantWM pages report (about 71 % in the first 8 principal
  directions, "Flickering after quantization?" PSAC paragraph; review Fig. 4).

Every draw comes from numpy's Philox bit generator keyed by a SeedSequence of
``(seed, kind, frame, head)``; values are drawn in fp64, rounded to fp32 and
then to bf16 (round to nearest even).  Tensors are token-major ``[n][H][d]``
bf16, returned as ``uint16`` bit patterns.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = ["LayerConfig", "CONFIGS", "get_config", "FrameSource", "f32_to_bf16_bits",
           "bf16_bits_to_f32"]


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    heads: int
    head_dim: int
    frames: int
    tokens_per_frame: int
    q_rows: int
    n_centroids: int
    group: int
    n_cand: int
    rank: int
    refresh_every: int
    seed: int
    n_outlier: int
    outlier_scale: float
    drift: str            # "none" | "iid" | "walk"
    drift_sigma: float
    query_kind: str       # "rank4" | "rank8"
    kmeans_iters: int = 10

    @property
    def total_tokens(self) -> int:
        return self.frames * self.tokens_per_frame


CONFIGS = {
    "tiny": LayerConfig("tiny", 1, 64, 2, 256, 64, 16, 16, 4, 4, 1, 0, 4, 8.0,
                        "none", 0.0, "rank4"),
    "small": LayerConfig("small", 12, 128, 9, 880, 880, 256, 32, 4, 8, 1, 1, 8, 6.0,
                         "iid", 0.3, "rank8"),
    "480p": LayerConfig("480p", 40, 128, 24, 1560, 1560, 256, 32, 4, 8, 1, 2, 8, 6.0,
                        "iid", 0.3, "rank8"),
    "720p": LayerConfig("720p", 40, 128, 21, 3600, 3600, 512, 32, 4, 8, 1, 3, 8, 6.0,
                        "iid", 0.3, "rank8"),
    "1min": LayerConfig("1min", 40, 128, 241, 1560, 1560, 512, 32, 4, 8, 8, 4, 8, 6.0,
                        "walk", 0.05, "rank8"),
}

_KIND = {"key": 1, "value": 2, "query": 3, "outlier": 4, "drift": 5, "qbasis": 6}


def get_config(name: str) -> LayerConfig:
    return CONFIGS[name]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    nan = np.isnan(x)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int, kind: str, frame: int, head: int) -> np.random.Generator:
    ss = np.random.SeedSequence([int(seed), _KIND[kind], int(frame), int(head)])
    return np.random.Generator(np.random.Philox(ss))


class FrameSource:
    """Deterministic per-frame Q/K/V for one layer configuration.

    ``frame(f)`` returns ``(Q, K, V)`` for frame ``f`` as uint16 bf16 bit arrays of
    shapes ``[q_rows][H][d]``, ``[N][H][d]`` and ``[N][H][d]``.  ``heads`` may
    restrict generation to a subset of heads (same values as the full draw).
    """

    def __init__(self, cfg: LayerConfig, seed: int | None = None):
        self.cfg = cfg
        self.seed = cfg.seed if seed is None else int(seed)
        d, H = cfg.head_dim, cfg.heads
        self._w = np.ones((H, d), dtype=np.float64)
        self._qbasis = []
        for h in range(H):
            g = _rng(self.seed, "outlier", 0, h)
            ch = g.permutation(d)[: cfg.n_outlier]
            self._w[h, ch] = cfg.outlier_scale
            gb = _rng(self.seed, "qbasis", 0, h)
            if cfg.query_kind == "rank4":
                self._qbasis.append(gb.standard_normal((4, d)))
            else:
                a = gb.standard_normal((d, 8))
                qmat, _ = np.linalg.qr(a)
                self._qbasis.append(qmat[:, :8])
        self._walk_cache = {0: np.zeros((H, d))}

    # ----- drift of the key mean --------------------------------------------------
    def _drift(self, f: int) -> np.ndarray:
        cfg = self.cfg
        H, d = cfg.heads, cfg.head_dim
        if cfg.drift == "none":
            return np.zeros((H, d))
        if cfg.drift == "iid":
            out = np.empty((H, d))
            for h in range(H):
                out[h] = cfg.drift_sigma * _rng(self.seed, "drift", f, h).standard_normal(d)
            return out
        # random walk, mu_0 = 0
        last = max(k for k in self._walk_cache if k <= f)
        mu = self._walk_cache[last].copy()
        for g in range(last + 1, f + 1):
            step = np.empty((H, d))
            for h in range(H):
                step[h] = _rng(self.seed, "drift", g, h).standard_normal(d)
            mu = mu + cfg.drift_sigma * step
            if g % 16 == 0:
                self._walk_cache[g] = mu.copy()
        return mu

    def keys(self, f: int, heads=None) -> np.ndarray:
        cfg = self.cfg
        hs = range(cfg.heads) if heads is None else heads
        mu = self._drift(f)
        n, d = cfg.tokens_per_frame, cfg.head_dim
        out = np.empty((n, len(hs), d), dtype=np.float64)
        for i, h in enumerate(hs):
            z = _rng(self.seed, "key", f, h).standard_normal((n, d))
            out[:, i, :] = (z + mu[h]) * self._w[h]
        return f32_to_bf16_bits(out.astype(np.float32))

    def values(self, f: int, heads=None) -> np.ndarray:
        cfg = self.cfg
        hs = range(cfg.heads) if heads is None else heads
        n, d = cfg.tokens_per_frame, cfg.head_dim
        out = np.empty((n, len(hs), d), dtype=np.float64)
        for i, h in enumerate(hs):
            out[:, i, :] = _rng(self.seed, "value", f, h).standard_normal((n, d))
        return f32_to_bf16_bits(out.astype(np.float32))

    def queries(self, f: int, heads=None, rows: int | None = None) -> np.ndarray:
        cfg = self.cfg
        hs = range(cfg.heads) if heads is None else heads
        n = cfg.q_rows if rows is None else rows
        d = cfg.head_dim
        out = np.empty((n, len(hs), d), dtype=np.float64)
        for i, h in enumerate(hs):
            g = _rng(self.seed, "query", f, h)
            if cfg.query_kind == "rank4":
                fct = g.standard_normal((n, 4))
                z = g.standard_normal((n, d))
                out[:, i, :] = fct @ self._qbasis[h] + 0.1 * z
            else:
                fct = g.standard_normal((n, 8))
                z = g.standard_normal((n, d))
                out[:, i, :] = (math.sqrt(10.88) * (fct @ self._qbasis[h].T)
                                + math.sqrt(0.32) * z)
        return f32_to_bf16_bits(out.astype(np.float32))

    def frame(self, f: int, heads=None):
        return self.queries(f, heads), self.keys(f, heads), self.values(f, heads)

    def query_basis(self, h: int) -> np.ndarray:
        """The planted low-rank query directions of head ``h`` (for tests)."""
        return self._qbasis[h]
