"""Seeded synthetic inputs for the quantized KV cache path.

This module holds no quantization or attention arithmetic: it only draws the
fp32 K, V and q tensors that both the CUDA path and the CPU oracle consume.
Every value is a pure function of (seed, tensor id, flat index), so any slice
of a tensor can be regenerated on its own:

    bits(seed, tid, j) = mix64(mix64(mix64(seed) + tid) + j)
    u(j)               = ((bits >> 11) + 0.5) * 2**-53            in (0, 1)
    z(i)               = sqrt(-2 ln u(2i)) * cos(2 pi u(2i+1))    (Box-Muller)

mix64 is the SplitMix64 step (add the golden-ratio increment, then the
xor-shift-multiply finaliser), all in wrapping uint64 arithmetic. The normal
draw is done in float64 and rounded once to float32.

Tensor shapes follow the cache's input layout: K and V are [layer][batch]
[token][kv_head][head_dim], q is [batch][q_head][head_dim] (decode) or
[batch][row][q_head][head_dim] (prefill). Flat indices are taken over the
full-length tensor of a workload, so a chunk of tokens [t0, t1) always gets the
same numbers whatever the chunking.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# tensor ids
TID_K = 1
TID_V = 2
TID_Q_DECODE = 3
TID_Q_PREFILL = 4
TID_OUTLIER = 5
TID_OFFSET = 6
TID_SAMPLE = 7


def _mix64(x: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = x + _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def _key(seed: int, tid: int) -> np.uint64:
    s = _mix64(np.array([seed], dtype=np.uint64))
    with np.errstate(over="ignore"):
        k = _mix64(s + np.uint64(tid))
    return k[0]


def bits(seed: int, tid: int, j: np.ndarray) -> np.ndarray:
    """64-bit counter-based draw for integer counters j (uint64 array)."""
    with np.errstate(over="ignore"):
        return _mix64(_key(seed, tid) + j.astype(np.uint64))


def uniform(seed: int, tid: int, j: np.ndarray) -> np.ndarray:
    b = bits(seed, tid, j)
    return ((b >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(seed: int, tid: int, idx: np.ndarray) -> np.ndarray:
    """Standard normal (float64) at flat indices idx."""
    idx = idx.astype(np.uint64)
    u1 = uniform(seed, tid, idx * np.uint64(2))
    u2 = uniform(seed, tid, idx * np.uint64(2) + np.uint64(1))
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def normal_range(seed: int, tid: int, start: int, count: int) -> np.ndarray:
    return normal(seed, tid, np.arange(start, start + count, dtype=np.uint64))


@dataclass
class KVRecipe:
    """Distribution of the K/V inputs of one workload.

    kind: "iid"      K, V ~ N(0,1)
          "outlier"  K ~ N(0,1) with `n_outliers` seeded channels per
                     (layer, kv head) multiplied by `outlier_scale`; V ~ N(0,1)
          "offset"   K ~ N(0,1) + a per-(layer, kv head, channel) constant drawn
                     from N(0, offset_std^2); V ~ N(0,1)
    """
    kind: str = "iid"
    n_outliers: int = 8
    outlier_scale: float = 8.0
    offset_std: float = 0.5


@dataclass
class Workload:
    n_layers: int
    batch: int
    n_kv_heads: int
    n_q_heads: int
    head_dim: int
    total_tokens: int          # full context length the inputs span
    recipe: KVRecipe = field(default_factory=KVRecipe)
    seed: int = 0

    # -- per-(layer, head) structure --------------------------------------
    def outlier_channels(self, layer: int, h: int) -> np.ndarray:
        D = self.head_dim
        base = (layer * self.n_kv_heads + h) * D
        keys = bits(self.seed, TID_OUTLIER, np.arange(base, base + D, dtype=np.uint64))
        order = np.argsort(keys, kind="stable")
        return np.sort(order[: self.recipe.n_outliers])

    def channel_offsets(self, layer: int, h: int) -> np.ndarray:
        D = self.head_dim
        base = (layer * self.n_kv_heads + h) * D
        return self.recipe.offset_std * normal_range(self.seed, TID_OFFSET, base, D)

    def _k_modifier(self, layer: int):
        """(scale[H][D], offset[H][D]) applied to the N(0,1) K draw."""
        H, D = self.n_kv_heads, self.head_dim
        scale = np.ones((H, D), dtype=np.float64)
        offset = np.zeros((H, D), dtype=np.float64)
        if self.recipe.kind == "outlier":
            for h in range(H):
                scale[h, self.outlier_channels(layer, h)] = self.recipe.outlier_scale
        elif self.recipe.kind == "offset":
            for h in range(H):
                offset[h] = self.channel_offsets(layer, h)
        elif self.recipe.kind != "iid":
            raise ValueError(self.recipe.kind)
        return scale, offset

    # -- K / V ------------------------------------------------------------
    def kv_chunk(self, layer: int, t0: int, t1: int, which: str, b0: int = 0, b1: int | None = None):
        """fp32 array [b1-b0][t1-t0][H][D] of K ('k') or V ('v')."""
        if b1 is None:
            b1 = self.batch
        H, D, T = self.n_kv_heads, self.head_dim, self.total_tokens
        assert 0 <= t0 <= t1 <= T
        tid = TID_K if which == "k" else TID_V
        n = t1 - t0
        out = np.empty((b1 - b0, n, H, D), dtype=np.float32)
        if n == 0:
            return out
        if which == "k":
            scale, offset = self._k_modifier(layer)
        for bi, b in enumerate(range(b0, b1)):
            start = ((layer * self.batch + b) * T + t0) * H * D
            z = normal_range(self.seed, tid, start, n * H * D).reshape(n, H, D)
            if which == "k":
                z = z * scale[None] + offset[None]
            out[bi] = z.astype(np.float32)
        return out

    def kv_rows(self, layer: int, b: int, h: int, t0: int, t1: int, which: str) -> np.ndarray:
        """fp32 [t1-t0][D] rows of one (batch, kv head); same numbers as kv_chunk."""
        H, D, T = self.n_kv_heads, self.head_dim, self.total_tokens
        tid = TID_K if which == "k" else TID_V
        t = np.arange(t0, t1, dtype=np.uint64)[:, None]
        c = np.arange(D, dtype=np.uint64)[None, :]
        idx = ((np.uint64(layer * self.batch + b) * np.uint64(T) + t) * np.uint64(H) + np.uint64(h)) * np.uint64(D) + c
        z = normal(self.seed, tid, idx.reshape(-1)).reshape(t1 - t0, D)
        if which == "k":
            scale, offset = self._k_modifier(layer)
            z = z * scale[h][None] + offset[h][None]
        return z.astype(np.float32)

    # -- queries -----------------------------------------------------------
    def q_decode(self, layer: int, step: int) -> np.ndarray:
        """fp32 [B][Hq][D], N(0,1)/sqrt(D)."""
        B, Hq, D = self.batch, self.n_q_heads, self.head_dim
        n = B * Hq * D
        start = (layer * (1 << 20) + step) * n
        z = normal_range(self.seed, TID_Q_DECODE, start, n) / math.sqrt(D)
        return z.astype(np.float32).reshape(B, Hq, D)

    def q_prefill(self, layer: int, n_chunk: int, chunk_id: int = 0) -> np.ndarray:
        """fp32 [B][n_chunk][Hq][D], N(0,1)/sqrt(D)."""
        B, Hq, D = self.batch, self.n_q_heads, self.head_dim
        n = B * n_chunk * Hq * D
        start = (layer * (1 << 16) + chunk_id) * (1 << 32)
        z = normal_range(self.seed, TID_Q_PREFILL, start, n) / math.sqrt(D)
        return z.astype(np.float32).reshape(B, n_chunk, Hq, D)

    def sample_indices(self, count: int, upper: int, salt: int = 0) -> np.ndarray:
        """`count` distinct seeded indices in [0, upper), sorted."""
        keys = bits(self.seed, TID_SAMPLE, np.arange(upper, dtype=np.uint64) + np.uint64(salt) * np.uint64(1 << 40))
        return np.sort(np.argsort(keys, kind="stable")[: min(count, upper)])
