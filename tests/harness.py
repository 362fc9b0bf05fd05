"""Shared helpers of the parity tests: run the same seeded schedule through the
CUDA library (via its C ABI binding) and through the CPU oracle, and compare.

Tolerance (attention outputs, whole output tensor of one call):
    ||gpu - oracle||_2 / ||oracle||_2 <= 1e-4   and   max|gpu - oracle| <= 1e-3 * max|V|
with max|V| over the layer's raw float32 V input. Stored codes, scales and mins
are compared byte for byte through the canonical export.
"""
from __future__ import annotations

import numpy as np

import oracle as orc
from quantized_mixed_precision_qx_b200.synth import KVRecipe, Workload

REL_L2 = 1e-4
MAX_ABS_FRAC = 1e-3


def check_close(gpu: np.ndarray, ref: np.ndarray, vmax: float, what: str = ""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    diff = gpu - ref
    rel = np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-30)
    mx = np.abs(diff).max()
    assert rel <= REL_L2, f"{what}: relative L2 {rel:.3e} > {REL_L2}"
    assert mx <= MAX_ABS_FRAC * vmax, f"{what}: max abs {mx:.3e} > {MAX_ABS_FRAC} * {vmax:.3e}"
    return rel, mx


def make_pair(wl: Workload, k_fmt, v_fmt, tail_fmt=orc.NONE, W=0, kvarn=0, max_ctx=None, calib=512):
    import torch
    from quantized_mixed_precision_qx_b200.kvq import KVCache
    max_ctx = max_ctx or wl.total_tokens
    g = KVCache(wl.n_layers, wl.batch, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, max_ctx, k_fmt, v_fmt,
                tail_fmt, W, kvarn=kvarn, calib=calib)
    o = orc.Cache(wl.n_layers, wl.batch, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, max_ctx, k_fmt, v_fmt,
                  tail_fmt, W, kvarn=kvarn, calib=calib)
    return g, o


def to_dev(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def append_both(g, o, wl: Workload, layer: int, t0: int, t1: int):
    k = wl.kv_chunk(layer, t0, t1, "k")
    v = wl.kv_chunk(layer, t0, t1, "v")
    g.append(layer, to_dev(k), to_dev(v))
    o.append(layer, k, v)
    return float(np.abs(v).max()) if v.size else 0.0


def compare_bytes(g, o, layer: int, B: int, H: int, n: int, W: int):
    """Every stored byte of the layer that the oracle defines: low-bit rows [0, n - W)
    (all rows written so far) and every ring slot."""
    n_main = n - min(n, W) if W else n
    for b in range(B):
        for h in range(H):
            for kv in range(2):
                if n_main:
                    a = g.export(layer, b, h, kv, 0, 0, n_main)
                    r = o.export(layer, b, h, kv, 0, 0, n_main)
                    if not (a == r).all():
                        bad = np.nonzero(a != r)[0][:8]
                        raise AssertionError(f"main bytes differ (b={b} h={h} kv={kv}) at {bad}: {a[bad]} vs {r[bad]}")
                if W:
                    slots = min(n, W)
                    a = g.export(layer, b, h, kv, 1, 0, slots)
                    r = o.export(layer, b, h, kv, 1, 0, slots)
                    if not (a == r).all():
                        bad = np.nonzero(a != r)[0][:8]
                        raise AssertionError(f"ring bytes differ (b={b} h={h} kv={kv}) at {bad}: {a[bad]} vs {r[bad]}")


def decode_both(g, o, wl: Workload, layer: int, step: int, vmax: float, scale: float = 1.0, what=""):
    q = wl.q_decode(layer, step)
    out = g.decode(layer, to_dev(q), scale).cpu().numpy()
    ref = o.decode(layer, q, scale)
    return check_close(out, ref, vmax, what)
