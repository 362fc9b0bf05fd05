"""GPU parity at the full sizes of the benchmarked workloads, in the launch configuration
the benchmark uses (appends of 8,192 positions, a 4,096-row prefill chunk, one decode),
on sampled outputs the oracle computes one by one: stored bytes of sampled position ranges
and the whole ring (bit-exact), the decode output of every query head, and the prefill
output of rows on both sides of the window boundary.

Inputs: one seeded chunk of 8,192 positions per workload from the shared generator; later
chunks are that chunk rolled along the positions and scaled by 1 + c/64 (chunk c), so both
sides see the same Gaussian-with-outliers data at full length without generating every
value from scratch."""
import numpy as np
import pytest

import oracle as orc
from quantized_mixed_precision_qx_b200.synth import KVRecipe, Workload
from harness import check_close, to_dev

pytestmark = pytest.mark.gpu

CH = 8192


def _chunks(wl, n):
    base_k = wl.kv_chunk(0, 0, CH, "k")
    base_v = wl.kv_chunk(0, 0, CH, "v")
    t, c = 0, 0
    while t < n:
        m = min(CH, n - t)
        s = np.float32(1.0 + c / 64.0)
        k = np.ascontiguousarray(np.roll(base_k, 37 * c, axis=1)[:, :m] * s)
        v = np.ascontiguousarray(np.roll(base_v, 91 * c, axis=1)[:, :m] * s)
        yield t, k, v
        t += m
        c += 1


def _fill(g, o, wl, n):
    vmax = 0.0
    for _, k, v in _chunks(wl, n):
        g.append(0, to_dev(k), to_dev(v))
        o.append(0, k, v)
        vmax = max(vmax, float(np.abs(v).max()))
    return vmax


def _bytes_sampled(g, o, B, H, n, W, ranges):
    n_main = n - min(n, W) if W else n
    for b in range(B):
        for h in range(H):
            for kv in range(2):
                for p0, cnt in ranges:
                    p0 = max(0, min(p0, n_main - cnt))
                    a = g.export(0, b, h, kv, 0, p0, cnt)
                    r = o.export(0, b, h, kv, 0, p0, cnt)
                    assert (a == r).all(), f"main bytes differ b={b} h={h} kv={kv} rows {p0}+{cnt}"
                if W:
                    a = g.export(0, b, h, kv, 1, 0, min(n, W))
                    r = o.export(0, b, h, kv, 1, 0, min(n, W))
                    assert (a == r).all(), f"ring bytes differ b={b} h={h} kv={kv}"


def test_full_length_layer():
    """One full-length layer: K q6_0 / V q5_0, q8_0 ring of 2,048; fill 257,984, a
    4,096-row chunk, prefill of the chunk, decode at 262,080."""
    B, H, Hq, D, W = 1, 4, 24, 256, 2048
    n_fill, C = 257984, 4096
    wl = Workload(1, B, H, Hq, D, CH, KVRecipe("outlier"), seed=21)
    from quantized_mixed_precision_qx_b200.kvq import KVCache
    g = KVCache(1, B, H, Hq, D, 262144, orc.Q6_0, orc.Q5_0, orc.Q8_0, W, ws_rows=C)
    o = orc.Cache(1, B, H, Hq, D, 262144, orc.Q6_0, orc.Q5_0, orc.Q8_0, W)
    vmax = _fill(g, o, wl, n_fill + C)
    n = n_fill + C
    _bytes_sampled(g, o, B, H, n, W, [(0, 64), (131040, 64), (n - W - 64, 64)])
    q = wl.q_prefill(0, C)
    out = g.prefill(0, to_dev(q), 1.0).cpu().numpy()
    rows = [0, 1, 2047, 2048, 4094, 4095]            # chunk row 2048 is position n - W
    ref = o.prefill(0, q, 1.0, rows=rows)
    check_close(out[:, rows], ref[:, rows], vmax, "full-length prefill rows")
    qd = wl.q_decode(0, 0)
    check_close(g.decode(0, to_dev(qd), 1.0).cpu().numpy(), o.decode(0, qd, 1.0), vmax, "full-length decode")


def test_kvarn_full():
    """KVarN q6_0 / V q5_0, no tail: batch 8, 2 KV heads x 256, 16 query heads, 131,072."""
    B, H, Hq, D, n = 8, 2, 16, 256, 131072
    wl = Workload(1, B, H, Hq, D, CH, KVRecipe("outlier"), seed=22)
    from quantized_mixed_precision_qx_b200.kvq import KVCache
    g = KVCache(1, B, H, Hq, D, n, orc.Q6_0, orc.Q5_0, orc.NONE, 0, kvarn=1)
    o = orc.Cache(1, B, H, Hq, D, n, orc.Q6_0, orc.Q5_0, orc.NONE, 0, kvarn=1)
    vmax = _fill(g, o, wl, n)
    _bytes_sampled(g, o, B, H, n, 0, [(0, 32), (65536, 32), (n - 32, 32)])
    qd = wl.q_decode(0, 0)
    check_close(g.decode(0, to_dev(qd), 1.0).cpu().numpy(), o.decode(0, qd, 1.0), vmax, "kvarn decode")


def test_asymmetric_full():
    """K q3_1 / V q2_1 with a bf16 ring of 1,024: batch 4, 4 KV heads x 256, 24 query
    heads, 65,536 positions."""
    B, H, Hq, D, n, W = 4, 4, 24, 256, 65536, 1024
    wl = Workload(1, B, H, Hq, D, CH, KVRecipe("offset"), seed=23)
    from quantized_mixed_precision_qx_b200.kvq import KVCache
    g = KVCache(1, B, H, Hq, D, n, orc.Q3_1, orc.Q2_1, orc.BF16, W)
    o = orc.Cache(1, B, H, Hq, D, n, orc.Q3_1, orc.Q2_1, orc.BF16, W)
    vmax = _fill(g, o, wl, n)
    _bytes_sampled(g, o, B, H, n, W, [(0, 32), (32768, 32), (n - W - 32, 32)])
    qd = wl.q_decode(0, 0)
    check_close(g.decode(0, to_dev(qd), 1.0).cpu().numpy(), o.decode(0, qd, 1.0), vmax, "asymmetric decode")
