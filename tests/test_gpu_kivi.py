"""GPU parity of per-channel (token-axis) K blocks against the oracle: the group blocks and
the pending rows bit for bit, the ring and the V rows bit for bit, decode, prefill and the
index-gather decode within the stated tolerance; formats with and without a ring (window
sizes that are and are not multiples of 32), head dims 64, 128 and 256, appends of 1, 31,
33 and thousands of positions (several groups completed by one append), chunk invariance,
and a larger cache of 4 KV heads x 256 at 40,000 positions."""
import numpy as np
import pytest

import oracle as orc
from quantized_mixed_precision_qx_b200.synth import KVRecipe, Workload
from harness import check_close, to_dev

pytestmark = pytest.mark.gpu


def _pair(wl, kf, vf, tail, W, max_ctx=None):
    from quantized_mixed_precision_qx_b200.kvq import KVCache
    max_ctx = max_ctx or wl.total_tokens
    g = KVCache(wl.n_layers, wl.batch, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, max_ctx, kf, vf, tail, W,
                k_per_channel=1)
    o = orc.Cache(wl.n_layers, wl.batch, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, max_ctx, kf, vf, tail, W, kivi=1)
    return g, o


def _compare_store(g, o, B, H, n, W):
    entered = max(0, n - W) if W else n
    G, P = entered // 32, entered % 32
    for b in range(B):
        for h in range(H):
            if G:
                a, r = g.export(0, b, h, 0, 0, 0, G), o.export(0, b, h, 0, 0, 0, G)
                assert np.array_equal(a, r), f"K groups differ b={b} h={h}"
            if P:
                a, r = g.export(0, b, h, 0, 2, 0, P), o.export(0, b, h, 0, 2, 0, P)
                assert np.array_equal(a, r), f"K pending rows differ b={b} h={h}"
            if entered:
                a, r = g.export(0, b, h, 1, 0, 0, entered), o.export(0, b, h, 1, 0, 0, entered)
                assert np.array_equal(a, r), f"V rows differ b={b} h={h}"
            if W:
                for kv in range(2):
                    a, r = g.export(0, b, h, kv, 1, 0, min(n, W)), o.export(0, b, h, kv, 1, 0, min(n, W))
                    assert np.array_equal(a, r), f"ring differs b={b} h={h} kv={kv}"


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("kf,vf,tail,W", [(orc.Q5_0, orc.Q5_0, orc.NONE, 0), (orc.Q4_1, orc.Q3_1, orc.NONE, 0),
                                          (orc.Q6_0, orc.Q5_0, orc.Q8_0, 64), (orc.Q3_1, orc.Q4_0, orc.BF16, 40),
                                          (orc.Q8_0, orc.Q8_1, orc.F16, 100), (orc.Q2_0, orc.Q6_1, orc.NONE, 0)])
def test_per_channel_k(D, kf, vf, tail, W):
    T = 900
    wl = Workload(1, 2, 2, 12, D, T, KVRecipe("outlier" if kf % 2 == 0 else "offset"), seed=120 + kf)
    g, o = _pair(wl, kf, vf, tail, W)
    t, vmax = 0, 0.0
    for step, c in enumerate([1, 31, 33, 300, 5, 530]):
        k, v = wl.kv_chunk(0, t, t + c, "k"), wl.kv_chunk(0, t, t + c, "v")
        g.append(0, to_dev(k), to_dev(v))
        o.append(0, k, v)
        vmax = max(vmax, float(np.abs(v).max()))
        t += c
        _compare_store(g, o, 2, 2, t, W)
        q = wl.q_decode(0, step)
        check_close(g.decode(0, to_dev(q), 0.8).cpu().numpy(), o.decode(0, q, 0.8), vmax,
                    f"per-channel K decode n={t} D={D} kf={kf} tail={tail}")
    C = 120
    qp = wl.q_prefill(0, C)
    check_close(g.prefill(0, to_dev(qp), 0.8).cpu().numpy(), o.prefill(0, qp, 0.8), vmax,
                f"per-channel K prefill D={D} kf={kf} tail={tail}")
    import torch
    rng = np.random.default_rng(D)
    idx = np.stack([np.stack([rng.choice(T, 300, replace=False) for _ in range(2)]) for _ in range(2)]).astype(np.int32)
    q = wl.q_decode(0, 99)
    check_close(g.decode_indexed(0, to_dev(q), torch.from_numpy(idx).cuda(), 0.8).cpu().numpy(),
                o.decode_indexed(0, q, idx, 0.8), vmax, f"per-channel K gather D={D} kf={kf} tail={tail}")


def test_per_channel_k_chunk_invariance():
    from quantized_mixed_precision_qx_b200.kvq import KVCache
    T, W = 500, 96
    wl = Workload(1, 1, 2, 4, 128, T, KVRecipe("outlier"), seed=130)
    blobs = []
    for chunks in ([1] * 70 + [430], [7] * 71 + [3], [64, 436], [500]):
        g = KVCache(1, 1, 2, 4, 128, T, orc.Q5_1, orc.Q3_0, orc.Q8_0, W, k_per_channel=1)
        t = 0
        for c in chunks:
            g.append(0, to_dev(wl.kv_chunk(0, t, t + c, "k")), to_dev(wl.kv_chunk(0, t, t + c, "v")))
            t += c
        entered = T - W
        blobs.append(np.concatenate([g.export(0, 0, h, 0, 0, 0, entered // 32) for h in range(2)] +
                                    [g.export(0, 0, h, 0, 2, 0, entered % 32) for h in range(2)] +
                                    [g.export(0, 0, h, kv, 1, 0, W) for h in range(2) for kv in range(2)]))
    for b in blobs[1:]:
        assert np.array_equal(b, blobs[0])


def test_per_channel_k_larger_cache():
    """4 KV heads x 256, 24 query heads, 40,000 positions in appends of 8,192, K q5_0 per
    channel, V q5_0, without a window (the setting where the pages found it helps)."""
    T = 40000
    wl = Workload(1, 1, 4, 24, 256, T, KVRecipe("outlier"), seed=131)
    g, o = _pair(wl, orc.Q5_0, orc.Q5_0, orc.NONE, 0)
    vmax = 0.0
    for t in range(0, T, 8192):
        c = min(8192, T - t)
        k, v = wl.kv_chunk(0, t, t + c, "k"), wl.kv_chunk(0, t, t + c, "v")
        g.append(0, to_dev(k), to_dev(v))
        o.append(0, k, v)
        vmax = max(vmax, float(np.abs(v).max()))
    _compare_store(g, o, 1, 4, T, 0)
    q = wl.q_decode(0, 0)
    check_close(g.decode(0, to_dev(q), 1.0).cpu().numpy(), o.decode(0, q, 1.0), vmax, "per-channel K at 40,000")
