"""GPU parity at the full sizes of all five workloads, in the launch configurations the
benchmark uses, on outputs the oracle computes one by one:
- the tiny workload (2,048 positions) runs whole in test_gpu_parity.py;
- config D on its exact schedule: 32 appends of 1,024 to 32,768 positions with a
  2,048-row q8_0 ring, a decode after every append, every stored byte compared;
- the four asymmetric pairs at batch 4 x 4 KV heads x 65,536 with a bf16 ring of 1,024;
- KVarN at batch 8 x 2 KV heads x 131,072;
- the full-length cache on two seeded layers: fill 257,984, append the 4,096-row chunk,
  prefill it (rows on both sides of the window boundary and seeded random rows), then 8 of
  its (append 1 + decode) steps at 262,081..262,088, and an index-gather decode of 2,048
  positions per kv head.
Stored bytes of sampled position ranges and the whole ring are bit-exact; decode and
prefill outputs are within the stated tolerance.

Inputs: config D draws every position from the shared generator. The larger workloads use
one seeded chunk of 8,192 positions per layer from the generator; later chunks are that
chunk rolled along the positions and scaled by 1 + c/64 (chunk c), so both sides see the
same Gaussian-with-outliers data at full length without generating every value from
scratch."""
import numpy as np
import pytest

import oracle as orc
from quantized_mixed_precision_qx_b200.synth import KVRecipe, Workload
from harness import check_close, to_dev

pytestmark = pytest.mark.gpu

CH = 8192


def _chunks(wl, n, layer=0):
    base_k = wl.kv_chunk(layer, 0, CH, "k")
    base_v = wl.kv_chunk(layer, 0, CH, "v")
    t, c = 0, 0
    while t < n:
        m = min(CH, n - t)
        s = np.float32(1.0 + c / 64.0)
        k = np.ascontiguousarray(np.roll(base_k, 37 * c, axis=1)[:, :m] * s)
        v = np.ascontiguousarray(np.roll(base_v, 91 * c, axis=1)[:, :m] * s)
        yield t, k, v
        t += m
        c += 1


def _fill(g, o, wl, n, layer=0):
    vmax = 0.0
    for _, k, v in _chunks(wl, n, layer):
        g.append(layer, to_dev(k), to_dev(v))
        o.append(layer, k, v)
        vmax = max(vmax, float(np.abs(v).max()))
    return vmax


def _bytes_sampled(g, o, B, H, n, W, ranges, layer=0):
    n_main = n - min(n, W) if W else n
    for b in range(B):
        for h in range(H):
            for kv in range(2):
                for p0, cnt in ranges:
                    p0 = max(0, min(p0, n_main - cnt))
                    a = g.export(layer, b, h, kv, 0, p0, cnt)
                    r = o.export(layer, b, h, kv, 0, p0, cnt)
                    assert (a == r).all(), f"main bytes differ b={b} h={h} kv={kv} rows {p0}+{cnt}"
                if W:
                    a = g.export(layer, b, h, kv, 1, 0, min(n, W))
                    r = o.export(layer, b, h, kv, 1, 0, min(n, W))
                    assert (a == r).all(), f"ring bytes differ b={b} h={h} kv={kv}"


def test_config_d_exact_schedule():
    """Config D: 1 layer, batch 1, 4 KV heads x 256, 24 query heads, K q6_0 / V q5_0 with a
    2,048-row q8_0 ring; 32 appends of 1,024 positions (0 -> 32,768) with a decode after
    each, every decode compared, every stored byte compared at the window crossings and at
    the end."""
    from harness import append_both, compare_bytes, decode_both, make_pair
    B, H, Hq, D, W, CTX, CHUNK = 1, 4, 24, 256, 2048, 32768, 1024
    wl = Workload(1, B, H, Hq, D, CTX, KVRecipe("outlier"), seed=0)
    g, o = make_pair(wl, orc.Q6_0, orc.Q5_0, orc.Q8_0, W)
    vmax = 0.0
    for s in range(CTX // CHUNK):
        t = s * CHUNK
        vmax = max(vmax, append_both(g, o, wl, 0, t, t + CHUNK))
        if s in (0, 1, 2, 3, 15, 31):
            compare_bytes(g, o, 0, B, H, t + CHUNK, W)
        decode_both(g, o, wl, 0, s, vmax, what=f"config D step {s} n={t + CHUNK}")


def test_full_length_two_layers():
    """The full-length cache on two seeded layers: K q6_0 / V q5_0, q8_0 ring of 2,048;
    fill 257,984, append the 4,096-row chunk, prefill it, then 8 of the (append 1 + decode)
    steps. Prefill rows: the first and last, the rows on both sides of position n - W, and
    seeded random rows."""
    B, H, Hq, D, W = 1, 4, 24, 256, 2048
    n_fill, C, steps = 257984, 4096, 8
    wl = Workload(2, B, H, Hq, D, CH, KVRecipe("outlier"), seed=21)
    from quantized_mixed_precision_qx_b200.kvq import KVCache
    g = KVCache(2, B, H, Hq, D, 262144, orc.Q6_0, orc.Q5_0, orc.Q8_0, W, ws_rows=C)
    o = orc.Cache(2, B, H, Hq, D, 262144, orc.Q6_0, orc.Q5_0, orc.Q8_0, W)
    for layer in range(2):
        vmax = _fill(g, o, wl, n_fill + C, layer)
        n = n_fill + C
        _bytes_sampled(g, o, B, H, n, W, [(0, 64), (131040, 64), (n - W - 64, 64)], layer)
        q = wl.q_prefill(layer, C)
        out = g.prefill(layer, to_dev(q), 1.0).cpu().numpy()
        rand = [int(r) for r in wl.sample_indices(6, C, salt=layer)]
        rows = sorted(set([0, 1, 2047, 2048, 2049, 4094, 4095] + rand))   # chunk row 2048 is position n - W
        ref = o.prefill(layer, q, 1.0, rows=rows)
        check_close(out[:, rows], ref[:, rows], vmax, f"full-length prefill rows, layer {layer}")
        # decode steps: each appends one position (the window slides by one) and attends
        extra = Workload(2, B, H, Hq, D, steps, KVRecipe("outlier"), seed=22)
        for s in range(steps):
            k = extra.kv_chunk(layer, s, s + 1, "k")
            v = extra.kv_chunk(layer, s, s + 1, "v")
            g.append(layer, to_dev(k), to_dev(v))
            o.append(layer, k, v)
            vmax = max(vmax, float(np.abs(v).max()))
            qd = wl.q_decode(layer, s)
            check_close(g.decode(layer, to_dev(qd), 1.0).cpu().numpy(), o.decode(layer, qd, 1.0), vmax,
                        f"full-length decode layer {layer} step {s} n={n + s + 1}")
        _bytes_sampled(g, o, B, H, n + steps, W, [(n - W - 8, 16)], layer)
        # index-gather decode with the QSA budget: 2,048 seeded positions per kv head over the
        # whole context, the newest ones (in the ring) included
        import torch
        rng = np.random.default_rng(50 + layer)
        nn = n + steps
        idx = np.stack([np.concatenate([np.arange(nn - 16, nn), rng.choice(nn - 16, 2032, replace=False)])
                        for _ in range(H)])[None].astype(np.int32)
        qd = wl.q_decode(layer, 100)
        out = g.decode_indexed(layer, to_dev(qd), torch.from_numpy(idx).cuda(), 1.0).cpu().numpy()
        check_close(out, o.decode_indexed(layer, qd, idx, 1.0), vmax, f"full-length gather layer {layer}")


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


@pytest.mark.parametrize("kf,vf", [(orc.Q4_1, orc.Q4_1), (orc.Q4_1, orc.Q3_1), (orc.Q3_1, orc.Q2_1),
                                   (orc.Q2_0, orc.Q2_0)])
def test_asymmetric_full(kf, vf):
    """The asymmetric low-bit sweep with a bf16 ring of 1,024: batch 4, 4 KV heads x 256,
    24 query heads, 65,536 positions, each of its four K/V format pairs."""
    B, H, Hq, D, n, W = 4, 4, 24, 256, 65536, 1024
    wl = Workload(1, B, H, Hq, D, CH, KVRecipe("offset"), seed=23)
    from quantized_mixed_precision_qx_b200.kvq import KVCache
    g = KVCache(1, B, H, Hq, D, n, kf, vf, orc.BF16, W)
    o = orc.Cache(1, B, H, Hq, D, n, kf, vf, orc.BF16, W)
    vmax = _fill(g, o, wl, n)
    _bytes_sampled(g, o, B, H, n, W, [(0, 32), (32768, 32), (n - W - 32, 32)])
    qd = wl.q_decode(0, 0)
    check_close(g.decode(0, to_dev(qd), 1.0).cpu().numpy(), o.decode(0, qd, 1.0), vmax, "asymmetric decode")
