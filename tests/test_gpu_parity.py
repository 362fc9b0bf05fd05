"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on the
same seeded inputs. Codes, scales and mins bit-exact; attention within the stated
tolerance (see tests/harness.py). Shapes follow the five workloads at sizes the
oracle finishes in seconds, spanning several tiles with ragged tails, plus every
format x tail x KVarN combination on small shapes.
"""
import numpy as np
import pytest

import oracle as orc
from quantized_mixed_precision_qx_b200.synth import KVRecipe, Workload
from harness import append_both, check_close, compare_bytes, decode_both, make_pair, to_dev

pytestmark = pytest.mark.gpu


def test_tiny_q8_workload():
    """1 layer, batch 1, 1 KV head x 128, 4 query heads, 2,048 tokens of q8_0."""
    wl = Workload(1, 1, 1, 4, 128, 2048, KVRecipe("iid"), seed=0)
    g, o = make_pair(wl, orc.Q8_0, orc.Q8_0)
    vmax = append_both(g, o, wl, 0, 0, 2048)
    compare_bytes(g, o, 0, 1, 1, 2048, 0)
    q = wl.q_decode(0, 0) * np.float32(1.0)
    decode_both(g, o, wl, 0, 0, vmax, what="tiny")


def test_config_d_schedule_scaled():
    """K q6_0 / V q5_0 with a q8_0 ring, grown by ragged appends, decode after each."""
    W = 256
    wl = Workload(1, 1, 4, 24, 256, 1500, KVRecipe("outlier"), seed=1)
    g, o = make_pair(wl, orc.Q6_0, orc.Q5_0, orc.Q8_0, W)
    t, vmax = 0, 0.0
    for step, c in enumerate([100, 1, 200, 300, 57, 1, 512, 329]):
        vmax = max(vmax, append_both(g, o, wl, 0, t, t + c))
        t += c
        compare_bytes(g, o, 0, 1, 4, t, W)
        decode_both(g, o, wl, 0, step, vmax, what=f"step {step} n={t}")


@pytest.mark.parametrize("kf,vf", [(orc.Q4_1, orc.Q4_1), (orc.Q4_1, orc.Q3_1), (orc.Q3_1, orc.Q2_1),
                                   (orc.Q2_0, orc.Q2_0)])
def test_asymmetric_sweep_scaled(kf, vf):
    W = 128
    wl = Workload(1, 4, 4, 24, 256, 1200, KVRecipe("offset"), seed=2)
    g, o = make_pair(wl, kf, vf, orc.BF16, W)
    vmax = append_both(g, o, wl, 0, 0, 700)
    vmax = max(vmax, append_both(g, o, wl, 0, 700, 1200))
    compare_bytes(g, o, 0, 4, 4, 1200, W)
    decode_both(g, o, wl, 0, 0, vmax, what="sweep")


def test_kvarn_scaled():
    wl = Workload(1, 8, 2, 16, 256, 1300, KVRecipe("outlier"), seed=3)
    g, o = make_pair(wl, orc.Q6_0, orc.Q5_0, kvarn=1)
    vmax = append_both(g, o, wl, 0, 0, 600)
    vmax = max(vmax, append_both(g, o, wl, 0, 600, 1300))
    sK_ref, sV_ref = o.channel_scales(0)
    compare_bytes(g, o, 0, 8, 2, 1300, 0)
    decode_both(g, o, wl, 0, 0, vmax, what="kvarn")


def test_prefill_scaled():
    """Chunked prefill over the post-append cache, causal, rows on both sides of n - W."""
    W = 128
    wl = Workload(2, 1, 4, 24, 256, 900, KVRecipe("outlier"), seed=4)
    g, o = make_pair(wl, orc.Q6_0, orc.Q5_0, orc.Q8_0, W)
    for layer in range(2):
        vmax = append_both(g, o, wl, layer, 0, 700)
        vmax = max(vmax, append_both(g, o, wl, layer, 700, 900))
        q = wl.q_prefill(layer, 200)
        out = g.prefill(layer, to_dev(q), 1.0).cpu().numpy()
        ref = o.prefill(layer, q, 1.0)
        check_close(out, ref, vmax, f"prefill layer {layer}")
        compare_bytes(g, o, layer, 1, 4, 900, W)
        decode_both(g, o, wl, layer, 0, vmax, what="after prefill")


FORMATS = list(range(12))


@pytest.mark.parametrize("tail", [orc.NONE, orc.Q8_0, orc.BF16, orc.F16])
@pytest.mark.parametrize("D", [32, 64, 128, 256])
def test_all_formats(tail, D):
    """Every low-bit format as K (and the next one as V), each tail format, each head
    dim; with and without KVarN; appends of 1, 31, and a chunk longer than W."""
    W = 0 if tail == orc.NONE else 40
    for kf in FORMATS:
        vf = FORMATS[(kf + 5) % 12]
        for kvarn in (0, 1):
            T = 700 if kvarn else 170
            wl = Workload(1, 2, 2, 6, D, T, KVRecipe("offset" if kf % 2 else "outlier"), seed=10 + kf)
            g, o = make_pair(wl, kf, vf, tail, W, kvarn=kvarn, calib=64)
            chunks = [T - 32, 1, 31] if kvarn else [1, 31, 100, 38]
            t, vmax = 0, 0.0
            for c in chunks:
                vmax = max(vmax, append_both(g, o, wl, 0, t, t + c))
                t += c
            compare_bytes(g, o, 0, 2, 2, t, W)
            decode_both(g, o, wl, 0, kf, vmax, scale=0.9, what=f"kf={kf} vf={vf} tail={tail} D={D} kvarn={kvarn}")


def test_chunk_invariance_gpu():
    W = 64
    wl = Workload(1, 1, 2, 4, 128, 400, KVRecipe("outlier"), seed=5)
    blobs = []
    for chunks in ([1] * 80 + [320], [7] * 57 + [1], [64, 336], [400]):
        from quantized_mixed_precision_qx_b200.kvq import KVCache
        g = KVCache(1, 1, 2, 4, 128, 400, orc.Q5_1, orc.Q3_0, orc.Q8_0, W)
        t = 0
        for c in chunks:
            g.append(0, to_dev(wl.kv_chunk(0, t, t + c, "k")), to_dev(wl.kv_chunk(0, t, t + c, "v")))
            t += c
        blobs.append(np.concatenate([g.export(0, 0, h, kv, r, 0, (400 - W) if r == 0 else W)
                                     for h in range(2) for kv in range(2) for r in range(2)]))
    for b in blobs[1:]:
        assert (b == blobs[0]).all()


def test_decode_is_deterministic():
    import torch
    wl = Workload(1, 2, 4, 24, 256, 3000, KVRecipe("outlier"), seed=6)
    from quantized_mixed_precision_qx_b200.kvq import KVCache
    g = KVCache(1, 2, 4, 24, 256, 3000, orc.Q6_0, orc.Q5_0, orc.Q8_0, 512)
    g.append(0, to_dev(wl.kv_chunk(0, 0, 3000, "k")), to_dev(wl.kv_chunk(0, 0, 3000, "v")))
    q = to_dev(wl.q_decode(0, 0))
    a = g.decode(0, q).clone()
    for _ in range(3):
        assert torch.equal(g.decode(0, q), a)


def test_error_paths_gpu():
    import torch
    from quantized_mixed_precision_qx_b200 import kvq
    g = kvq.KVCache(1, 1, 2, 4, 64, 32, orc.Q4_0, orc.Q4_0)
    q = torch.zeros(1, 4, 64, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        g.decode(0, q)
    assert e.value.status == kvq.ERR_EMPTY
    k = torch.zeros(1, 40, 2, 64, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        g.append(0, k, k)
    assert e.value.status == kvq.ERR_CAPACITY and g.length(0) == 0
    k = torch.zeros(1, 8, 2, 64 + 1, device="cuda")[..., 1:]
    kk = k.contiguous()
    mis = torch.zeros(1 * 8 * 2 * 64 + 1, device="cuda")[1:].view(1, 8, 2, 64)
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_append(g.handle, 0, mis, kk, 8)
    assert e.value.status == kvq.ERR_ALIGNMENT and g.length(0) == 0
    gk = kvq.KVCache(1, 1, 2, 4, 64, 2048, orc.Q4_0, orc.Q4_0, kvarn=1)
    k = torch.zeros(1, 100, 2, 64, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        gk.append(0, k, k)
    assert e.value.status == kvq.ERR_CALIBRATION and gk.length(0) == 0
    # decode with a too-small workspace
    g.append(0, torch.zeros(1, 4, 2, 64, device="cuda"), torch.zeros(1, 4, 2, 64, device="cuda"))
    out = torch.empty_like(q)
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_decode_attention(g.handle, 0, q, 1.0, out, g.ws, 4)
    assert e.value.status == kvq.ERR_CAPACITY


@pytest.mark.parametrize("D", [128, 256])
@pytest.mark.parametrize("tail,W", [(orc.NONE, 0), (orc.Q8_0, 96), (orc.BF16, 40), (orc.F16, 300)])
def test_prefill_formats(D, tail, W):
    """Tensor-core prefill: chunks longer and shorter than the window, ragged row
    counts (C * G not a multiple of 128), symmetric and asymmetric formats, KVarN."""
    for kf, vf, kvarn, G in [(orc.Q6_0, orc.Q5_0, 0, 6), (orc.Q4_1, orc.Q3_1, 0, 8), (orc.Q8_0, orc.Q2_1, 1, 3),
                             (orc.Q5_1, orc.Q8_1, 0, 1)]:
        H = 2
        T = 700
        wl = Workload(1, 1, H, H * G, D, T, KVRecipe("outlier" if kf % 2 == 0 else "offset"), seed=40 + kf)
        g, o = make_pair(wl, kf, vf, tail, W, kvarn=kvarn, calib=64)
        vmax = append_both(g, o, wl, 0, 0, 517)
        vmax = max(vmax, append_both(g, o, wl, 0, 517, T))
        C = T - 517
        q = wl.q_prefill(0, C)
        out = g.prefill(0, to_dev(q), 0.75).cpu().numpy()
        ref = o.prefill(0, q, 0.75)
        check_close(out, ref, vmax, f"prefill kf={kf} vf={vf} tail={tail} W={W} D={D} kvarn={kvarn}")


@pytest.mark.parametrize("tail,W", [(orc.NONE, 0), (orc.Q8_0, 8)])
def test_append_half_step_ties(tail, W):
    """Values placed exactly on code half-steps (x / d = k + 1/2, and (x - m) / d = k + 1/2
    for qX_1): the quantizer must round them away from zero exactly as the oracle's IEEE
    division does, for every format (the kernel's division-free path falls back to a true
    division next to half-steps)."""
    import torch
    from quantized_mixed_precision_qx_b200.kvq import KVCache
    rng = np.random.default_rng(77)
    T, H, D = 40, 1, 64
    for f in range(12):
        X = orc.fmt_bits(f)
        d = np.float32(2.0 ** -5)
        x = np.empty((1, T, H, D), np.float32)
        for t in range(T):
            for blk in range(D // 32):
                if orc.fmt_asym(f):
                    umax = (1 << X) - 1
                    m = np.float32(-0.375)
                    k = rng.integers(0, umax, 32).astype(np.float32)
                    vals = m + (k + np.float32(0.5)) * d
                    vals[0] = m                       # min -> m exactly
                    vals[1] = m + umax * d            # max -> d = (max - min) / umax exactly
                else:
                    qmax = (1 << (X - 1)) - 1
                    k = rng.integers(-qmax, qmax, 32).astype(np.float32)
                    vals = (k + np.float32(0.5)) * d
                    vals[0] = qmax * d                # absmax -> d exactly
                x[0, t, 0, 32 * blk:32 * blk + 32] = vals.astype(np.float32)
        g = KVCache(1, 1, H, 2, D, T, f, f, tail, W)
        o = orc.Cache(1, 1, H, 2, D, T, f, f, tail, W)
        g.append(0, torch.from_numpy(x).cuda(), torch.from_numpy(x).cuda())
        o.append(0, x, x)
        compare_bytes(g, o, 0, 1, H, T, W)


@pytest.mark.parametrize("D", [128, 256])
def test_multi_query_chunks(D):
    """Multi-query verification (a few draft tokens appended, then attended causally): chunks
    of 1, 2 and 8 rows through the prefill entry point, the window boundary inside the cache."""
    W = 96
    wl = Workload(1, 1, 2, 12, D, 1200, KVRecipe("outlier"), seed=60)
    g, o = make_pair(wl, orc.Q6_0, orc.Q5_0, orc.Q8_0, W)
    vmax = append_both(g, o, wl, 0, 0, 1189)
    t = 1189
    for cid, C in enumerate([1, 2, 8]):
        vmax = max(vmax, append_both(g, o, wl, 0, t, t + C))
        t += C
        q = wl.q_prefill(0, C, chunk_id=cid)
        out = g.prefill(0, to_dev(q), 1.0).cpu().numpy()
        ref = o.prefill(0, q, 1.0)
        check_close(out, ref, vmax, f"multi-query C={C} D={D}")
