"""Pins of the oracle's cache (ring, requantization, KVarN) and attention.

Attention is checked against torch's scaled_dot_product_attention run in float64
on the CPU (an independent library routine, with its own GQA grouping and causal
masking) on the rows the oracle says it stored; plus exact special cases (one
token, identical keys, zero query), the tail identity of "Hard numbers on
Qwen3.8-27B's KV cache" (section "KV cache low-bit storage": with context below
the window the output equals the 8-bit cache's), the lossless q8_0 -> q8_0
eviction, chunk invariance and the KVarN closed form.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as orc
from quantized_mixed_precision_qx_b200.synth import KVRecipe, Workload


def _wl(B=1, H=2, Hq=4, D=64, T=96, kind="iid", seed=0):
    return Workload(n_layers=1, batch=B, n_kv_heads=H, n_q_heads=Hq, head_dim=D,
                    total_tokens=T, recipe=KVRecipe(kind=kind), seed=seed)


def _fill(cache, wl, chunks):
    t = 0
    for c in chunks:
        cache.append(0, wl.kv_chunk(0, t, t + c, "k"), wl.kv_chunk(0, t, t + c, "v"))
        t += c
    return t


def _stored(cache, B, H, n):
    """Dequantized K and V rows as the oracle's attention reads them: [B][H][n][D]."""
    K = np.stack([np.stack([np.stack([cache.position_row(0, b, h, 0, t) for t in range(n)])
                            for h in range(H)]) for b in range(B)])
    V = np.stack([np.stack([np.stack([cache.position_row(0, b, h, 1, t) for t in range(n)])
                            for h in range(H)]) for b in range(B)])
    return K, V


def _sdpa(q, K, V, scale, causal_rows=None):
    """q [B][Hq][R][D], K/V [B][H][n][D] -> [B][Hq][R][D] in float64 via torch."""
    qt = torch.from_numpy(q.astype(np.float64))
    Kt = torch.from_numpy(K.astype(np.float64))
    Vt = torch.from_numpy(V.astype(np.float64))
    mask = None
    if causal_rows is not None:
        n = K.shape[2]
        pos = torch.as_tensor(causal_rows)[:, None]
        mask = torch.arange(n)[None, :] <= pos
    return F.scaled_dot_product_attention(qt, Kt, Vt, attn_mask=mask, scale=scale, enable_gqa=True).numpy()


@pytest.mark.parametrize("kf,vf,tf,W", [
    (orc.Q8_0, orc.Q8_0, orc.NONE, 0),
    (orc.Q6_0, orc.Q5_0, orc.Q8_0, 32),
    (orc.Q4_1, orc.Q3_1, orc.BF16, 16),
    (orc.Q2_0, orc.Q2_0, orc.F16, 40),
    (orc.Q3_1, orc.Q2_1, orc.BF16, 8),
])
def test_decode_matches_library_attention(kf, vf, tf, W):
    wl = _wl(B=2, H=2, Hq=6, D=64, T=90, kind="outlier")
    c = orc.Cache(1, 2, 2, 6, 64, 128, kf, vf, tf, W)
    n = _fill(c, wl, [50, 3, 37])
    K, V = _stored(c, 2, 2, n)
    q = wl.q_decode(0, 0)
    out = c.decode(0, q, scale=1.0)
    ref = _sdpa(q[:, :, None, :], K, V, 1.0)[:, :, 0, :]
    np.testing.assert_allclose(out, ref, rtol=1e-6, atol=1e-7)


def test_prefill_matches_library_attention():
    wl = _wl(B=1, H=2, Hq=4, D=64, T=80, kind="offset")
    c = orc.Cache(1, 1, 2, 4, 64, 128, orc.Q6_0, orc.Q5_0, orc.Q8_0, 24)
    _fill(c, wl, [40])
    C = 40
    c.append(0, wl.kv_chunk(0, 40, 80, "k"), wl.kv_chunk(0, 40, 80, "v"))
    n = 80
    K, V = _stored(c, 1, 2, n)
    q = wl.q_prefill(0, C)                                   # [B][C][Hq][D]
    out = c.prefill(0, q, scale=0.7)
    rows = np.arange(n - C, n)
    ref = _sdpa(q.transpose(0, 2, 1, 3), K, V, 0.7, causal_rows=rows).transpose(0, 2, 1, 3)
    np.testing.assert_allclose(out, ref, rtol=1e-6, atol=1e-7)
    # the last chunk row sees the whole cache: same as decode with that query
    dec = c.decode(0, np.ascontiguousarray(q[:, -1]), scale=0.7)
    assert (dec == out[:, -1]).all()
    # a row subset computes exactly those rows
    sub = c.prefill(0, q, scale=0.7, rows=[0, 17, 39])
    assert (sub[:, [0, 17, 39]] == out[:, [0, 17, 39]]).all()
    assert (sub[:, 1] == 0).all()


def test_single_token_returns_its_value():
    wl = _wl(T=1)
    for kf, vf in [(orc.Q4_0, orc.Q5_1), (orc.Q2_1, orc.Q8_0)]:
        c = orc.Cache(1, 1, 2, 4, 64, 8, kf, vf)
        _fill(c, wl, [1])
        out = c.decode(0, wl.q_decode(0, 3))
        for hq in range(4):
            assert (out[0, hq] == c.position_row(0, 0, hq // 2, 1, 0)).all()


def test_identical_keys_and_zero_query_give_mean_value():
    wl = _wl(T=64)
    c = orc.Cache(1, 1, 2, 4, 64, 64, orc.Q5_1, orc.Q6_0)
    k = np.repeat(wl.kv_chunk(0, 0, 1, "k"), 64, axis=1)
    v = wl.kv_chunk(0, 0, 64, "v")
    c.append(0, k, v)
    _, V = _stored(c, 1, 2, 64)
    mean = V.astype(np.float64).mean(axis=2)                 # [B][H][D]
    out = c.decode(0, wl.q_decode(0, 0))
    for hq in range(4):
        np.testing.assert_allclose(out[0, hq], mean[0, hq // 2], rtol=1e-6, atol=1e-7)
    c2 = orc.Cache(1, 1, 2, 4, 64, 64, orc.Q5_1, orc.Q6_0)
    c2.append(0, wl.kv_chunk(0, 0, 64, "k"), v)
    out2 = c2.decode(0, np.zeros((1, 4, 64), np.float32))
    for hq in range(4):
        np.testing.assert_allclose(out2[0, hq], mean[0, hq // 2], rtol=1e-6, atol=1e-7)


def test_bf16_tail_only_is_textbook_attention_on_bf16_inputs():
    """n <= W with a bf16 ring: every row is the bf16 rounding of its input, so the
    output is plain attention over torch-rounded inputs."""
    wl = _wl(B=2, H=2, Hq=4, D=64, T=48)
    c = orc.Cache(1, 2, 2, 4, 64, 128, orc.Q2_0, orc.Q3_1, orc.BF16, 64)
    n = _fill(c, wl, [20, 28])
    kb = torch.from_numpy(wl.kv_chunk(0, 0, n, "k")).bfloat16().double().numpy()
    vb = torch.from_numpy(wl.kv_chunk(0, 0, n, "v")).bfloat16().double().numpy()
    q = wl.q_decode(0, 1)
    out = c.decode(0, q, scale=1.0)
    ref = _sdpa(q[:, :, None, :], kb.transpose(0, 2, 1, 3), vb.transpose(0, 2, 1, 3), 1.0)[:, :, 0, :]
    np.testing.assert_allclose(out, ref, rtol=1e-6, atol=1e-7)


def test_tail_identity_below_window():
    """Context <= W: (q6_0, q5_0, q8_0 tail) gives bit-identical output to all-q8_0."""
    wl = _wl(B=1, H=2, Hq=6, D=128, T=100, kind="outlier")
    a = orc.Cache(1, 1, 2, 6, 128, 256, orc.Q6_0, orc.Q5_0, orc.Q8_0, 128)
    b = orc.Cache(1, 1, 2, 6, 128, 256, orc.Q8_0, orc.Q8_0)
    _fill(a, wl, [60, 40])
    _fill(b, wl, [100])
    q = wl.q_decode(0, 0)
    assert (a.decode(0, q) == b.decode(0, q)).all()


def test_q8_tail_to_q8_main_is_lossless():
    wl = _wl(B=1, H=1, Hq=1, D=64, T=100)
    c = orc.Cache(1, 1, 1, 1, 64, 128, orc.Q8_0, orc.Q8_0, orc.Q8_0, 16)
    _fill(c, wl, [33, 1, 66])
    k = wl.kv_chunk(0, 0, 100, "k")[0, :, 0]
    main = c.export(0, 0, 0, 0, 0, 0, 84).reshape(84, -1)
    for t in range(84):
        assert (main[t] == orc.quantize_row(orc.Q8_0, k[t])).all()


def test_ring_placement_and_requantization():
    """Ring slot p mod W holds bf16(x_p) for the last W positions (torch's bf16
    rounding); main rows hold Q_low of the tail-rounded value."""
    W, n = 16, 70
    wl = _wl(B=1, H=1, Hq=2, D=64, T=n)
    c = orc.Cache(1, 1, 1, 2, 64, 128, orc.Q4_1, orc.Q4_1, orc.BF16, W)
    _fill(c, wl, [5, 30, 35])
    k = wl.kv_chunk(0, 0, n, "k")[0, :, 0]
    ring = c.export(0, 0, 0, 0, 1, 0, W).reshape(W, 64 * 2).view(np.uint16)
    kb = torch.from_numpy(k).bfloat16().view(torch.int16).numpy().view(np.uint16)
    for p in range(n - W, n):
        assert (ring[p % W] == kb[p]).all()
    main = c.export(0, 0, 0, 0, 0, 0, n - W).reshape(n - W, -1)
    kbf = torch.from_numpy(k).bfloat16().float().numpy()
    for p in range(n - W):
        assert (main[p] == orc.quantize_row(orc.Q4_1, kbf[p])).all()


@pytest.mark.parametrize("tf,W", [(orc.NONE, 0), (orc.Q8_0, 32), (orc.F16, 7)])
def test_chunk_invariance(tf, W):
    wl = _wl(B=2, H=2, Hq=4, D=64, T=100, kind="offset")
    ref = None
    for chunks in ([1] * 100, [7] * 14 + [2], [64, 36], [100]):
        c = orc.Cache(1, 2, 2, 4, 64, 128, orc.Q3_0, orc.Q6_1, tf, W)
        _fill(c, wl, chunks)
        blobs = [c.export(0, b, h, kv, 0, 0, 128) for b in range(2) for h in range(2) for kv in range(2)]
        if W:
            blobs += [c.export(0, b, h, kv, 1, 0, W) for b in range(2) for h in range(2) for kv in range(2)]
        blob = np.concatenate(blobs)
        if ref is None:
            ref = blob
        assert (blob == ref).all()


def test_kvarn_constant_channel_closed_form():
    """A channel equal to a over the first 512 tokens has s = sqrt(a^2 + 1e-6),
    whatever comes after."""
    B, H, D, T = 1, 2, 64, 700
    rng = np.random.default_rng(3)
    k = rng.standard_normal((B, T, H, D)).astype(np.float32)
    v = rng.standard_normal((B, T, H, D)).astype(np.float32)
    consts = rng.standard_normal(H * D).astype(np.float32).reshape(H, D)
    k[:, :512] = consts[None, None]
    c = orc.Cache(1, B, H, 2 * H, D, 1024, orc.Q6_0, orc.Q5_0, kvarn=1)
    c.append(0, k, v)
    sK, sV = c.channel_scales(0)
    expect = np.array([[np.float32(math.sqrt(float(a) * float(a) + 1e-6)) for a in row] for row in consts])
    assert (sK[0] == expect).all()
    # V: mean of squares over the first 512 tokens (any summation order agrees to 1e-12)
    ms = (v[:, :512].astype(np.float64) ** 2).mean(axis=1)
    np.testing.assert_allclose(sV.astype(np.float64) ** 2, ms + 1e-6, rtol=2e-7)
    # later tokens do not move the statistics
    k2 = k.copy()
    k2[:, 512:] *= 100
    c2 = orc.Cache(1, B, H, 2 * H, D, 1024, orc.Q6_0, orc.Q5_0, kvarn=1)
    c2.append(0, k2, v)
    assert (c2.channel_scales(0)[0] == sK).all()


def test_kvarn_storage_is_normalised_quantization():
    """Main rows hold Q(x / s); attention reads s * deq."""
    B, H, D, T = 1, 1, 64, 520
    rng = np.random.default_rng(4)
    k = (rng.standard_normal((B, T, H, D)) * np.linspace(0.1, 10, D)).astype(np.float32)
    v = rng.standard_normal((B, T, H, D)).astype(np.float32)
    c = orc.Cache(1, B, H, 2, D, 1024, orc.Q4_0, orc.Q4_0, kvarn=1)
    c.append(0, k, v)
    sK, _ = c.channel_scales(0)
    row = c.export(0, 0, 0, 0, 0, 519, 1)
    y = (k[0, 519, 0] / sK[0, 0]).astype(np.float32)
    assert (row == orc.quantize_row(orc.Q4_0, y)).all()
    got = c.position_row(0, 0, 0, 0, 519)
    assert (got == (sK[0, 0] * orc.dequant_row(orc.Q4_0, row, D)).astype(np.float32)).all()


def test_error_paths():
    wl = _wl(T=64)
    c = orc.Cache(1, 1, 2, 4, 64, 32, orc.Q4_0, orc.Q4_0)
    with pytest.raises(orc.OracleError) as e:
        c.decode(0, wl.q_decode(0, 0))
    assert e.value.code == 5                                   # empty
    with pytest.raises(orc.OracleError) as e:
        c.append(0, wl.kv_chunk(0, 0, 40, "k"), wl.kv_chunk(0, 0, 40, "v"))
    assert e.value.code == 3 and c.length(0) == 0               # capacity, nothing stored
    kv = orc.Cache(1, 1, 2, 4, 64, 2048, orc.Q4_0, orc.Q4_0, kvarn=1)
    with pytest.raises(orc.OracleError) as e:
        kv.append(0, wl.kv_chunk(0, 0, 64, "k"), wl.kv_chunk(0, 0, 64, "v"))
    assert e.value.code == 4 and kv.length(0) == 0              # calibration needs 512 tokens
    with pytest.raises(ValueError):
        orc.Cache(1, 1, 2, 4, 64, 32, orc.Q4_0, orc.Q4_0, orc.Q8_0, 0)   # tail without window
