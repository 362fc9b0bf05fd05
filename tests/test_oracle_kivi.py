"""Pins of the oracle's per-channel (token-axis) K mode ("Hard numbers on Qwen3.8-27B's KV
cache", section "Reddit reactions": quantizing K along the token axis, as KIVI does, instead
of in blocks of 32 values per token).

Reading: a K block holds 32 consecutive positions of one channel; a position enters the K
store with the same value as for per-token blocks (its tail rounding with a ring, the raw
value without one); a group is quantized when its last position enters; until then the
entered positions wait in a 32-row fp32 pending buffer. V keeps per-token blocks.

Pins (none re-types the per-channel code):
- every stored block equals the block quantizer (pinned by brute force in
  test_oracle_formats.py) applied to the token-axis group, assembled here by slicing the
  inputs (tail-rounded through the pinned row codec when there is a ring);
- every stored code is the nearest code to its value under the stored scale (and min), by
  brute force over all codes, with ties away from zero;
- the pending buffer holds exactly the entered positions of the unfinished group;
- bytes and pending rows do not depend on how the positions are chunked;
- the dequantized rows attention reads are the exported blocks decoded with the pinned
  block codec, and decode / prefill match torch's scaled_dot_product_attention in float64
  over those rows;
- the pages' measurement: without a window, per-channel 5-bit K has a smaller attention
  error than per-token 5-bit K on keys with outlier channels.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as orc
from quantized_mixed_precision_qx_b200.synth import KVRecipe, Workload

D = 64


def _entered_values(x_rows, tf):
    """Values with which positions enter the K store: the rows' tail rounding with a ring
    (pinned row codec), the raw rows without one. x_rows [n][D]."""
    if tf == orc.NONE:
        return x_rows.astype(np.float32)
    return np.stack([orc.dequant_row(tf, orc.quantize_row(tf, r), D) for r in x_rows])


def _fill(kf, tf, W, chunks, T, seed=1, kind="outlier", B=1, H=2):
    wl = Workload(1, B, H, 2 * H, D, T, KVRecipe(kind), seed=seed)
    c = orc.Cache(1, B, H, 2 * H, D, T + 64, kf, orc.Q8_0, tf, W, kivi=1)
    t = 0
    for ch in chunks:
        c.append(0, wl.kv_chunk(0, t, t + ch, "k"), wl.kv_chunk(0, t, t + ch, "v"))
        t += ch
    return wl, c, t


CASES = [(orc.Q5_0, orc.NONE, 0), (orc.Q4_1, orc.NONE, 0), (orc.Q6_0, orc.Q8_0, 48), (orc.Q3_1, orc.BF16, 40),
         (orc.Q8_0, orc.F16, 32), (orc.Q2_0, orc.NONE, 0)]


@pytest.mark.parametrize("kf,tf,W", CASES)
def test_blocks_are_token_axis_groups(kf, tf, W):
    T = 205
    wl, c, n = _fill(kf, tf, W, [100, 105], T)
    entered = n - W if W else n
    G = entered // 32
    bb = orc.block_bytes(kf)
    for h in range(2):
        x = wl.kv_chunk(0, 0, n, "k")[0, :, h, :]
        vals = _entered_values(x[:entered], tf)
        got = c.export(0, 0, h, 0, 0, 0, G)
        for g in range(G):
            for ch in range(D):
                u, d16, m16 = orc.quantize_codes(kf, vals[32 * g:32 * g + 32, ch])
                want = orc.pack_block(kf, u, d16, m16)
                off = (g * D + ch) * bb
                assert (got[off:off + bb] == want).all(), (g, ch)
        pend = c.export(0, 0, h, 0, 2, 0, entered - 32 * G).view(np.float32).reshape(-1, D)
        assert np.array_equal(pend, vals[32 * G:entered])


@pytest.mark.parametrize("kf", [orc.Q5_0, orc.Q3_1, orc.Q8_1])
def test_codes_are_nearest_by_brute_force(kf):
    wl, c, n = _fill(kf, orc.NONE, 0, [160], 160)
    X = orc.fmt_bits(kf)
    bb = orc.block_bytes(kf)
    x = wl.kv_chunk(0, 0, n, "k")[0, :, 0, :]
    got = c.export(0, 0, 0, 0, 0, 0, n // 32)
    for g in range(n // 32):
        for ch in range(0, D, 7):
            u, d16, m16 = orc.unpack_block(kf, got[(g * D + ch) * bb:(g * D + ch + 1) * bb])
            cand = np.array([orc.dequant_code(kf, d16, m16, k) for k in range(1 << X)], dtype=np.float64)
            for t in range(32):
                v = float(x[32 * g + t, ch])
                err = np.abs(v - cand)
                best = np.flatnonzero(err <= err.min() * (1 + 1e-6) + 1e-12)
                assert u[t] in best, (g, ch, t, v, u[t], best)


@pytest.mark.parametrize("kf,tf,W", [(orc.Q5_0, orc.NONE, 0), (orc.Q6_0, orc.Q8_0, 48), (orc.Q3_1, orc.BF16, 40)])
def test_chunk_invariance(kf, tf, W):
    blobs = []
    for chunks in ([1] * 150, [7] * 21 + [3], [33, 33, 33, 51], [150]):
        _, c, n = _fill(kf, tf, W, chunks, 150)
        entered = n - W if W else n
        parts = [c.export(0, 0, h, 0, 0, 0, entered // 32) for h in range(2)]
        parts += [c.export(0, 0, h, 0, 2, 0, entered % 32) for h in range(2)]
        if W:
            parts += [c.export(0, 0, h, 0, 1, 0, W) for h in range(2)]
        blobs.append(np.concatenate(parts))
    for b in blobs[1:]:
        assert np.array_equal(b, blobs[0])


@pytest.mark.parametrize("kf,tf,W", CASES)
def test_rows_and_attention(kf, tf, W):
    T = 173
    wl, c, n = _fill(kf, tf, W, [90, 83], T)
    entered = n - W if W else n
    G = entered // 32
    bb = orc.block_bytes(kf)
    # the rows attention reads: decoded exported blocks, pending rows, ring rows
    for h in range(2):
        got = c.export(0, 0, h, 0, 0, 0, G)
        for p in list(range(0, n, 11)) + [32 * G - 1, entered - 1, n - 1]:
            row = c.position_row(0, 0, h, 0, p)
            if p < 32 * G:
                want = []
                for ch in range(D):
                    u, d16, m16 = orc.unpack_block(kf, got[((p // 32) * D + ch) * bb:((p // 32) * D + ch + 1) * bb])
                    want.append(orc.dequant_code(kf, d16, m16, u[p % 32]))
                assert np.array_equal(row, np.array(want, dtype=np.float32))
            elif p < entered:
                pend = c.export(0, 0, h, 0, 2, p % 32, 1).view(np.float32)
                assert np.array_equal(row, pend)
    K = np.stack([np.stack([c.position_row(0, 0, h, 0, t) for t in range(n)]) for h in range(2)])[None]
    V = np.stack([np.stack([c.position_row(0, 0, h, 1, t) for t in range(n)]) for h in range(2)])[None]
    q = wl.q_decode(0, 0)
    ref = F.scaled_dot_product_attention(torch.from_numpy(q[:, :, None, :].astype(np.float64)),
                                         torch.from_numpy(K.astype(np.float64)), torch.from_numpy(V.astype(np.float64)),
                                         scale=1.0, enable_gqa=True).numpy()[:, :, 0, :]
    np.testing.assert_allclose(c.decode(0, q, 1.0), ref, rtol=1e-6, atol=1e-7)
    C = 40
    qp = wl.q_prefill(0, C)
    rows = np.arange(n - C, n)
    mask = torch.arange(n)[None, :] <= torch.as_tensor(rows)[:, None]
    refp = F.scaled_dot_product_attention(torch.from_numpy(qp.transpose(0, 2, 1, 3).astype(np.float64)),
                                          torch.from_numpy(K.astype(np.float64)),
                                          torch.from_numpy(V.astype(np.float64)), attn_mask=mask, scale=1.0,
                                          enable_gqa=True).numpy().transpose(0, 2, 1, 3)
    np.testing.assert_allclose(c.prefill(0, qp, 1.0), refp, rtol=1e-6, atol=1e-7)


def test_per_channel_k_helps_without_a_window():
    """The pages: without a window, per-channel 5-bit K reduced the error of the attention
    output. Keys with 8 outlier channels per head (x8), V in q8_0, decode error against
    exact attention over the raw inputs."""
    T, H, Hq = 2048, 2, 12
    wl = Workload(1, 1, H, Hq, 128, T, KVRecipe("outlier"), seed=9)
    k, v = wl.kv_chunk(0, 0, T, "k"), wl.kv_chunk(0, 0, T, "v")
    G = Hq // H
    errs = {}
    for kivi in (0, 1):
        c = orc.Cache(1, 1, H, Hq, 128, T, orc.Q5_0, orc.Q8_0, kivi=kivi)
        c.append(0, k, v)
        num = den = 0.0
        for step in range(4):
            q = wl.q_decode(0, step)
            out = c.decode(0, q, 1.0)
            kk = torch.from_numpy(k[0].transpose(1, 0, 2).astype(np.float64)).repeat_interleave(G, 0)
            vv = torch.from_numpy(v[0].transpose(1, 0, 2).astype(np.float64)).repeat_interleave(G, 0)
            ref = torch.softmax(torch.einsum("hd,hnd->hn", torch.from_numpy(q[0].astype(np.float64)), kk), -1)
            ref = torch.einsum("hn,hnd->hd", ref, vv).numpy()
            num += float(((out[0] - ref) ** 2).sum())
            den += float((ref ** 2).sum())
        errs[kivi] = (num / den) ** 0.5
    assert errs[1] < errs[0], errs
