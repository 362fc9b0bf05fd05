"""Pins of the oracle's index-gather decode ("You can offload most of Qwen3.8-Flash-Next's
KV cache to RAM with little decode slowdown": the QSA indexer picks a budget of 2,048
positions per step and attention reads only those).

Reading: each (batch, kv head) lists k positions; entries outside [0, n) are skipped, the
others enter in list order (a repeated position counts once per entry); with no valid
entry the output is zero.

Pins (none re-types the function's arithmetic):
- the full list 0..n-1 reproduces the oracle's pinned decode bit for bit (ring, KVarN and
  asymmetric formats);
- a one-entry list, and a position listed twice, return that position's dequantized V;
- skipped entries change nothing; a list with no valid entry gives zeros;
- the full list twice over gives the decode again (every weight doubles);
- an arbitrary subset equals torch's scaled_dot_product_attention in float64 over the
  gathered dequantized rows (an independent library routine, with its own GQA grouping).
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as orc
from quantized_mixed_precision_qx_b200.synth import KVRecipe, Workload

CASES = [(orc.Q8_0, orc.Q8_0, orc.NONE, 0, 0), (orc.Q6_0, orc.Q5_0, orc.Q8_0, 32, 0),
         (orc.Q4_1, orc.Q3_1, orc.BF16, 16, 0), (orc.Q6_0, orc.Q5_0, orc.NONE, 0, 1)]


def _cache(kf, vf, tf, W, kvarn, T=150, B=2, H=2, Hq=6, D=64):
    wl = Workload(1, B, H, Hq, D, T, KVRecipe("outlier"), seed=5)
    c = orc.Cache(1, B, H, Hq, D, T, kf, vf, tf, W, kvarn=kvarn, calib=64)
    c.append(0, wl.kv_chunk(0, 0, 100, "k"), wl.kv_chunk(0, 0, 100, "v"))
    c.append(0, wl.kv_chunk(0, 100, T, "k"), wl.kv_chunk(0, 100, T, "v"))
    return wl, c


@pytest.mark.parametrize("kf,vf,tf,W,kvarn", CASES)
def test_full_list_is_the_decode(kf, vf, tf, W, kvarn):
    wl, c = _cache(kf, vf, tf, W, kvarn)
    n = c.length(0)
    q = wl.q_decode(0, 0)
    idx = np.broadcast_to(np.arange(n, dtype=np.int32), (2, 2, n)).copy()
    assert np.array_equal(c.decode_indexed(0, q, idx, 0.7), c.decode(0, q, 0.7))
    # twice over: every weight doubles, the normalised result is the decode again
    idx2 = np.concatenate([idx, idx], axis=2)
    np.testing.assert_allclose(c.decode_indexed(0, q, idx2, 0.7), c.decode(0, q, 0.7), rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("kf,vf,tf,W,kvarn", CASES)
def test_single_and_repeated_position(kf, vf, tf, W, kvarn):
    wl, c = _cache(kf, vf, tf, W, kvarn)
    q = wl.q_decode(0, 1)
    for t in (0, 77, 149):
        for reps in (1, 2):
            idx = np.full((2, 2, reps), t, dtype=np.int32)
            out = c.decode_indexed(0, q, idx)
            for b in range(2):
                for hq in range(6):
                    assert np.array_equal(out[b, hq], c.position_row(0, b, hq // 3, 1, t))


def test_skipped_entries_and_empty_lists():
    wl, c = _cache(orc.Q6_0, orc.Q5_0, orc.Q8_0, 32, 0)
    n = c.length(0)
    q = wl.q_decode(0, 2)
    sub = np.array([3, 140, 9, 120, 60], dtype=np.int32)
    base = c.decode_indexed(0, q, np.broadcast_to(sub, (2, 2, 5)).copy())
    noisy = np.concatenate([sub[:2], [-1, n, n + 7], sub[2:]]).astype(np.int32)
    assert np.array_equal(c.decode_indexed(0, q, np.broadcast_to(noisy, (2, 2, 8)).copy()), base)
    empty = np.array([-5, n, 1 << 30], dtype=np.int32)
    assert not c.decode_indexed(0, q, np.broadcast_to(empty, (2, 2, 3)).copy()).any()


@pytest.mark.parametrize("kf,vf,tf,W,kvarn", CASES)
def test_subset_matches_library_attention(kf, vf, tf, W, kvarn):
    wl, c = _cache(kf, vf, tf, W, kvarn)
    n = c.length(0)
    rng = np.random.default_rng(3)
    k = 40
    idx = np.stack([np.stack([rng.choice(n, k, replace=False) for _ in range(2)]) for _ in range(2)]).astype(np.int32)
    q = wl.q_decode(0, 3)
    out = c.decode_indexed(0, q, idx, 0.9)
    for b in range(2):
        K = np.stack([np.stack([c.position_row(0, b, h, 0, int(t)) for t in idx[b, h]]) for h in range(2)])
        V = np.stack([np.stack([c.position_row(0, b, h, 1, int(t)) for t in idx[b, h]]) for h in range(2)])
        qt = torch.from_numpy(q[b][:, None, :].astype(np.float64))[None]      # [1][Hq][1][D]
        ref = F.scaled_dot_product_attention(qt, torch.from_numpy(K.astype(np.float64))[None],
                                             torch.from_numpy(V.astype(np.float64))[None], scale=0.9,
                                             enable_gqa=True).numpy()[0, :, 0, :]
        np.testing.assert_allclose(out[b], ref, rtol=1e-6, atol=1e-7)
