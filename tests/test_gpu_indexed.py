"""GPU parity of the index-gather decode (kvq_decode_attention_indexed) against the oracle:
per (batch, kv head) lists of up to 2,048 positions (the QSA budget of "You can offload most
of Qwen3.8-Flash-Next's KV cache to RAM"), drawn over the whole context so that they hit
both the low-bit store and the ring; ragged list lengths; entries outside [0, n), repeated
positions and lists with no valid entry; every format family, KVarN, head dims 64 (CUDA
cores), 128 and 256 (tensor cores); and the full list, which must agree with the decode."""
import numpy as np
import pytest

import oracle as orc
from quantized_mixed_precision_qx_b200.synth import KVRecipe, Workload
from harness import append_both, check_close, make_pair, to_dev

pytestmark = pytest.mark.gpu


def _lists(rng, B, H, n, k, extra=None):
    idx = np.stack([np.stack([rng.choice(n, k, replace=k > n) for _ in range(H)]) for _ in range(B)])
    if extra is not None:
        idx[..., :len(extra)] = extra
    return idx.astype(np.int32)


def _compare(g, o, wl, idx, vmax, what, step=0, scale=1.0):
    import torch
    q = wl.q_decode(0, step)
    out = g.decode_indexed(0, to_dev(q), torch.from_numpy(idx).cuda(), scale).cpu().numpy()
    ref = o.decode_indexed(0, q, idx, scale)
    return check_close(out, ref, vmax, what), out, ref


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("kf,vf,tail,W,kvarn", [(orc.Q6_0, orc.Q5_0, orc.Q8_0, 512, 0),
                                                (orc.Q4_1, orc.Q3_1, orc.BF16, 256, 0),
                                                (orc.Q8_0, orc.Q2_1, orc.NONE, 0, 0),
                                                (orc.Q6_0, orc.Q5_0, orc.NONE, 0, 1)])
def test_gather_lists(D, kf, vf, tail, W, kvarn):
    T = 6000
    wl = Workload(1, 2, 2, 12, D, T, KVRecipe("outlier" if kf % 2 == 0 else "offset"), seed=100 + kf)
    g, o = make_pair(wl, kf, vf, tail, W, kvarn=kvarn, calib=64)
    vmax = append_both(g, o, wl, 0, 0, 4000)
    vmax = max(vmax, append_both(g, o, wl, 0, 4000, T))
    rng = np.random.default_rng(D + kf)
    for k in (2048, 1, 37, 700):
        # the newest positions (in the ring when there is one) and the oldest always listed
        extra = np.array([T - 1, T - 2, 0, T // 2], dtype=np.int32)[:k]
        idx = _lists(rng, 2, 2, T, k, extra)
        _compare(g, o, wl, idx, vmax, f"gather k={k} D={D} kf={kf} vf={vf} tail={tail} kvarn={kvarn}", step=k % 7)


@pytest.mark.parametrize("D", [64, 256])
def test_gather_edge_entries(D):
    """Entries outside [0, n) are skipped, repeated entries count once each, a list with no
    valid entry gives zeros; the full list in order is the decode."""
    import torch
    T, W = 900, 128
    wl = Workload(1, 1, 2, 12, D, T, KVRecipe("outlier"), seed=110)
    g, o = make_pair(wl, orc.Q6_0, orc.Q5_0, orc.Q8_0, W)
    vmax = append_both(g, o, wl, 0, 0, T)
    rng = np.random.default_rng(4)
    base = rng.choice(T, 50, replace=False).astype(np.int32)
    noisy = np.concatenate([base[:20], [-1, T, T + 1000, -(1 << 30)], base[20:], base[:10]]).astype(np.int32)
    idx = np.broadcast_to(noisy, (1, 2, noisy.size)).copy()
    _compare(g, o, wl, idx, vmax, "skipped and repeated entries")
    empty = np.broadcast_to(np.array([-3, T, 1 << 30], dtype=np.int32), (1, 2, 3)).copy()
    out = g.decode_indexed(0, to_dev(wl.q_decode(0, 0)), torch.from_numpy(empty).cuda()).cpu().numpy()
    assert not out.any()
    full = np.broadcast_to(np.arange(T, dtype=np.int32), (1, 2, T)).copy()
    _, outf, reff = _compare(g, o, wl, full, vmax, "full list")
    q = wl.q_decode(0, 0)
    check_close(outf, g.decode(0, to_dev(q), 1.0).cpu().numpy(), vmax, "full list vs decode")
