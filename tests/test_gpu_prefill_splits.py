"""GPU parity of the tensor-core prefill when its 128-row M-tiles are split over the key range
(a CTA per split, partial O with the row's running max and sum, then a merge). Staged kernel:
few M-tiles against a long context, where the split count that best fills the SMs is the
largest (4); batch 2 (the grid's batch / split index); head dims 128 and 256; formats with a
q8_0 / bf16 ring and without one; a context too short to split (the first M-tile must keep 32
tiles per split), whose rows are finished in place. Verify chunks of 1 to 8 rows over a
20,000-position context: the split-K decode kernel up to 4 rows, then the on-the-fly tcgen05
kernel (one M-tile per kv head) split many ways."""
import numpy as np
import pytest

import oracle as orc
from quantized_mixed_precision_qx_b200.synth import KVRecipe, Workload
from harness import append_both, check_close, make_pair, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D", [128, 256])
@pytest.mark.parametrize("kf,vf,tail,W", [(orc.Q6_0, orc.Q5_0, orc.Q8_0, 512), (orc.Q4_1, orc.Q3_1, orc.BF16, 256),
                                          (orc.Q8_0, orc.Q5_1, orc.NONE, 0)])
def test_split_prefill(D, kf, vf, tail, W):
    # 300 rows x 6 query heads per kv head = 15 M-tiles per (b, h): 60 CTAs before splitting
    T, C = 9000, 300
    wl = Workload(1, 2, 2, 12, D, T, KVRecipe("outlier" if kf % 2 == 0 else "offset"), seed=140 + kf)
    g, o = make_pair(wl, kf, vf, tail, W)
    vmax = append_both(g, o, wl, 0, 0, T - C)
    vmax = max(vmax, append_both(g, o, wl, 0, T - C, T))
    q = wl.q_prefill(0, C)
    check_close(g.prefill(0, to_dev(q), 0.9).cpu().numpy(), o.prefill(0, q, 0.9), vmax,
                f"split prefill D={D} kf={kf} vf={vf} tail={tail}")


@pytest.mark.parametrize("T,C", [(1500, 1200), (4200, 300)])
def test_short_context_prefill(T, C):
    """n - C of 300 (10 tiles) leaves no split; 3,900 (122 tiles) allows up to 3."""
    wl = Workload(1, 1, 2, 12, 256, T, KVRecipe("outlier"), seed=150)
    g, o = make_pair(wl, orc.Q6_0, orc.Q5_0, orc.Q8_0, 256)
    vmax = append_both(g, o, wl, 0, 0, T)
    q = wl.q_prefill(0, C)
    check_close(g.prefill(0, to_dev(q), 1.0).cpu().numpy(), o.prefill(0, q, 1.0), vmax,
                f"prefill n={T} C={C}")


@pytest.mark.parametrize("D", [128, 256])
@pytest.mark.parametrize("C", [1, 3, 4, 5, 8])
def test_short_chunk_split(D, C):
    """A multi-query verify chunk (C rows, one M-tile per kv head) over a long context: up to 4
    rows take the split-K decode kernel (one pass per row); from 5 rows the on-the-fly tcgen05
    kernel splits the key range over many CTAs (here up to 19 per M-tile)."""
    T = 20000
    wl = Workload(1, 2, 2, 12, D, T, KVRecipe("outlier"), seed=160 + C)
    g, o = make_pair(wl, orc.Q6_0, orc.Q5_0, orc.Q8_0, 1024)
    vmax = append_both(g, o, wl, 0, 0, T - C)
    vmax = max(vmax, append_both(g, o, wl, 0, T - C, T))
    q = wl.q_prefill(0, C)
    check_close(g.prefill(0, to_dev(q), 1.0).cpu().numpy(), o.prefill(0, q, 1.0), vmax,
                f"verify chunk C={C} D={D}")
