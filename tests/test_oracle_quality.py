"""Quantization error of the oracle's block formats on Gaussian data: more bits give a
smaller error within each family (qX_0 and qX_1), and the asymmetric format of a width is
no worse than the symmetric one by more than a small factor. These are properties of the
block rules (scale = range / code span), independent of any implementation detail."""
import numpy as np

import oracle as orc


def _rel_err(fmt, x):
    q = orc.quantize_row(fmt, x)
    y = orc.dequant_row(fmt, q, x.size)
    return float(np.linalg.norm(y - x) / np.linalg.norm(x))


def test_error_decreases_with_bits():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(32 * 256).astype(np.float32)
    sym = [orc.Q2_0, orc.Q3_0, orc.Q4_0, orc.Q5_0, orc.Q6_0, orc.Q8_0]
    asym = [orc.Q2_1, orc.Q3_1, orc.Q4_1, orc.Q5_1, orc.Q6_1, orc.Q8_1]
    for fam in (sym, asym):
        errs = [_rel_err(f, x) for f in fam]
        assert all(a > b for a, b in zip(errs, errs[1:])), errs
        # each extra bit roughly halves the step: the error ratio per bit is near 2
        # (q8 skips a width: ratio near 4)
        ratios = [a / b for a, b in zip(errs, errs[1:])]
        assert all(1.5 < r < 3.0 for r in ratios[:-1]), ratios
        assert 3.0 < ratios[-1] < 6.0, ratios
    for s, a in zip(sym, asym):
        assert _rel_err(a, x) < 1.5 * _rel_err(s, x)
