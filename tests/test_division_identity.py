"""The append kernel computes absmax / (2^k - 1) and (max - min) / (2^k - 1) without a
divide: q = fl(a * y) with y = fl(1 / b), refined once to fl(q + fl(a - q * b) * y) with
fused multiply-adds (Markstein's division by a constant). This pins the identity with the
IEEE quotient on the host CPU over a stride sample of every non-negative finite float32 for
each b = 2^k - 1 the formats use (an exhaustive run over all 2^31 values found no mismatch),
and pins the reciprocal constants the kernel embeds."""
import os
import shutil
import subprocess
import tempfile

import pytest

SRC = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
static const float B[] = {1.f, 3.f, 7.f, 15.f, 31.f, 63.f, 127.f, 255.f};
static const float Y[] = {0x1p+0f, 0x1.555556p-2f, 0x1.24924ap-3f, 0x1.111112p-4f,
                          0x1.08421p-5f, 0x1.041042p-6f, 0x1.020408p-7f, 0x1.010102p-8f};
int main(void) {
    long bad = 0;
    for (int k = 0; k < 8; ++k) {
        volatile float one = 1.0f;
        const float y = one / B[k];
        if (memcmp(&y, &Y[k], 4) != 0) { printf("constant %d differs\n", k); return 2; }
        for (uint32_t u = 0; u < 0x7F800000u; u += 61u) {
            float a; memcpy(&a, &u, 4);
            const float q = a * y;
            const float r = fmaf(-q, B[k], a);
            const float q2 = fmaf(r, y, q);
            const float ref = a / B[k];
            if (memcmp(&q2, &ref, 4) != 0) { if (bad < 4) printf("b=%g a=%a\n", B[k], a); ++bad; }
        }
    }
    printf("mismatches %ld\n", bad);
    return bad != 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_division_by_code_range_is_ieee():
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "div.c")
        exe = os.path.join(d, "div")
        open(c, "w").write(SRC)
        # no contraction: q = a * y and the reference a / b must each round once; fmaf fuses
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", c, "-o", exe, "-lm"])
        r = subprocess.run([exe], capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stdout + r.stderr
        assert "mismatches 0" in r.stdout


def test_kernel_reciprocal_table():
    """The table in the append kernel holds fl(1 / (2^k - 1)), k = 1..8."""
    import re

    import numpy as np
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = open(os.path.join(root, "quantized_mixed_precision_qx_b200", "csrc", "kvq_append.cu")).read()
    body = re.search(r"c_rcp_range\[9\]\s*=\s*\{([^}]*)\}", src).group(1)
    vals = [float.fromhex(v.strip().rstrip("f")) if "0x" in v else float(v.strip().rstrip("f"))
            for v in body.split(",")]
    assert len(vals) == 9
    for k in range(1, 9):
        want = np.float32(1.0) / np.float32((1 << k) - 1)
        assert np.float32(vals[k]) == want and float(np.float32(vals[k])) == vals[k], (k, vals[k], want)
