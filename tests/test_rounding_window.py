"""The append kernel rounds codes without dividing: r = x * rd with rd within 1 ulp of 1/d
(the hardware reciprocal), r clamped to the code range, the nearest integer taken by adding
1.5 * 2^23, and the correctly rounded quotient (round half away from zero) used instead
whenever r lies within 4e-7 * lim of a half-integer. This checks, in float32 arithmetic on
the host, that the procedure returns exactly clamp(rhaz(fl(x / d))) for every positive fp16
scale d, with rd taken 1 ulp below, at and 1 ulp above fl(1 / d), on random values and on
values placed a few ulps around every code half-step."""
import numpy as np

MAGIC = np.float32(12582912.0)


def _rhaz(q):
    return np.sign(q) * np.floor(np.abs(q) + np.float32(0.5))


def _kernel_codes(x, d, rd, lo, hi):
    tol = np.float32(4e-7) * np.float32(max(-lo, hi))
    r = np.clip((x * rd).astype(np.float32), np.float32(lo), np.float32(hi))
    t = (r + MAGIC).astype(np.float32)
    kf = (t - MAGIC).astype(np.float32)
    e = (r - kf).astype(np.float32)
    near = np.abs(np.abs(e) - np.float32(0.5)) <= tol
    exact = np.clip(_rhaz((x / d).astype(np.float32)), lo, hi)
    return np.where(near, exact, kf), exact


def test_division_free_rounding_matches_ieee():
    rng = np.random.default_rng(11)
    d_all = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)   # every positive finite fp16
    for lo, hi in [(-1, 1), (-15, 15), (-127, 127), (0, 3), (0, 63), (0, 255)]:
        d = np.repeat(d_all, 8)
        span = np.float32(hi - lo)
        x = (np.float32(lo) + rng.random(d.size, dtype=np.float32) * span) * d
        # adversarial: a few ulps around the half-steps k + 1/2 of the code range
        k = rng.integers(lo, hi, size=d.size).astype(np.float32) + np.float32(0.5)
        xh = (k * d).astype(np.float32)
        xh = np.nextafter(xh, np.float32(np.inf) * rng.choice([-1, 1], d.size)).astype(np.float32)
        for xs in (x.astype(np.float32), xh):
            y = (np.float32(1) / d).astype(np.float32)
            for rd in (np.nextafter(y, np.float32(0)), y, np.nextafter(y, np.float32(np.inf))):
                got, want = _kernel_codes(xs, d, rd.astype(np.float32), lo, hi)
                bad = np.nonzero(got != want)[0]
                assert bad.size == 0, (lo, hi, xs[bad[:3]], d[bad[:3]], got[bad[:3]], want[bad[:3]])


def test_division_free_rounding_matches_ieee_asymmetric():
    """The qX_1 form: the kernel rounds v = fl(x - m) (m the block's fp16 min) by the same
    division-free procedure over the code range [0, 2^X - 1]; it must equal
    clamp(rhaz(fl(fl(x - m) / d))) for every positive fp16 d, on random x and on x a few
    ulps around every half-step m + (k + 1/2) d."""
    rng = np.random.default_rng(12)
    d_all = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    for X in (2, 3, 4, 5, 6, 8):
        hi = (1 << X) - 1
        d = np.repeat(d_all, 4)
        # block minimum: an fp16 value of either sign, up to a few code ranges away from 0
        m = (rng.standard_normal(d.size) * d * hi).astype(np.float16).astype(np.float32)
        m[~np.isfinite(m)] = 0.0
        x = (m + rng.random(d.size, dtype=np.float32) * np.float32(hi) * d).astype(np.float32)
        k = rng.integers(0, hi, size=d.size).astype(np.float32) + np.float32(0.5)
        xh = (m + (k * d).astype(np.float32)).astype(np.float32)
        xh = np.nextafter(xh, np.float32(np.inf) * rng.choice([-1, 1], d.size)).astype(np.float32)
        for xs in (x, xh):
            ok = np.isfinite(xs)
            v = (xs[ok] - m[ok]).astype(np.float32)
            dd = d[ok]
            y = (np.float32(1) / dd).astype(np.float32)
            for rd in (np.nextafter(y, np.float32(0)), y, np.nextafter(y, np.float32(np.inf))):
                got, want = _kernel_codes(v, dd, rd.astype(np.float32), 0, hi)
                bad = np.nonzero(got != want)[0]
                assert bad.size == 0, (X, v[bad[:3]], dd[bad[:3]], got[bad[:3]], want[bad[:3]])
