"""Pins of the oracle's block formats against what the pages and arithmetic fix.

* byte counts: the cache-size percentages of the KLD table on "KV cache quant
  benchmarks: KVarN 6-bit matches q8_0" and the KV-MiB table on "BeeLlama.cpp
  v0.4.1" (tests/golden);
* fp16 / bf16 rounding: every one of the 2^32 float32 bit patterns against the
  host's hardware conversion (torch CPU, F16C) and torch's bfloat16 rounding;
* quantizer: brute-force nearest-code search on random blocks, exhaustive code
  vectors on mini-blocks, and idempotence on dequantized blocks;
* serialisation: plane packing checked bit by bit against an independent
  bit-string construction.
"""
import os

import numpy as np
import pytest
import torch

import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _fmt(name):
    return orc.FMT_NAMES.index(name)


# ---------------------------------------------------------------- byte counts
def test_block_bytes_match_cache_size_table():
    """Pair size / bf16 size, rounded to 0.1%, equals the printed percentage."""
    for kf, vf, pct in _read("cache_size_table.txt"):
        kb = orc.block_bytes(_fmt(kf))
        vb = orc.block_bytes(_fmt(vf))
        ratio = 100.0 * (kb + vb) / (2 * 64)
        assert round(ratio, 1) == float(pct), (kf, vf, ratio, pct)


def test_block_bytes_match_kv_mib_table():
    """16 attention layers x 4 KV heads x 256 dims x (K, V) at 65,536 tokens is
    2^26 blocks, so MiB = 64 x block bytes; a bf16 tail of T tokens adds
    T x 32,768 values x 2 bytes. The table's fixed +32 MiB engine overhead on
    tail rows is not part of the cache and is removed before comparing."""
    values_per_token = 16 * 4 * 256 * 2
    bf16_row = orc.row_bytes(orc.BF16, 256)
    assert bf16_row == 512
    rows = _read("kv_mib_64k.txt")
    for fmt, tail, mib in rows:
        f = _fmt(fmt)
        blocks = 65536 * values_per_token // 32
        main = blocks * orc.block_bytes(f)
        tail_bytes = int(tail) * values_per_token * 2
        total_mib = (main + tail_bytes) / 2**20
        overhead = 0 if int(tail) == 0 else 32
        assert total_mib + overhead == float(mib), (fmt, tail, total_mib, mib)
    # the two tail sizes differ by exactly 1024 bf16 rows of every layer/head
    by = {(r[0], int(r[1])): float(r[2]) for r in rows}
    for fmt in ("q8_0", "q6_0", "q5_0", "q4_0"):
        assert by[(fmt, 2048)] - by[(fmt, 1024)] == 1024 * values_per_token * 2 / 2**20


def test_row_arithmetic():
    g = {k: float(v) for k, v in _read("row_arithmetic.txt")}
    per_token = 2 * 2 * orc.row_bytes(orc.BF16, 256)       # 2 heads x (K + V) bf16 rows
    assert per_token == g["bytes_per_token_per_layer"]
    assert per_token * 262144 / 2**20 == g["mib_per_layer_at_262144"]
    assert 12 * per_token * 262144 / 2**30 == g["gib_all_12_layers_at_262144"]
    assert per_token * 2048 / 2**20 == g["mib_per_layer_at_2048_selected"]
    assert 12 * per_token * 2048 / 2**20 == g["mib_per_token_all_12_layers_at_2048_selected"]


def test_config_d_memory_consistency():
    """q8_0 K+V minus (q6_0 K + q5_0 V) per token over 16 layers x 4 heads, times
    120k tokens, minus the 2,048-row q8_0 ring: about the 1.1 GB the page reports."""
    g = {k: float(v) for k, v in _read("config_d_memory.txt")}
    units = g["attention_layers"] * g["kv_heads"]
    q8 = units * 2 * orc.row_bytes(orc.Q8_0, 256)
    d = units * (orc.row_bytes(orc.Q6_0, 256) + orc.row_bytes(orc.Q5_0, 256))
    assert q8 == 34816 and d == 24576
    saved = (q8 - d) * g["context_tokens"] - g["ring_tokens"] * q8
    reported = (g["gb_q8_0"] - g["gb_config_d"]) * 1e9
    assert abs(saved - reported) < 0.1e9, (saved, reported)


# ---------------------------------------------------------- fp16 / bf16 rounding
@pytest.mark.parametrize("which", ["f16", "bf16"])
def test_conversion_exhaustive(which):
    """All 2^32 float32 patterns: oracle rounding == host conversion (NaN: any NaN)."""
    chunk = 1 << 26
    exp_mask, man_mask = (0x7C00, 0x03FF) if which == "f16" else (0x7F80, 0x007F)
    for c in range((1 << 32) // chunk):
        u = np.arange(c * chunk, (c + 1) * chunk, dtype=np.uint32)
        x = u.view(np.float32)
        t = torch.from_numpy(x)
        if which == "f16":
            ref = t.half().view(torch.int16).numpy().view(np.uint16)
            got = orc.f32_to_f16_bits(x)
        else:
            ref = t.bfloat16().view(torch.int16).numpy().view(np.uint16)
            got = orc.f32_to_bf16_bits(x)
        miss = np.nonzero(got != ref)[0]
        if miss.size:                       # only NaN payloads may differ
            r, g = ref[miss], got[miss]
            ref_nan = ((r & exp_mask) == exp_mask) & ((r & man_mask) != 0)
            got_nan = ((g & exp_mask) == exp_mask) & ((g & man_mask) != 0)
            bad = miss[~(ref_nan & got_nan)][:5]
            assert bad.size == 0, f"{which}: {[(hex(int(u[i])), hex(int(got[i])), hex(int(ref[i]))) for i in bad]}"


def test_f16_decode_exhaustive():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = orc.f16_bits_to_f32(h)
    ref = torch.from_numpy(h.view(np.int16)).view(torch.float16).float().numpy()
    same = (got.view(np.uint32) == ref.view(np.uint32)) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


# -------------------------------------------------------------------- quantizer
def _f16(h):
    return float(orc.f16_bits_to_f32(np.array([h], dtype=np.uint16))[0])


def _code_set(f):
    X = orc.fmt_bits(f)
    if orc.fmt_asym(f):
        return np.arange(0, 1 << X)
    off = 1 << (X - 1)
    return np.arange(1, 1 << X)          # signed -qmax..qmax


def _value(f, d, m, u):
    X = orc.fmt_bits(f)
    if orc.fmt_asym(f):
        return d * u + m
    return d * (u - (1 << (X - 1)))


def _check_nearest(f, x, u, d16, m16):
    """Each code is the nearest representable value (fp64 distance), ties away
    from zero; a miss is allowed only where the fp32 quotient crossed a .5."""
    d, m = _f16(d16), (_f16(m16) if orc.fmt_asym(f) else 0.0)
    X = orc.fmt_bits(f)
    if d == 0.0:
        expect = 0 if orc.fmt_asym(f) else (1 << (X - 1))
        assert (u == expect).all()
        return 0
    cs = _code_set(f)
    vals = np.array([_value(f, d, m, c) for c in cs], dtype=np.float64)
    explained = 0
    for i, xi in enumerate(x.astype(np.float64)):
        dist = np.abs(xi - vals)
        best = np.nonzero(dist == dist.min())[0]
        if len(best) > 1:                       # tie: away from zero in code space
            center = 0 if orc.fmt_asym(f) else (1 << (X - 1))
            best = [max(best, key=lambda j: abs(cs[j] - center))]
        if cs[best[0]] == u[i]:
            continue
        # the only allowed miss: the float32 subtraction / division rounded the
        # quotient onto or across a half step that the exact quotient does not reach
        num = np.float32(xi) if not orc.fmt_asym(f) else np.float32(np.float32(xi) - np.float32(m))
        q32 = float(np.float32(num / np.float32(d)))
        qex = (xi - m) / d
        k = np.floor(qex) + 0.5
        assert (q32 - k) * (qex - k) <= 0 and q32 != qex, (f, xi, u[i], cs[best[0]], q32, qex)
        explained += 1
    return explained


@pytest.mark.parametrize("f", orc.LOWBIT)
def test_quantizer_nearest_code(f):
    rng = np.random.default_rng(100 + f)
    misses = 0
    for trial in range(300):
        kind = trial % 5
        if kind == 0:
            x = rng.standard_normal(32)
        elif kind == 1:
            x = rng.standard_normal(32) * 10 ** rng.uniform(-6, 3)
        elif kind == 2:
            x = rng.uniform(0.5, 2.0, 32) + rng.standard_normal() * 3
        elif kind == 3:                       # values on exact half steps
            x = (rng.integers(-20, 21, 32) + 0.5) * 0.03125
        else:
            x = np.zeros(32)
            x[rng.integers(0, 32)] = rng.standard_normal()
        x = x.astype(np.float32)
        u, d16, m16 = orc.quantize_codes(f, x)
        misses += _check_nearest(f, x, u, d16, m16)
    assert misses < 10


def test_quantizer_zero_block():
    for f in orc.LOWBIT:
        u, d16, m16 = orc.quantize_codes(f, np.zeros(32, np.float32))
        assert d16 == 0
        X = orc.fmt_bits(f)
        assert (u == (0 if orc.fmt_asym(f) else 1 << (X - 1))).all()


def test_quantizer_scale_saturates():
    x = np.full(32, 3.0e38, np.float32)
    for f in orc.LOWBIT:
        u, d16, m16 = orc.quantize_codes(f, x)
        assert d16 == 0x7BFF or orc.fmt_asym(f)   # 65504


def _check_nearest_batch(f, x, u, d16, m16):
    """Vectorised _check_nearest over rows of x (N x k): returns the number of
    misses, after asserting every miss is a float32 rounding across a half step."""
    X = orc.fmt_bits(f)
    asym = orc.fmt_asym(f)
    d = orc.f16_bits_to_f32(d16.astype(np.uint16)).astype(np.float64)
    m = orc.f16_bits_to_f32(m16.astype(np.uint16)).astype(np.float64) if asym else np.zeros_like(d)
    cs = _code_set(f)
    center = 0 if asym else (1 << (X - 1))
    vals = (d[:, None] * (cs[None, :] - (0 if asym else center))) + m[:, None]   # N x C
    xx = x.astype(np.float64)
    dist = np.abs(xx[:, :, None] - vals[:, None, :])                              # N x k x C
    mn = dist.min(axis=2, keepdims=True)
    # among the minimisers pick the one farthest from the centre (ties away from zero)
    score = np.where(dist == mn, np.abs(cs - center)[None, None, :], -1)
    best = cs[score.argmax(axis=2)]
    zero = d == 0.0
    expect = np.where(zero[:, None], center if not asym else 0, best)
    miss = np.argwhere(expect != u)
    for r, i in miss:
        assert not zero[r]
        num = np.float32(x[r, i]) if not asym else np.float32(np.float32(x[r, i]) - np.float32(m[r]))
        q32 = float(np.float32(num / np.float32(d[r])))
        qex = (float(x[r, i]) - m[r]) / d[r]
        k = np.floor(qex) + 0.5
        assert (q32 - k) * (qex - k) <= 0 and q32 != qex, (f, x[r, i], u[r, i], expect[r, i])
    return len(miss)


@pytest.mark.parametrize("f", orc.LOWBIT)
def test_quantizer_exhaustive_minis(f):
    """Every code vector of a mini-block (k = 4 values for X <= 4, k = 2 above):
    dequantize with a fixed fp16 scale (and min), re-quantize, and require the
    nearest-code property; where the vector holds the extreme code(s) that
    reproduce the scale, the codes must come back exactly."""
    X = orc.fmt_bits(f)
    k = 4 if X <= 4 else 2
    cs = _code_set(f)
    d16 = int(orc.f32_to_f16_bits(np.array([0.0371], np.float32))[0])
    m16 = int(orc.f32_to_f16_bits(np.array([-0.4375], np.float32))[0])
    d, m = _f16(d16), _f16(m16)
    grids = np.array(np.meshgrid(*([cs] * k), indexing="ij")).reshape(k, -1).T
    N = grids.shape[0]
    xs = np.empty((N, k), np.float32)
    us = np.empty((N, k), np.uint8)
    ds = np.empty(N, np.int64)
    ms = np.empty(N, np.int64)
    for r, vec in enumerate(grids):
        x = np.array([_value(f, d, m, c) for c in vec], dtype=np.float32)
        u, dd, mm = orc.quantize_codes(f, x)
        xs[r], us[r], ds[r], ms[r] = x, u, dd, mm
    _check_nearest_batch(f, xs, us, ds, ms)
    if orc.fmt_asym(f):
        extreme = (grids.min(axis=1) == 0) & (grids.max(axis=1) == cs[-1])
    else:
        extreme = np.abs(grids - (1 << (X - 1))).max(axis=1) == (1 << (X - 1)) - 1
    assert extreme.any()
    assert (ds[extreme] == d16).all()
    assert (us[extreme] == grids[extreme]).all()
    if orc.fmt_asym(f):
        assert (ms[extreme] == m16).all()


@pytest.mark.parametrize("f", orc.LOWBIT)
def test_quantizer_idempotent_blocks(f):
    """Quantize a random block, dequantize it, quantize again: same bytes."""
    rng = np.random.default_rng(7 + f)
    for _ in range(200):
        x = rng.standard_normal(32).astype(np.float32)
        b1 = orc.quantize_row(f, x)
        y = orc.dequant_row(f, b1, 32)
        b2 = orc.quantize_row(f, y)
        assert (b1 == b2).all()


# --------------------------------------------------------------- serialisation
def _bitstring_pack(f, u, d16, m16):
    """Independent construction: build each plane as a list of bits."""
    X = orc.fmt_bits(f)
    widths = {8: [8], 6: [4, 2], 5: [4, 1], 4: [4], 3: [2, 1], 2: [2]}[X]
    out = [d16 & 0xFF, d16 >> 8]
    if orc.fmt_asym(f):
        out += [m16 & 0xFF, m16 >> 8]
    low = 0
    for w in widths:
        bitlist = []
        for code in u:
            field = (int(code) >> low) & ((1 << w) - 1)
            bitlist += [(field >> j) & 1 for j in range(w)]
        for byte in range(len(bitlist) // 8):
            out.append(sum(bitlist[8 * byte + j] << j for j in range(8)))
        low += w
    return np.array(out, dtype=np.uint8)


@pytest.mark.parametrize("f", orc.LOWBIT)
def test_pack_layout(f):
    rng = np.random.default_rng(f)
    cs = _code_set(f)
    for _ in range(50):
        u = rng.choice(cs, 32).astype(np.uint8)
        d16, m16 = int(rng.integers(0, 0x7C00)), int(rng.integers(0, 0xFC00))
        if not orc.fmt_asym(f):
            m16 = 0
        raw = orc.pack_block(f, u, d16, m16)
        assert raw.size == orc.block_bytes(f)
        assert (raw == _bitstring_pack(f, u, d16, m16)).all()
        u2, d2, m2 = orc.unpack_block(f, raw)
        assert (u2 == u).all() and d2 == d16 and m2 == m16
