"""CPU oracle for the block-quantized, mixed-precision KV cache.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the benchmark's
CPU-baseline leg are the only callers. The product path never imports this
package, and this package imports nothing from the product.

The arithmetic lives in ``kvq_oracle.cpp`` (plain scalar C++, fp64 attention);
this module builds it with g++ and wraps it with ctypes and numpy.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.cpp")
_LIB = os.path.join(_HERE, "libkvq_oracle.so")

# Format ids: same numbering as the public ABI's enum (interface contract).
Q2_0, Q2_1, Q3_0, Q3_1, Q4_0, Q4_1, Q5_0, Q5_1, Q6_0, Q6_1, Q8_0, Q8_1, BF16, F16, NONE = range(15)
LOWBIT = list(range(12))
FMT_NAMES = ["q2_0", "q2_1", "q3_0", "q3_1", "q4_0", "q4_1", "q5_0", "q5_1",
             "q6_0", "q6_1", "q8_0", "q8_1", "bf16", "f16", "none"]


def build(force: bool = False) -> str:
    """Compile the oracle (no FMA contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c++17",
                               "-shared", "-fPIC", "-o", tmp, _SRC, "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        c_i, c_i64, c_f, c_d, c_p = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_void_p
        sig = {
            "orc_fmt_bits": (c_i, [c_i]),
            "orc_fmt_asym": (c_i, [c_i]),
            "orc_block_bytes": (c_i, [c_i]),
            "orc_f32_to_f16_array": (None, [c_p, c_p, c_i64]),
            "orc_f32_to_bf16_array": (None, [c_p, c_p, c_i64]),
            "orc_f16_to_f32_array": (None, [c_p, c_p, c_i64]),
            "orc_quantize_codes": (c_i, [c_i, c_p, c_i, c_p, c_p, c_p]),
            "orc_dequant_code": (c_f, [c_i, ctypes.c_uint16, ctypes.c_uint16, c_i]),
            "orc_pack_block": (c_i, [c_i, c_p, ctypes.c_uint16, ctypes.c_uint16, c_p]),
            "orc_unpack_block": (c_i, [c_i, c_p, c_p, c_p, c_p]),
            "orc_quantize_row": (c_i, [c_i, c_p, c_i, c_p]),
            "orc_dequant_row": (c_i, [c_i, c_p, c_i, c_p]),
            "orc_cache_new": (c_p, [c_i, c_i, c_i, c_i, c_i, c_i64, c_i, c_i, c_i, c_i, c_i, c_i, c_d, c_i]),
            "orc_cache_free": (None, [c_p]),
            "orc_length": (c_i64, [c_p, c_i]),
            "orc_set_channel_scales": (c_i, [c_p, c_i, c_p, c_p]),
            "orc_get_channel_scales": (c_i, [c_p, c_i, c_p, c_p]),
            "orc_append": (c_i, [c_p, c_i, c_p, c_p, c_i, c_i]),
            "orc_export": (c_i, [c_p, c_i, c_i, c_i, c_i, c_i, c_i64, c_i64, c_p]),
            "orc_position_row": (c_i, [c_p, c_i, c_i, c_i, c_i, c_i64, c_p]),
            "orc_decode": (c_i, [c_p, c_i, c_p, c_f, c_p, c_i]),
            "orc_decode_indexed": (c_i, [c_p, c_i, c_p, c_f, c_p, c_i, c_p, c_i]),
            "orc_prefill": (c_i, [c_p, c_i, c_p, c_i, c_f, c_p, c_p, c_i, c_i]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def fmt_bits(f): return lib().orc_fmt_bits(f)
def fmt_asym(f): return bool(lib().orc_fmt_asym(f))
def block_bytes(f): return lib().orc_block_bytes(f)


def row_bytes(f, D):
    return block_bytes(f) * (D // 32)


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    y = np.empty(x.shape, dtype=np.uint16)
    lib().orc_f32_to_f16_array(_ptr(x), _ptr(y), x.size)
    return y


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    y = np.empty(x.shape, dtype=np.uint16)
    lib().orc_f32_to_bf16_array(_ptr(x), _ptr(y), x.size)
    return y


def f16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    y = np.empty(h.shape, dtype=np.float32)
    lib().orc_f16_to_f32_array(_ptr(h), _ptr(y), h.size)
    return y


def quantize_codes(f, x):
    """(codes uint8[k], d16, m16) for k <= 32 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = np.empty(x.size, dtype=np.uint8)
    d = np.zeros(1, dtype=np.uint16)
    m = np.zeros(1, dtype=np.uint16)
    rc = lib().orc_quantize_codes(f, _ptr(x), x.size, _ptr(u), _ptr(d), _ptr(m))
    assert rc == 0
    return u, int(d[0]), int(m[0])


def dequant_code(f, d16, m16, u):
    return lib().orc_dequant_code(f, d16, m16, int(u))


def pack_block(f, codes, d16, m16):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    assert codes.size == 32
    out = np.empty(block_bytes(f), dtype=np.uint8)
    assert lib().orc_pack_block(f, _ptr(codes), d16, m16, _ptr(out)) == 0
    return out


def unpack_block(f, raw):
    raw = np.ascontiguousarray(raw, dtype=np.uint8)
    u = np.empty(32, dtype=np.uint8)
    d = np.zeros(1, dtype=np.uint16)
    m = np.zeros(1, dtype=np.uint16)
    assert lib().orc_unpack_block(f, _ptr(raw), _ptr(u), _ptr(d), _ptr(m)) == 0
    return u, int(d[0]), int(m[0])


def quantize_row(f, x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(row_bytes(f, x.size), dtype=np.uint8)
    assert lib().orc_quantize_row(f, _ptr(x), x.size, _ptr(out)) == 0
    return out


def dequant_row(f, raw, D):
    raw = np.ascontiguousarray(raw, dtype=np.uint8)
    out = np.empty(D, dtype=np.float32)
    assert lib().orc_dequant_row(f, _ptr(raw), D, _ptr(out)) == 0
    return out


class OracleError(RuntimeError):
    def __init__(self, code, what):
        super().__init__(f"oracle {what} returned status {code}")
        self.code = code


class Cache:
    """Oracle cache: same semantics as the library's cache, canonical bytes."""

    def __init__(self, n_layers, batch, n_kv_heads, n_q_heads, head_dim, max_ctx,
                 k_fmt, v_fmt, tail_fmt=NONE, W=0, kvarn=0, calib=512, eps=1e-6, threads=None, kivi=0):
        self.L, self.B, self.H, self.Hq, self.D = n_layers, batch, n_kv_heads, n_q_heads, head_dim
        self.max_ctx, self.kf, self.vf, self.tf, self.W = max_ctx, k_fmt, v_fmt, tail_fmt, W
        self.kivi = kivi
        self.threads = threads or (os.cpu_count() or 1)
        self._h = lib().orc_cache_new(n_layers, batch, n_kv_heads, n_q_heads, head_dim, max_ctx,
                                      k_fmt, v_fmt, tail_fmt, W, kvarn, calib, eps, kivi)
        if not self._h:
            raise ValueError("oracle rejected the cache description")

    def __del__(self):
        if getattr(self, "_h", None):
            lib().orc_cache_free(self._h)
            self._h = None

    def _chk(self, rc, what):
        if rc != 0:
            raise OracleError(rc, what)

    def length(self, layer):
        return lib().orc_length(self._h, layer)

    def append(self, layer, k, v):
        k = np.ascontiguousarray(k, dtype=np.float32)
        v = np.ascontiguousarray(v, dtype=np.float32)
        assert k.shape == v.shape and k.shape[0] == self.B and k.shape[2:] == (self.H, self.D)
        self._chk(lib().orc_append(self._h, layer, _ptr(k), _ptr(v), k.shape[1], self.threads), "append")

    def set_channel_scales(self, layer, sK, sV):
        sK = np.ascontiguousarray(sK, dtype=np.float32)
        sV = np.ascontiguousarray(sV, dtype=np.float32)
        self._chk(lib().orc_set_channel_scales(self._h, layer, _ptr(sK), _ptr(sV)), "set_channel_scales")

    def channel_scales(self, layer):
        sK = np.empty((self.B, self.H, self.D), dtype=np.float32)
        sV = np.empty_like(sK)
        self._chk(lib().orc_get_channel_scales(self._h, layer, _ptr(sK), _ptr(sV)), "channel_scales")
        return sK, sV

    def export(self, layer, b, h, kv, region, pos0, count):
        """region 0: low-bit rows pos0.. (per-channel K: groups pos0.., D blocks each);
        region 1: ring slots; region 2 (per-channel K): pending slots as fp32 rows."""
        f = (self.tf if region == 1 else (self.vf if kv else self.kf))
        if region == 2:
            out = np.empty(count * self.D * 4, dtype=np.uint8)
        elif region == 0 and kv == 0 and self.kivi:
            out = np.empty(count * self.D * block_bytes(self.kf), dtype=np.uint8)
        else:
            out = np.empty(count * row_bytes(f, self.D), dtype=np.uint8)
        self._chk(lib().orc_export(self._h, layer, b, h, kv, region, pos0, count, _ptr(out)), "export")
        return out

    def position_row(self, layer, b, h, kv, pos):
        out = np.empty(self.D, dtype=np.float32)
        self._chk(lib().orc_position_row(self._h, layer, b, h, kv, pos, _ptr(out)), "position_row")
        return out

    def decode(self, layer, q, scale=1.0):
        q = np.ascontiguousarray(q, dtype=np.float32)
        assert q.shape == (self.B, self.Hq, self.D)
        out = np.zeros_like(q)
        self._chk(lib().orc_decode(self._h, layer, _ptr(q), scale, _ptr(out), self.threads), "decode")
        return out

    def decode_indexed(self, layer, q, idx, scale=1.0):
        """Decode over the positions listed per (batch, kv head): idx int32 [B][H][k]."""
        q = np.ascontiguousarray(q, dtype=np.float32)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        assert q.shape == (self.B, self.Hq, self.D) and idx.shape[:2] == (self.B, self.H)
        out = np.zeros_like(q)
        self._chk(lib().orc_decode_indexed(self._h, layer, _ptr(q), scale, _ptr(idx), idx.shape[2], _ptr(out),
                                           self.threads), "decode_indexed")
        return out

    def prefill(self, layer, q, scale=1.0, rows=None):
        q = np.ascontiguousarray(q, dtype=np.float32)
        assert q.shape[0] == self.B and q.shape[2:] == (self.Hq, self.D)
        C = q.shape[1]
        out = np.zeros_like(q)
        if rows is None:
            rc = lib().orc_prefill(self._h, layer, _ptr(q), C, scale, _ptr(out), None, 0, self.threads)
        else:
            r = np.ascontiguousarray(rows, dtype=np.int32)
            rc = lib().orc_prefill(self._h, layer, _ptr(q), C, scale, _ptr(out), _ptr(r), r.size, self.threads)
        self._chk(rc, "prefill")
        return out
