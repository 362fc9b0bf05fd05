"""ctypes binding of libkvq (include/kvq.h): argument marshalling only.

Every function has the C name and passes plain pointers and sizes; device tensors
are torch CUDA tensors whose data_ptr() is handed to the library, and streams are
torch.cuda.Stream objects (or None for the current stream). The binding never
computes any part of the cache or attention itself, and it refuses to load
anything but the in-tree CUDA library: a missing libkvq.so raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvq.so")

# formats (kvq_fmt)
Q2_0, Q2_1, Q3_0, Q3_1, Q4_0, Q4_1, Q5_0, Q5_1, Q6_0, Q6_1, Q8_0, Q8_1, BF16, F16, NONE = range(15)
FMT_NAMES = ["q2_0", "q2_1", "q3_0", "q3_1", "q4_0", "q4_1", "q5_0", "q5_1",
             "q6_0", "q6_1", "q8_0", "q8_1", "bf16", "f16", "none"]

# status codes (kvq_status)
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_FMT, ERR_CAPACITY, ERR_CALIBRATION, ERR_EMPTY, \
    ERR_ALIGNMENT, ERR_NOT_BOUND, ERR_CUDA, ERR_DEVICE_TIMEOUT = range(10)

EXPORTED = ["kvq_cache_create", "kvq_cache_required_bytes", "kvq_cache_bind", "kvq_cache_destroy",
            "kvq_append", "kvq_decode_workspace_bytes", "kvq_decode_attention", "kvq_prefill_attention",
            "kvq_length", "kvq_set_channel_scales", "kvq_export_blocks", "kvq_status_string",
            "kvq_decode_attention_noalloc", "kvq_get_channel_scales", "kvq_device_status",
            "kvq_selftest_wait_timeout", "kvq_decode_attention_indexed"]
MAX_GATHER = 65536                    # KVQ_MAX_GATHER
NOALLOC_WORKSPACE_BYTES = 8 << 20     # KVQ_NOALLOC_WORKSPACE_MIB


class kvq_layout(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("batch", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("kvarn", ctypes.c_int32),
                ("max_ctx", ctypes.c_int64), ("kvarn_calib_tokens", ctypes.c_int32),
                ("k_per_channel", ctypes.c_int32), ("kvarn_eps", ctypes.c_double)]


class KVQError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


_lib = None


def lib():
    """Load libkvq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libkvq.so not built at {LIB_PATH}; run quantized_mixed_precision_qx_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        p, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        sigs = {
            "kvq_cache_create": [ctypes.POINTER(kvq_layout), i32, i32, i32, i32, ctypes.POINTER(p)],
            "kvq_cache_required_bytes": [p, ctypes.POINTER(sz)],
            "kvq_cache_bind": [p, p, sz, p],
            "kvq_cache_destroy": [p],
            "kvq_append": [p, i32, p, p, i32, p],
            "kvq_decode_workspace_bytes": [p, i32, ctypes.POINTER(sz)],
            "kvq_decode_attention": [p, i32, p, f32, p, p, sz, p],
            "kvq_prefill_attention": [p, i32, p, i32, f32, p, p, sz, p],
            "kvq_decode_attention_noalloc": [p, i32, p, f32, p, p],
            "kvq_decode_attention_indexed": [p, i32, p, f32, p, i32, p, p, sz, p],
            "kvq_length": [p, i32, ctypes.POINTER(i64)],
            "kvq_set_channel_scales": [p, i32, p, p, p],
            "kvq_get_channel_scales": [p, i32, p, p],
            "kvq_device_status": [p, p],
            "kvq_selftest_wait_timeout": [p, ctypes.c_uint64, p],
            "kvq_export_blocks": [p, i32, i32, i32, i32, i32, i64, i64, p, sz],
        }
        for name, args in sigs.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.kvq_status_string.argtypes = [ctypes.c_int]
        L.kvq_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().kvq_status_string(status).decode()


def _check(status: int, what: str):
    if status != OK:
        raise KVQError(status, what)


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(getattr(stream, "cuda_stream", stream))


def _dptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


# ---------------------------------------------------------------- same-name calls
def kvq_cache_create(layout: kvq_layout, k_fmt: int, v_fmt: int, tail_fmt: int, W: int):
    h = ctypes.c_void_p()
    _check(lib().kvq_cache_create(ctypes.byref(layout), k_fmt, v_fmt, tail_fmt, W, ctypes.byref(h)),
           "kvq_cache_create")
    return h


def kvq_cache_required_bytes(cache) -> int:
    n = ctypes.c_size_t()
    _check(lib().kvq_cache_required_bytes(cache, ctypes.byref(n)), "kvq_cache_required_bytes")
    return n.value


def kvq_cache_bind(cache, dev_buf, nbytes: int, stream=None):
    _check(lib().kvq_cache_bind(cache, _dptr(dev_buf), nbytes, _stream(stream)), "kvq_cache_bind")


def kvq_cache_destroy(cache):
    _check(lib().kvq_cache_destroy(cache), "kvq_cache_destroy")


def kvq_append(cache, layer: int, k, v, n_new: int, stream=None):
    _check(lib().kvq_append(cache, layer, _dptr(k), _dptr(v), n_new, _stream(stream)), "kvq_append")


def kvq_decode_workspace_bytes(cache, n_query_rows: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().kvq_decode_workspace_bytes(cache, n_query_rows, ctypes.byref(n)), "kvq_decode_workspace_bytes")
    return n.value


def kvq_decode_attention(cache, layer: int, q, scale: float, out, ws, ws_bytes: int, stream=None):
    _check(lib().kvq_decode_attention(cache, layer, _dptr(q), scale, _dptr(out), _dptr(ws), ws_bytes,
                                      _stream(stream)), "kvq_decode_attention")


def kvq_decode_attention_indexed(cache, layer: int, q, scale: float, idx, n_idx: int, out, ws, ws_bytes: int,
                                 stream=None):
    _check(lib().kvq_decode_attention_indexed(cache, layer, _dptr(q), scale, _dptr(idx), n_idx, _dptr(out),
                                              _dptr(ws), ws_bytes, _stream(stream)), "kvq_decode_attention_indexed")


def kvq_prefill_attention(cache, layer: int, q, n_chunk: int, scale: float, out, ws, ws_bytes: int, stream=None):
    _check(lib().kvq_prefill_attention(cache, layer, _dptr(q), n_chunk, scale, _dptr(out), _dptr(ws), ws_bytes,
                                       _stream(stream)), "kvq_prefill_attention")


def kvq_decode_attention_noalloc(cache, layer: int, q, scale: float, out, stream=None):
    """Decode with the library's fixed device array as workspace (no allocation)."""
    _check(lib().kvq_decode_attention_noalloc(cache, layer, _dptr(q), scale, _dptr(out), _stream(stream)),
           "kvq_decode_attention_noalloc")


def kvq_length(cache, layer: int) -> int:
    n = ctypes.c_int64()
    _check(lib().kvq_length(cache, layer, ctypes.byref(n)), "kvq_length")
    return n.value


def kvq_set_channel_scales(cache, layer: int, sK, sV, stream=None):
    _check(lib().kvq_set_channel_scales(cache, layer, _dptr(sK), _dptr(sV), _stream(stream)),
           "kvq_set_channel_scales")


def kvq_get_channel_scales(cache, layer: int, host_sK, host_sV):
    """host_sK, host_sV: writable float32 numpy arrays [batch][n_kv_heads][head_dim]."""
    _check(lib().kvq_get_channel_scales(cache, layer, ctypes.c_void_p(host_sK.ctypes.data),
                                        ctypes.c_void_p(host_sV.ctypes.data)), "kvq_get_channel_scales")


def kvq_device_status(cache, stream=None) -> int:
    """Status code (OK or ERR_DEVICE_TIMEOUT) of the cache's device status word; clears it."""
    return lib().kvq_device_status(cache, _stream(stream))


def kvq_selftest_wait_timeout(cache, limit_ns: int, stream=None):
    _check(lib().kvq_selftest_wait_timeout(cache, limit_ns, _stream(stream)), "kvq_selftest_wait_timeout")


def kvq_export_blocks(cache, layer: int, b: int, h: int, kv: int, region: int, pos0: int, count: int,
                      host_dst) -> None:
    """host_dst: a writable numpy uint8 array."""
    _check(lib().kvq_export_blocks(cache, layer, b, h, kv, region, pos0, count,
                                   ctypes.c_void_p(host_dst.ctypes.data), host_dst.nbytes), "kvq_export_blocks")


# ---------------------------------------------------------------- convenience owner
class KVCache:
    """Owns a descriptor plus the torch device buffer and workspace it is bound to."""

    def __init__(self, n_layers, batch, n_kv_heads, n_q_heads, head_dim, max_ctx, k_fmt, v_fmt,
                 tail_fmt=NONE, W=0, kvarn=0, calib=512, eps=1e-6, device="cuda", stream=None,
                 ws_rows=1, k_per_channel=0):
        import torch
        self.layout = kvq_layout(n_layers, batch, n_kv_heads, n_q_heads, head_dim, kvarn, max_ctx, calib,
                                 k_per_channel, eps)
        self.k_per_channel = k_per_channel
        self.B, self.H, self.Hq, self.D, self.L = batch, n_kv_heads, n_q_heads, head_dim, n_layers
        self.k_fmt, self.v_fmt, self.tail_fmt, self.W = k_fmt, v_fmt, tail_fmt, W
        self.handle = kvq_cache_create(self.layout, k_fmt, v_fmt, tail_fmt, W)
        self.nbytes = kvq_cache_required_bytes(self.handle)
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self.buf.data_ptr()) % 256
        self.dev = self.buf[off:off + self.nbytes]
        kvq_cache_bind(self.handle, self.dev, self.nbytes, stream)
        self.ws = None
        self.ensure_workspace(ws_rows)

    def ensure_workspace(self, rows):
        import torch
        need = kvq_decode_workspace_bytes(self.handle, rows)
        if self.ws is None or self.ws.numel() < need:
            self.ws = torch.empty(max(need, 16), dtype=torch.uint8, device=self.dev.device)
        return self.ws

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and _lib is not None:
            _lib.kvq_cache_destroy(h)
            self.handle = None

    def length(self, layer=0):
        return kvq_length(self.handle, layer)

    def append(self, layer, k, v, stream=None):
        assert k.is_contiguous() and v.is_contiguous() and k.shape == v.shape
        kvq_append(self.handle, layer, k, v, k.shape[1], stream)

    def decode(self, layer, q, scale=1.0, out=None, stream=None):
        import torch
        if out is None:
            out = torch.empty_like(q)
        ws = self.ensure_workspace(1)
        kvq_decode_attention(self.handle, layer, q, scale, out, ws, ws.numel(), stream)
        return out

    def decode_indexed(self, layer, q, idx, scale=1.0, out=None, stream=None):
        """idx: int32 device tensor [batch][n_kv_heads][n_idx]."""
        import torch
        if out is None:
            out = torch.empty_like(q)
        ws = self.ensure_workspace(1)
        kvq_decode_attention_indexed(self.handle, layer, q, scale, idx, idx.shape[2], out, ws, ws.numel(), stream)
        return out

    def prefill(self, layer, q, scale=1.0, out=None, stream=None):
        import torch
        if out is None:
            out = torch.empty_like(q)
        ws = self.ensure_workspace(q.shape[1])
        kvq_prefill_attention(self.handle, layer, q, q.shape[1], scale, out, ws, ws.numel(), stream)
        return out

    def set_channel_scales(self, layer, sK, sV, stream=None):
        kvq_set_channel_scales(self.handle, layer, sK, sV, stream)

    def channel_scales(self, layer):
        import numpy as np
        sK = np.empty((self.B, self.H, self.D), dtype=np.float32)
        sV = np.empty_like(sK)
        kvq_get_channel_scales(self.handle, layer, sK, sV)
        return sK, sV

    def row_bytes(self, region, kv):
        f = self.tail_fmt if region == 1 else (self.v_fmt if kv else self.k_fmt)
        bb = {Q2_0: 10, Q2_1: 12, Q3_0: 14, Q3_1: 16, Q4_0: 18, Q4_1: 20, Q5_0: 22, Q5_1: 24,
              Q6_0: 26, Q6_1: 28, Q8_0: 34, Q8_1: 36, BF16: 64, F16: 64}[f]
        return bb * (self.D // 32)

    def export(self, layer, b, h, kv, region, pos0, count):
        """region 0: low-bit rows (per-channel K: groups of D blocks); 1: ring slots;
        2 (per-channel K): pending slots as float32 rows."""
        import numpy as np
        if region == 2:
            n = count * self.D * 4
        elif region == 0 and kv == 0 and self.k_per_channel:
            n = count * self.row_bytes(0, 0) * 32
        else:
            n = count * self.row_bytes(region, kv)
        out = np.empty(n, dtype=np.uint8)
        kvq_export_blocks(self.handle, layer, b, h, kv, region, pos0, count, out)
        return out
