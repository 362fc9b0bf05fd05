"""CPU-side checks of the C ABI library: it loads, exports every entry point the
header declares, validates arguments without a GPU, and its memory map equals
the block-size closed form (the KV-MiB table on "BeeLlama.cpp v0.4.1": at 64k
context, 16 attention layers x 4 KV heads x 256 dims, q8_0 = 2,176 MiB,
q6_0 = 1,664, q5_0 = 1,408, q4_0 = 1,152; a bf16 tail adds 64 MiB per 1,024
tokens)."""
import ctypes
import os
import re
import subprocess

import pytest

from quantized_mixed_precision_qx_b200 import kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    return re.findall(r"KVQ_API\s+[\w\s\*]+?\b(kvq_\w+)\s*\(", text)


def test_exports_every_header_symbol():
    syms = header_symbols()
    assert len(syms) == 17
    assert sorted(syms) == sorted(kvq.EXPORTED)
    out = subprocess.check_output(["nm", "-D", "--defined-only", kvq.LIB_PATH]).decode()
    exported = set(re.findall(r"\bT (kvq_\w+)", out))
    assert set(syms) <= exported
    L = kvq.lib()
    for s in syms:
        assert getattr(L, s) is not None


def _layout(L=16, B=1, H=4, Hq=24, D=256, ctx=65536, kvarn=0):
    return kvq.kvq_layout(L, B, H, Hq, D, kvarn, ctx, 512, 0, 1e-6)


def _meta(L=16, B=1, H=4):
    """The metadata region the cache adds after the block store: a 256-byte header and
    four 32-bit value bounds per (layer, batch element, kv head), rounded up to 256."""
    return -(-(256 + 16 * L * B * H) // 256) * 256


@pytest.mark.parametrize("fmt,mib", [(kvq.Q8_0, 2176), (kvq.Q6_0, 1664), (kvq.Q5_0, 1408), (kvq.Q4_0, 1152)])
def test_required_bytes_closed_form(fmt, mib):
    h = kvq.kvq_cache_create(_layout(), fmt, fmt, kvq.NONE, 0)
    assert kvq.kvq_cache_required_bytes(h) == mib * 2**20 + _meta()
    kvq.kvq_cache_destroy(h)
    for W in (1024, 2048):
        h = kvq.kvq_cache_create(_layout(), fmt, fmt, kvq.BF16, W)
        assert kvq.kvq_cache_required_bytes(h) == (mib + 64 * W // 1024) * 2**20 + _meta()
        kvq.kvq_cache_destroy(h)


def test_required_bytes_config_d():
    """Config D at 262,144 positions: (208 + 176) bytes x 4 heads x 16 layers per position
    plus a 2,048-row q8_0 ring of 272-byte rows."""
    h = kvq.kvq_cache_create(_layout(ctx=262144), kvq.Q6_0, kvq.Q5_0, kvq.Q8_0, 2048)
    assert kvq.kvq_cache_required_bytes(h) == 262144 * 384 * 64 + 2048 * 544 * 64 + _meta()
    kvq.kvq_cache_destroy(h)


@pytest.mark.parametrize("bad", [
    dict(D=96), dict(D=512), dict(Hq=36), dict(Hq=6, H=4), dict(ctx=0), dict(L=0),
])
def test_create_rejects_bad_layouts(bad):
    kw = dict(L=1, B=1, H=4, Hq=24, D=256, ctx=1024)
    kw.update(bad)
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_cache_create(_layout(**kw), kvq.Q4_0, kvq.Q4_0, kvq.NONE, 0)
    assert e.value.status == kvq.ERR_INVALID_ARG


def test_create_rejects_bad_formats():
    lay = _layout(L=1, ctx=1024)
    for kf, vf, tf, W, st in [(kvq.BF16, kvq.Q4_0, kvq.NONE, 0, kvq.ERR_UNSUPPORTED_FMT),
                              (kvq.Q4_0, kvq.NONE, kvq.NONE, 0, kvq.ERR_UNSUPPORTED_FMT),
                              (kvq.Q4_0, kvq.Q4_0, kvq.Q4_0, 16, kvq.ERR_UNSUPPORTED_FMT),
                              (kvq.Q4_0, kvq.Q4_0, kvq.Q8_0, 0, kvq.ERR_INVALID_ARG),
                              (kvq.Q4_0, kvq.Q4_0, kvq.NONE, 16, kvq.ERR_UNSUPPORTED_FMT),
                              (kvq.Q4_0, kvq.Q4_0, kvq.BF16, 4096, kvq.ERR_INVALID_ARG)]:
        with pytest.raises(kvq.KVQError) as e:
            kvq.kvq_cache_create(lay, kf, vf, tf, W)
        assert e.value.status == st, (kf, vf, tf, W)
    bad = _layout(L=1, ctx=1024, kvarn=1)
    bad.kvarn_calib_tokens = 500
    with pytest.raises(kvq.KVQError):
        kvq.kvq_cache_create(bad, kvq.Q4_0, kvq.Q4_0, kvq.NONE, 0)


def test_unbound_cache_launches_nothing():
    h = kvq.kvq_cache_create(_layout(L=2, ctx=1024), kvq.Q6_0, kvq.Q5_0, kvq.Q8_0, 128)
    fake = ctypes.c_void_p(1 << 20)
    L = kvq.lib()
    assert L.kvq_append(h, 0, fake, fake, 4, None) == kvq.ERR_NOT_BOUND
    assert L.kvq_decode_attention(h, 0, fake, ctypes.c_float(1.0), fake, fake, 1 << 20, None) == kvq.ERR_NOT_BOUND
    assert L.kvq_append(h, 2, fake, fake, 4, None) == kvq.ERR_INVALID_ARG
    assert L.kvq_append(h, 0, fake, fake, -1, None) == kvq.ERR_INVALID_ARG
    n = ctypes.c_int64(7)
    assert L.kvq_length(h, 0, ctypes.byref(n)) == kvq.OK and n.value == 0
    sz = ctypes.c_size_t()
    assert L.kvq_decode_workspace_bytes(h, 1, ctypes.byref(sz)) == kvq.ERR_NOT_BOUND
    assert L.kvq_cache_bind(h, ctypes.c_void_p(1 << 20 | 8), 1 << 40, None) == kvq.ERR_ALIGNMENT
    assert L.kvq_cache_bind(h, ctypes.c_void_p(1 << 20), 16, None) == kvq.ERR_CAPACITY
    kvq.kvq_cache_destroy(h)
    assert L.kvq_cache_destroy(None) == kvq.OK


def test_status_strings():
    for s in range(10):
        assert kvq.status_string(s)
    assert "unknown" in kvq.status_string(99)


def _declaration_comments():
    """(symbol, the comment block right above its declaration) for every KVQ_API function."""
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    out = []
    for m in re.finditer(r"KVQ_API\s+[\w\s\*]+?\b(kvq_\w+)\s*\(", text):
        head = text[:m.start()]
        end = head.rstrip().rfind("*/")
        start = head.rfind("/*", 0, end)
        between = head[end + 2:]
        # only #defines may sit between a comment and its declaration
        assert all(ln.strip() == "" or ln.strip().startswith("#define") for ln in between.splitlines()), m.group(1)
        out.append((m.group(1), head[start:end]))
    return out


def test_every_declaration_cites_its_passage():
    """Each entry point's comment names the page passage that defines the operation, or
    says that the pages have no counterpart (lifetime, status and deployment calls)."""
    decls = _declaration_comments()
    assert len(decls) == 17
    cites = ("[KVBENCH]", "[HARDNUM]", "[BEELLAMA]", "[OFFLOAD]")
    for sym, comment in decls:
        flat = " ".join(w for w in comment.split() if w not in ("*", "/*"))
        ok = any(c in flat for c in cites) or "no counterpart" in flat or "Nothing on the pages" in flat
        assert ok, f"{sym}: no citation in its comment"


def test_new_calls_validate_on_the_host():
    h = kvq.kvq_cache_create(_layout(L=1, ctx=1024), kvq.Q6_0, kvq.Q5_0, kvq.NONE, 0)
    L = kvq.lib()
    assert L.kvq_device_status(h, None) == kvq.ERR_NOT_BOUND
    assert L.kvq_selftest_wait_timeout(h, 1000, None) == kvq.ERR_NOT_BOUND
    assert L.kvq_get_channel_scales(h, 0, ctypes.c_void_p(16), ctypes.c_void_p(16)) == kvq.ERR_INVALID_ARG  # no KVarN
    assert L.kvq_device_status(None, None) == kvq.ERR_INVALID_ARG
    kvq.kvq_cache_destroy(h)
    hk = kvq.kvq_cache_create(_layout(L=1, ctx=1024, kvarn=1), kvq.Q6_0, kvq.Q5_0, kvq.NONE, 0)
    assert L.kvq_get_channel_scales(hk, 0, ctypes.c_void_p(16), ctypes.c_void_p(16)) == kvq.ERR_NOT_BOUND
    assert L.kvq_get_channel_scales(hk, 1, ctypes.c_void_p(16), ctypes.c_void_p(16)) == kvq.ERR_INVALID_ARG
    kvq.kvq_cache_destroy(hk)
