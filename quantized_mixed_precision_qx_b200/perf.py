"""Timing driver for single libkvq calls (used for the ncu captures under profiles/).

    python -m quantized_mixed_precision_qx_b200.perf decode  --n 131072 [shape/format options]
    python -m quantized_mixed_precision_qx_b200.perf prefill --n 32768 --chunk 1024
    python -m quantized_mixed_precision_qx_b200.perf append  --n 65536 --chunk 8192
    python -m quantized_mixed_precision_qx_b200.perf sweep   --n 32768 --step 1024

`sweep` fills the cache by appends of --step positions and times one decode after each
(the decode-after-append pattern of a generation loop), printing one JSON line per context.

The cache is filled with seeded device-generated inputs (K ~ N(0,1) with 8 channels per head
scaled x8, V ~ N(0,1)); the measured call is repeated --reps times (the first --warmup calls
untimed) with CUDA events, L2 flushed before every decode. Prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import statistics

FMTS = {"q2_0": 0, "q2_1": 1, "q3_0": 2, "q3_1": 3, "q4_0": 4, "q4_1": 5, "q5_0": 6, "q5_1": 7,
        "q6_0": 8, "q6_1": 9, "q8_0": 10, "q8_1": 11, "bf16": 12, "f16": 13, "none": 14}
BLOCK_BYTES = {0: 10, 1: 12, 2: 14, 3: 16, 4: 18, 5: 20, 6: 22, 7: 24, 8: 26, 9: 28, 10: 34, 11: 36, 12: 64, 13: 64}


def main():
    import torch
    from quantized_mixed_precision_qx_b200 import kvq

    ap = argparse.ArgumentParser()
    ap.add_argument("op", choices=["decode", "prefill", "append", "sweep"])
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--H", type=int, default=4)
    ap.add_argument("--Hq", type=int, default=24)
    ap.add_argument("--D", type=int, default=256)
    ap.add_argument("--n", type=int, default=131072, help="positions filled before the measured call")
    ap.add_argument("--chunk", type=int, default=8192, help="append chunk / prefill rows")
    ap.add_argument("--k", default="q6_0")
    ap.add_argument("--v", default="q5_0")
    ap.add_argument("--tail", default="q8_0")
    ap.add_argument("--W", type=int, default=2048)
    ap.add_argument("--kvarn", type=int, default=0)
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--step", type=int, default=1024, help="sweep: positions appended between decodes")
    ap.add_argument("--clean-flush", type=int, default=0,
                    help="after the 256 MB flush write, read another 256 MB so L2 holds clean lines")
    a = ap.parse_args()
    dev = torch.device("cuda")
    kf, vf, tf = FMTS[a.k], FMTS[a.v], FMTS[a.tail]
    W = a.W if tf != 14 else 0
    extra = a.chunk if a.op in ("prefill", "append") else 0
    cap = a.n + extra
    c = kvq.KVCache(1, a.B, a.H, a.Hq, a.D, cap, kf, vf, tf, W, kvarn=a.kvarn, device=dev,
                    ws_rows=a.chunk if a.op == "prefill" else 1)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234)
    scale = torch.ones(a.H, a.D, device=dev)
    for h in range(a.H):
        scale[h, torch.randperm(a.D, generator=gen, device=dev)[:8]] = 8.0

    def kv(rows):
        return (torch.randn(a.B, rows, a.H, a.D, device=dev, generator=gen) * scale,
                torch.randn(a.B, rows, a.H, a.D, device=dev, generator=gen))

    if a.op == "sweep":
        sweep(a, c, kv, kf, vf, tf, W, dev, gen)
        return
    t = 0
    while t < a.n:
        cc = min(8192, a.n - t)
        k, v = kv(cc)
        c.append(0, k, v)
        t += cc
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    times = []
    res = {"op": a.op, "n": a.n, "shape": [a.B, a.H, a.Hq, a.D], "k": a.k, "v": a.v, "tail": a.tail, "W": W}
    if a.op == "decode":
        q = torch.randn(a.B, a.Hq, a.D, device=dev, generator=gen) / math.sqrt(a.D)
        out = torch.empty_like(q)
        ws = c.ensure_workspace(1)
        for i in range(a.warmup + a.reps):
            flush.fill_(i & 0xFF)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            kvq.kvq_decode_attention(c.handle, 0, q, 1.0, out, ws, ws.numel())
            e1.record()
            torch.cuda.synchronize()
            if i >= a.warmup:
                times.append(e0.elapsed_time(e1) / 1e3)
        rk, rv = BLOCK_BYTES[kf] * a.D // 32, BLOCK_BYTES[vf] * a.D // 32
        rt = BLOCK_BYTES.get(tf, 0) * a.D // 32
        ring = min(a.n, W)
        nbytes = a.B * a.H * ((a.n - ring) * (rk + rv) + ring * 2 * rt) + 2 * a.B * a.Hq * a.D * 4
        tm = statistics.median(times)
        res.update(us=tm * 1e6, gbs=nbytes / tm / 1e9, algorithmic_bytes=nbytes)
    elif a.op == "prefill":
        k, v = kv(a.chunk)
        c.append(0, k, v)
        q = torch.randn(a.B, a.chunk, a.Hq, a.D, device=dev, generator=gen) / math.sqrt(a.D)
        out = torch.empty_like(q)
        ws = c.ensure_workspace(a.chunk)
        for i in range(a.warmup + a.reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            kvq.kvq_prefill_attention(c.handle, 0, q, a.chunk, 1.0, out, ws, ws.numel())
            e1.record()
            torch.cuda.synchronize()
            if i >= a.warmup:
                times.append(e0.elapsed_time(e1) / 1e3)
        keys = a.chunk * a.n + a.chunk * (a.chunk + 1) / 2
        flop = keys * a.Hq * 4 * a.D
        tm = min(times)
        res.update(ms=tm * 1e3, alg_tflops=flop / tm / 1e12, executed_tflops=3 * flop / tm / 1e12,
                   nan=bool(torch.isnan(out).any()))
    else:
        ins = [kv(a.chunk) for _ in range(a.warmup + a.reps)]
        for i, (k, v) in enumerate(ins):
            kvq.kvq_cache_bind(c.handle, c.dev, c.nbytes)
            for _ in range(a.n // a.chunk):
                c.append(0, k, v)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            c.append(0, k, v)
            e1.record()
            torch.cuda.synchronize()
            if i >= a.warmup:
                times.append(e0.elapsed_time(e1) / 1e3)
        tm = statistics.median(times)
        res.update(us=tm * 1e6, mtok_s=a.chunk * a.B / tm / 1e6)
    print(json.dumps(res), flush=True)


def decode_bytes(a, n, kf, vf, tf, W):
    rk, rv = BLOCK_BYTES[kf] * a.D // 32, BLOCK_BYTES[vf] * a.D // 32
    rt = BLOCK_BYTES.get(tf, 0) * a.D // 32
    ring = min(n, W)
    return a.B * a.H * ((n - ring) * (rk + rv) + ring * 2 * rt) + 2 * a.B * a.Hq * a.D * 4


def sweep(a, c, kv, kf, vf, tf, W, dev, gen):
    import torch
    from quantized_mixed_precision_qx_b200 import kvq
    q = torch.randn(a.B, a.Hq, a.D, device=dev, generator=gen) / math.sqrt(a.D)
    out = torch.empty_like(q)
    ws = c.ensure_workspace(1)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    clean = torch.ones(64 << 20, dtype=torch.int32, device=dev) if a.clean_flush else None
    chunks = [kv(a.step) for _ in range(a.n // a.step)]
    res = {}
    for rep in range(a.warmup + a.reps):
        kvq.kvq_cache_bind(c.handle, c.dev, c.nbytes)
        for i, (k, v) in enumerate(chunks):
            c.append(0, k, v)
            flush.fill_(rep & 0xFF)
            if clean is not None:
                clean.sum()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            kvq.kvq_decode_attention(c.handle, 0, q, 1.0, out, ws, ws.numel())
            e1.record()
            torch.cuda.synchronize()
            if rep >= a.warmup:
                res.setdefault(i, []).append(e0.elapsed_time(e1) / 1e3)
    for i, ts in sorted(res.items()):
        n = (i + 1) * a.step
        tm = statistics.median(ts)
        nb = decode_bytes(a, n, kf, vf, tf, W)
        print(json.dumps({"op": "decode", "n": n, "us": tm * 1e6, "gbs": nb / tm / 1e9,
                          "algorithmic_bytes": nb}), flush=True)


if __name__ == "__main__":
    main()
