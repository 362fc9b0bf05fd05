"""Benchmark of the quantized-KV hot path on B200.

Workload ("config D" of "Hard numbers on Qwen3.8-27B's KV cache", section "KV cache
low-bit storage"): 1 attention layer, batch 1, 4 KV heads x 256 dims, 24 query heads
(GQA 6), K q6_0 / V q5_0, a 2,048-token q8_0 ring. One step grows the context from 0
to 32,768 by 32 appends of 1,024 tokens (the ring evicts and requantizes) with a decode
step after each append. Inputs are seeded synthetic tensors (K ~ N(0,1) with 8
outlier channels per head x8, V ~ N(0,1), q ~ N(0,1)/16), resident in HBM before the
timed region (the e2e figure copies them from pinned host memory instead).

Metric: decode attention effective HBM GB/s = algorithmic bytes a decode must read
(packed rows, scales, ring rows, q and out) / device time of the decode calls. The
cache fits in L2, so L2 is flushed (256 MB write) before every decode and outside the
decode's timing. Append throughput (Mtok/s, one position of all heads' K and V) is
reported beside it.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# workload constants
L_, B_, H_, HQ_, D_ = 1, 1, 4, 24, 256
CTX, CHUNK, W_ = 32768, 1024, 2048
K_FMT, V_FMT, T_FMT = 8, 6, 10                # q6_0, q5_0, q8_0
ROW_K, ROW_V, ROW_T = 208, 176, 272           # bytes per row at D = 256
WORKLOAD = "config D: 1 layer, batch 1, 4 KV heads x 256, 24 q heads, K q6_0 / V q5_0, " \
           "2048-token q8_0 ring; context 0 -> 32768 by 32 appends of 1024, decode after each"
METRIC = "quantized-KV decode attention effective HBM GB/s (% of peak); append Mtok/s"


def decode_bytes(n: int) -> int:
    """Algorithmic bytes of one decode at context n: every stored row of every kv
    head (low-bit rows below the window, ring rows inside it), plus q and out."""
    ring = min(n, W_)
    main = n - ring
    rows = B_ * H_ * (main * (ROW_K + ROW_V) + ring * 2 * ROW_T)
    return rows + 2 * B_ * HQ_ * D_ * 4


def append_bytes(n0: int, c: int, W: int = W_, rowk: int = ROW_K, rowv: int = ROW_V, rowt: int = ROW_T,
                 B: int = B_, H: int = H_, D: int = D_) -> int:
    """Algorithmic bytes of appending c positions at context n0: fp32 K and V input,
    ring writes of the positions that end in the window, ring reads of evicted rows,
    and the low-bit rows written."""
    if W == 0:
        return B * H * c * (2 * D * 4 + rowk + rowv)
    n1 = n0 + c
    in_ring = min(c, W)                                   # new rows written to the ring
    evicted = max(0, min(n0, n1 - W) - max(0, n0 - W))    # old ring rows requantized
    direct = max(0, c - W)                                # enter-and-leave rows
    low = evicted + direct
    per_bh = c * 2 * D * 4 + in_ring * 2 * rowt + evicted * 2 * rowt + low * (rowk + rowv)
    return B * H * per_bh


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        h.update(open(os.path.join(ROOT, p), "rb").read())
    return h.hexdigest()[:12]


DECODE_SOURCES = ["quantized_mixed_precision_qx_b200/csrc/kvq_attention.cu",
                  "quantized_mixed_precision_qx_b200/csrc/kvq_decode_tc.cuh",
                  "quantized_mixed_precision_qx_b200/csrc/kvq_mma.cuh",
                  "quantized_mixed_precision_qx_b200/csrc/kvq_tc_launch.cuh",
                  "quantized_mixed_precision_qx_b200/csrc/kvq_internal.cuh"]


def recorded_traffic():
    """Per-launch DRAM bytes of the decode kernels from the committed ncu summary, if it
    was taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    want = source_hash(DECODE_SOURCES)
    for line in open(p):
        f = line.split()
        if len(f) >= 3 and not line.startswith("#") and f[0] == "decode_config_d" and f[2] == want:
            return float(f[1])
    return None


class ClockSampler:
    """nvidia-smi samples during the timed region."""
    Q = "index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active," \
        "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown," \
        "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap"

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------ oracle arm
def oracle_sample(budget_s: float = 15.0):
    """Time the CPU oracle on the leading steps of the same schedule until the budget
    is spent. Returns (decode GB/s, append Mtok/s, threads, description)."""
    import oracle as orc
    from quantized_mixed_precision_qx_b200.synth import KVRecipe, Workload
    wl = Workload(L_, B_, H_, HQ_, D_, CTX, KVRecipe("outlier"), seed=0)
    threads = os.cpu_count() or 1
    c = orc.Cache(L_, B_, H_, HQ_, D_, CTX, K_FMT, V_FMT, T_FMT, W_, threads=threads)
    t_dec = t_app = 0.0
    bytes_dec = 0
    toks = 0
    steps = 0
    n = 0
    t_start = time.perf_counter()
    while n < CTX and time.perf_counter() - t_start < budget_s:
        k = wl.kv_chunk(0, n, n + CHUNK, "k")
        v = wl.kv_chunk(0, n, n + CHUNK, "v")
        t0 = time.perf_counter()
        c.append(0, k, v)
        t_app += time.perf_counter() - t0
        n += CHUNK
        toks += CHUNK
        q = wl.q_decode(0, n // CHUNK - 1)
        t0 = time.perf_counter()
        c.decode(0, q, 1.0)
        t_dec += time.perf_counter() - t0
        bytes_dec += decode_bytes(n)
        steps += 1
    desc = f"first {steps} of 32 (append 1024 + decode) steps of the workload, context up to {n}"
    return bytes_dec / t_dec / 1e9, toks * B_ / t_app / 1e6, threads, desc, steps


def run_reference(args, rank):
    if rank != 0:
        return
    vals = []
    for _ in range(max(1, args.steps)):
        gbs, mtok, threads, desc, _ = oracle_sample(budget_s=min(20.0, 120.0 / max(1, args.steps + args.warmup)))
        vals.append(gbs)
    v = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "append_mtok_s": mtok}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------ ranks
def max_over_ranks(values, world, device):
    """Element-wise maximum of per-rank times over all ranks (every rank gets the result).
    The tensor lives on `device` (a CUDA device under NCCL, the CPU under gloo)."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_gbs(world, bytes_per_rank, max_seconds):
    """Whole-job throughput of `world` replicas that each moved `bytes_per_rank` algorithmic
    bytes, timed as the slowest rank (weak scaling)."""
    return world * bytes_per_rank / max_seconds / 1e9


# ------------------------------------------------------------------------ CUDA arm
def run_kvq(args, rank, world):
    import torch
    import torch.distributed as dist
    from quantized_mixed_precision_qx_b200 import kvq
    from quantized_mixed_precision_qx_b200.synth import KVRecipe, Workload

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    wl = Workload(L_, B_, H_, HQ_, D_, CTX, KVRecipe("outlier"), seed=rank)
    k_all = torch.from_numpy(wl.kv_chunk(0, 0, CTX, "k"))        # [1][CTX][4][256]
    v_all = torch.from_numpy(wl.kv_chunk(0, 0, CTX, "v"))
    q_all = torch.from_numpy(np.stack([wl.q_decode(0, s) for s in range(CTX // CHUNK)]))
    k_dev, v_dev, q_dev = k_all.to(dev), v_all.to(dev), q_all.to(dev)
    k_chunks = [k_dev[:, i:i + CHUNK].contiguous() for i in range(0, CTX, CHUNK)]
    v_chunks = [v_dev[:, i:i + CHUNK].contiguous() for i in range(0, CTX, CHUNK)]
    out_dev = torch.empty(CTX // CHUNK, B_, HQ_, D_, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    cache = kvq.KVCache(L_, B_, H_, HQ_, D_, CTX, K_FMT, V_FMT, T_FMT, W_, device=dev)
    h = cache.handle
    ws = cache.ensure_workspace(1)
    n_steps = CTX // CHUNK

    def rebind():
        kvq.kvq_cache_bind(h, cache.dev, cache.nbytes, stream)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(2 * n_steps)]

    def device_step():
        rebind()
        for s in range(n_steps):
            a0, a1 = ev[2 * s]
            a0.record(stream)
            kvq.kvq_append(h, 0, k_chunks[s], v_chunks[s], CHUNK, stream)
            a1.record(stream)
            flush.fill_(s & 0xFF)
            d0, d1 = ev[2 * s + 1]
            d0.record(stream)
            kvq.kvq_decode_attention(h, 0, q_dev[s], 1.0, out_dev[s], ws, ws.numel(), stream)
            d1.record(stream)

    def step_times():
        app = sum(ev[2 * s][0].elapsed_time(ev[2 * s][1]) for s in range(n_steps)) / 1e3
        dec = sum(ev[2 * s + 1][0].elapsed_time(ev[2 * s + 1][1]) for s in range(n_steps)) / 1e3
        return app, dec

    dec_bytes = sum(decode_bytes((s + 1) * CHUNK) for s in range(n_steps))
    app_bytes = sum(append_bytes(s * CHUNK, CHUNK) for s in range(n_steps))
    # launches of libkvq kernels per step: append 1 each; decode = low-bit pass (n > W),
    # ring pass (always, W > 0) and the merge
    launches = sum(1 + (1 if (s + 1) * CHUNK > W_ else 0) + 1 + 1 for s in range(n_steps))

    for _ in range(args.warmup):
        device_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    t_step0 = torch.cuda.Event(enable_timing=True)
    t_step1 = torch.cuda.Event(enable_timing=True)
    app_t = dec_t = 0.0
    dec_per_step = []
    torch.cuda.synchronize()
    t_step0.record(stream)
    for _ in range(args.steps):
        device_step()
        torch.cuda.synchronize()
        a, d = step_times()
        app_t += a
        dec_t += d
        dec_per_step.append(d)
    t_step1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clock_info = clocks.stop()
    step_ms = t_step0.elapsed_time(t_step1) / args.steps

    # ---- end to end: pinned host inputs, copies inside the timed region
    k_host = [c.cpu().pin_memory() for c in k_chunks]
    v_host = [c.cpu().pin_memory() for c in v_chunks]
    q_host = q_all.pin_memory()
    out_host = torch.empty(n_steps, B_, HQ_, D_).pin_memory()
    # inputs are double-buffered on the device and copied on a second stream, so the copy of
    # step s + 1's inputs overlaps the append and decode of step s (all inside the timing)
    copy_stream = torch.cuda.Stream(device=dev)
    k_in = [torch.empty_like(k_chunks[0]) for _ in range(2)]
    v_in = [torch.empty_like(v_chunks[0]) for _ in range(2)]
    q_in = [torch.empty(B_, HQ_, D_, device=dev) for _ in range(2)]
    copied = [torch.cuda.Event() for _ in range(n_steps)]
    consumed = [torch.cuda.Event() for _ in range(n_steps)]
    started = torch.cuda.Event()

    def issue_copy(s):
        b = s & 1
        with torch.cuda.stream(copy_stream):
            if s >= 2:
                copy_stream.wait_event(consumed[s - 2])      # buffer b is free again
            k_in[b].copy_(k_host[s], non_blocking=True)
            v_in[b].copy_(v_host[s], non_blocking=True)
            q_in[b].copy_(q_host[s], non_blocking=True)
            copied[s].record(copy_stream)

    def e2e_step():
        rebind()
        started.record(stream)
        copy_stream.wait_event(started)                      # no copy starts before the step
        issue_copy(0)
        for s in range(n_steps):
            if s + 1 < n_steps:
                issue_copy(s + 1)
            b = s & 1
            stream.wait_event(copied[s])
            kvq.kvq_append(h, 0, k_in[b], v_in[b], CHUNK, stream)
            kvq.kvq_decode_attention(h, 0, q_in[b], 1.0, out_dev[s], ws, ws.numel(), stream)
            consumed[s].record(stream)
            out_host[s].copy_(out_dev[s], non_blocking=True)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_s = e0.elapsed_time(e1) / 1e3 / args.steps
    h2d = n_steps * (2 * k_chunks[0].numel() * 4 + B_ * HQ_ * D_ * 4)
    d2h = n_steps * B_ * HQ_ * D_ * 4

    # ---- max over ranks
    dec_t, app_t, e2e_s, step_ms = max_over_ranks([dec_t, app_t, e2e_s, step_ms], world, dev)

    if rank != 0:
        return
    peak, peak_kind = read_peaks()
    value = whole_job_gbs(world, dec_bytes * args.steps, dec_t)
    achieved = dec_bytes * args.steps / dec_t / 1e9          # per GPU
    traffic = recorded_traffic()
    extra = supplementary(dev, peak) if not args.no_extra else None
    cpu = None
    if world == 1:
        gbs, mtok, threads, desc, _ = oracle_sample(budget_s=15.0)
        cpu = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc,
               "append_mtok_s": mtok}
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "l2": "flushed (256 MB write) before every decode, outside its timing",
                   "parallelism": f"replicas x{world}"},
        "decode_frac_of_peak": achieved / peak,
        "append_mtok_s": world * CTX * B_ * args.steps / app_t / 1e6,
        "append_gbs": world * app_bytes * args.steps / app_t / 1e9,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "peak_source": peak_kind,
                     "kernel": "decode (split-K pass 1 + merge), per call, summed over the 32 decodes of a step",
                     "algorithmic_bytes_per_step": dec_bytes},
        "cpu_baseline": cpu,
        "e2e": {"value": world * dec_bytes / e2e_s / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "note": "decode bytes / whole step time with appends and host copies"},
        "gpu_launches": launches * args.steps,
        "clocks": clock_info,
        "workloads": extra,
    }
    print(json.dumps(line), flush=True)


def supplementary(dev, peak):
    """Decode / append / prefill figures on the large workloads (one GPU, device-generated
    seeded inputs; parity for these shapes is covered by the tests). Each decode is timed
    with L2 flushed before it; caches are larger than L2 anyway."""
    import torch
    from quantized_mixed_precision_qx_b200 import kvq
    res = {}
    gen = torch.Generator(device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def rows_bytes(fmt, D):
        bb = {0: 10, 1: 12, 2: 14, 3: 16, 4: 18, 5: 20, 6: 22, 7: 24, 8: 26, 9: 28, 10: 34, 11: 36, 12: 64, 13: 64}[fmt]
        return bb * D // 32

    def fill(c, B, H, D, n, outlier=True, chunk=8192):
        gen.manual_seed(1234)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tot = 0.0
        t = 0
        scale = torch.ones(H, D, device=dev)
        if outlier:
            for h in range(H):
                scale[h, torch.randperm(D, generator=gen, device=dev)[:8]] = 8.0
        while t < n:
            cc = min(chunk, n - t)
            k = torch.randn(B, cc, H, D, device=dev, generator=gen) * scale
            v = torch.randn(B, cc, H, D, device=dev, generator=gen)
            torch.cuda.synchronize()
            ev0.record()
            c.append(0, k, v)
            ev1.record()
            torch.cuda.synchronize()
            tot += ev0.elapsed_time(ev1) / 1e3
            t += cc
            del k, v
        return tot

    def time_decode(c, B, Hq, D, reps=10):
        q = torch.randn(B, Hq, D, device=dev, generator=gen) / math.sqrt(D)
        out = torch.empty_like(q)
        ws = c.ensure_workspace(1)
        ts = []
        for i in range(reps + 3):
            flush.fill_(i & 0xFF)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            kvq.kvq_decode_attention(c.handle, 0, q, 1.0, out, ws, ws.numel())
            e1.record()
            torch.cuda.synchronize()
            if i >= 3:
                ts.append(e0.elapsed_time(e1) / 1e3)
        return statistics.median(ts)

    # full-length hybrid-model layer: fill 257,984, prefill 4,096, decode at 262,080
    B, H, Hq, D, W = 1, 4, 24, 256, 2048
    n_fill, C = 257984, 4096
    c = kvq.KVCache(1, B, H, Hq, D, 262144, K_FMT, V_FMT, T_FMT, W, device=dev, ws_rows=C)
    t_fill = fill(c, B, H, D, n_fill)
    fill_bytes = sum(append_bytes(t, min(8192, n_fill - t), W, ROW_K, ROW_V, ROW_T, B, H, D)
                     for t in range(0, n_fill, 8192))
    gen.manual_seed(99)
    kc = torch.randn(B, C, H, D, device=dev, generator=gen)
    vc = torch.randn(B, C, H, D, device=dev, generator=gen)
    c.append(0, kc, vc)
    n = n_fill + C
    q = torch.randn(B, C, Hq, D, device=dev, generator=gen) / math.sqrt(D)
    out = torch.empty_like(q)
    ws = c.ensure_workspace(C)
    kvq.kvq_prefill_attention(c.handle, 0, q, C, 1.0, out, ws, ws.numel())
    torch.cuda.synchronize()
    pts = []
    for _ in range(2):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        kvq.kvq_prefill_attention(c.handle, 0, q, C, 1.0, out, ws, ws.numel())
        e1.record()
        torch.cuda.synchronize()
        pts.append(e0.elapsed_time(e1) / 1e3)
    keys = C * n_fill + C * (C + 1) / 2
    pflop = keys * Hq * 4 * D
    tp = min(pts)
    td = time_decode(c, B, Hq, D)
    dbytes = B * H * ((n - W) * (ROW_K + ROW_V) + W * 2 * ROW_T) + 2 * B * Hq * D * 4
    res["full_length_layer"] = {
        "decode_gbs": dbytes / td / 1e9, "decode_frac": dbytes / td / 1e9 / peak, "decode_us": td * 1e6,
        "context": n, "append_fill_mtok_s": n_fill * B / t_fill / 1e6,
        "append_fill_gbs": fill_bytes / t_fill / 1e9, "append_fill_frac": fill_bytes / t_fill / 1e9 / peak,
        "prefill_ms": tp * 1e3, "prefill_alg_tflops": pflop / tp / 1e12,
        "prefill_executed_tflops": 3 * pflop / tp / 1e12,
        "note": "prefill FLOP = 4 x keys x heads x D (causal count); executed = 3 split-operand passes"}
    del c, kc, vc, q, out, ws
    torch.cuda.empty_cache()

    # KVarN: batch 8, 2 kv heads, 131,072 positions
    B, H, Hq, D, n = 8, 2, 16, 256, 131072
    c = kvq.KVCache(1, B, H, Hq, D, n, K_FMT, V_FMT, 14, 0, kvarn=1, device=dev)
    t_fill = fill(c, B, H, D, n, chunk=4096)
    fill_bytes = B * H * n * (2 * D * 4 + ROW_K + ROW_V)
    td = time_decode(c, B, Hq, D)
    dbytes = B * H * n * (ROW_K + ROW_V) + 2 * B * Hq * D * 4
    res["kvarn"] = {"decode_gbs": dbytes / td / 1e9, "decode_frac": dbytes / td / 1e9 / peak, "decode_us": td * 1e6,
                    "append_fill_mtok_s": n * B / t_fill / 1e6, "append_fill_gbs": fill_bytes / t_fill / 1e9,
                    "append_fill_frac": fill_bytes / t_fill / 1e9 / peak}
    del c
    torch.cuda.empty_cache()

    # asymmetric low-bit sweep: batch 4, 4 kv heads, 65,536 positions, bf16 tail 1,024
    B, H, Hq, D, n, W = 4, 4, 24, 256, 65536, 1024
    sweep = {}
    for kf, vf, name in [(5, 5, "q4_1/q4_1"), (5, 3, "q4_1/q3_1"), (3, 1, "q3_1/q2_1"), (0, 0, "q2_0/q2_0")]:
        c = kvq.KVCache(1, B, H, Hq, D, n, kf, vf, 12, W, device=dev)
        fill(c, B, H, D, n, outlier=False)
        td = time_decode(c, B, Hq, D)
        dbytes = B * H * ((n - W) * (rows_bytes(kf, D) + rows_bytes(vf, D)) + W * 2 * 512) + 2 * B * Hq * D * 4
        sweep[name] = {"decode_gbs": dbytes / td / 1e9, "decode_frac": dbytes / td / 1e9 / peak}
        del c
        torch.cuda.empty_cache()
    res["asymmetric_sweep"] = sweep
    res["quality_rel_l2_vs_fp32"] = quality(dev)
    return res


FMT_NAMES = ["q2_0", "q2_1", "q3_0", "q3_1", "q4_0", "q4_1", "q5_0", "q5_1", "q6_0", "q6_1", "q8_0", "q8_1"]


def quality(dev):
    """Relative L2 error of the decode output against softmax attention over the unquantized
    fp32 inputs (computed in float64), per format: K = V = the format, no tail, plus the
    config D formats with their q8_0 tail. Batch 1, 4 KV heads x 256, 24 query heads, 8192
    positions with 8 outlier K channels per head (x8), 4 query vectors."""
    import torch
    from quantized_mixed_precision_qx_b200 import kvq
    B, H, Hq, D, n, nq = 1, 4, 24, 256, 8192, 4
    G = Hq // H
    gen = torch.Generator(device=dev)
    gen.manual_seed(2024)
    scale = torch.ones(H, D, device=dev)
    for h in range(H):
        scale[h, torch.randperm(D, generator=gen, device=dev)[:8]] = 8.0
    k = torch.randn(B, n, H, D, device=dev, generator=gen) * scale
    v = torch.randn(B, n, H, D, device=dev, generator=gen)
    qs = [torch.randn(B, Hq, D, device=dev, generator=gen) / math.sqrt(D) for _ in range(nq)]
    # exact reference: query head j reads KV head j // G
    kk = k.double().permute(0, 2, 1, 3).repeat_interleave(G, dim=1)      # [B][Hq][n][D]
    vv = v.double().permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    refs = [torch.softmax(torch.einsum("bhd,bhnd->bhn", q.double(), kk), dim=-1).unsqueeze(2).matmul(vv).squeeze(2)
            for q in qs]
    cases = [(name, f, f, kvq.NONE, 0) for f, name in enumerate(FMT_NAMES)]
    cases.append(("q6_0/q5_0 + q8_0 tail 2048", K_FMT, V_FMT, T_FMT, W_))
    res = {}
    for name, kf, vf, tf, W in cases:
        c = kvq.KVCache(1, B, H, Hq, D, n, kf, vf, tf, W, device=dev)
        for t in range(0, n, 4096):
            c.append(0, k[:, t:t + 4096].contiguous(), v[:, t:t + 4096].contiguous())
        ws = c.ensure_workspace(1)
        num = den = 0.0
        for q, ref in zip(qs, refs):
            out = torch.empty_like(q)
            kvq.kvq_decode_attention(c.handle, 0, q, 1.0, out, ws, ws.numel())
            torch.cuda.synchronize()
            num += float(((out.double() - ref) ** 2).sum())
            den += float((ref ** 2).sum())
        res[name] = math.sqrt(num / den)
        del c
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--no-extra", action="store_true", help="skip the large-workload figures")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_kvq(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
