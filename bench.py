"""Benchmark of the quantized-KV hot path on B200.

Workload (the full-length hybrid-model cache of "Hard numbers on Qwen3.8-27B's KV cache",
section "KV cache low-bit storage": 262k context on the model's 16 attention layers):
16 attention layers, batch 1, 4 KV heads x 256 dims, 24 query heads (GQA 6), K q6_0 /
V q5_0, a 2,048-token q8_0 ring. One step runs the whole schedule from an empty cache:
  1. fill: 257,984 positions per layer in appends of 8,192 (quantize-on-append, ring
     eviction and requantization);
  2. per layer: append the 4,096-position prompt chunk and run its causal chunked prefill;
  3. 64 decode steps, each appending one position to every layer and attending over it
     (contexts 262,081 .. 262,144).
Inputs are seeded synthetic tensors generated on the device (K ~ N(0,1) with 8 outlier
channels per head x8, V ~ N(0,1), q ~ N(0,1)/16), resident in HBM before the timed region;
each layer's cache (404 MB) is larger than L2, and consecutive decodes read different layers.

Metric: decode attention effective HBM GB/s = algorithmic bytes the decodes must read
(packed rows, scales, ring rows, q and out) / device time of the 1,024 decode calls of a
step (CUDA events around each call, on the launching stream). Append (fill) and prefill
figures of the same step are reported beside it, each with its own roofline.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import platform
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# workload constants (full-length hybrid-model cache)
L_, B_, H_, HQ_, D_ = 16, 1, 4, 24, 256
N_FILL, C_PF, N_DEC = 257984, 4096, 64
CTX = N_FILL + C_PF + N_DEC                     # 262,144
W_ = 2048
FILL_CHUNK = 8192
K_FMT, V_FMT, T_FMT = 8, 6, 10                # q6_0, q5_0, q8_0
ROW_K, ROW_V, ROW_T = 208, 176, 272           # bytes per row at D = 256
WORKLOAD = ("full-length hybrid-model cache: 16 attention layers, batch 1, 4 KV heads x 256, 24 q heads, "
            "K q6_0 / V q5_0, 2048-token q8_0 ring; per step: fill 257,984 (appends of 8,192), append + "
            "prefill a 4,096-row chunk per layer, then 64 x (append 1 + decode) over all 16 layers "
            "(context 262,081..262,144)")
METRIC = "quantized-KV decode attention effective HBM GB/s (% of peak); append Mtok/s"

# config D (latency-bound extra: 1 layer, 32 appends of 1,024 to 32,768, decode after each)
CD_CTX, CD_CHUNK = 32768, 1024


def decode_bytes(n: int, W: int = W_, rowk: int = ROW_K, rowv: int = ROW_V, rowt: int = ROW_T,
                 B: int = B_, H: int = H_, Hq: int = HQ_, D: int = D_) -> int:
    """Algorithmic bytes of one decode of one layer at context n: every stored row of every
    kv head (low-bit rows below the window, ring rows inside it), plus q and out."""
    ring = min(n, W)
    main = n - ring
    rows = B * H * (main * (rowk + rowv) + ring * 2 * rowt)
    return rows + 2 * B * Hq * D * 4


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


def prefill_flops(n_before: int, C: int, Hq: int = HQ_, D: int = D_) -> float:
    """Algorithmic FLOP of a causal chunk of C rows appended after n_before positions: row i
    attends to n_before + i + 1 keys, 4 D FLOP per (key, query head) (QK^T and PV)."""
    keys = C * n_before + C * (C + 1) / 2
    return keys * Hq * 4 * D


def fill_plan(n: int = N_FILL, chunk: int = FILL_CHUNK):
    """(start, count) of the fill appends of one layer."""
    return [(t, min(chunk, n - t)) for t in range(0, n, chunk)]


def step_accounting():
    """Per-step totals of the headline schedule: decode bytes, fill bytes, fill positions,
    prefill FLOP, launches of libkvq kernels."""
    dec = sum(decode_bytes(N_FILL + C_PF + s + 1) for s in range(N_DEC)) * L_
    fill = sum(append_bytes(t, c) for t, c in fill_plan()) * L_
    chunk = append_bytes(N_FILL, C_PF) * L_
    dec_app = sum(append_bytes(N_FILL + C_PF + s, 1) for s in range(N_DEC)) * L_
    pf = prefill_flops(N_FILL, C_PF) * L_
    # launches: one per append; the prefill builds the tile images, runs the staged kernel
    # (its 768 M-tile CTAs split 4 ways over the key range on 148 SMs) and merges the
    # splits; decode = ring pass + low-bit pass + merge
    launches = L_ * (len(fill_plan()) + 1 + 3) + L_ * N_DEC * (1 + 3)
    return {"decode_bytes": dec, "fill_bytes": fill, "fill_positions": N_FILL * L_, "chunk_bytes": chunk,
            "decode_append_bytes": dec_app, "prefill_flop": pf, "launches": launches}


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


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


def recorded_traffic(key: str = "decode_full_length"):
    """DRAM bytes per decode call of the headline shape from the committed ncu record, if it
    was taken on the current decode source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    want = source_hash(DECODE_SOURCES)
    for line in open(p):
        f = line.split()
        if len(f) >= 3 and not line.startswith("#") and f[0] == key and f[2] == want:
            return float(f[1])
    return None


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


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
class OracleSample:
    """The CPU oracle on a labelled sample of the headline workload: one layer filled to
    262,080 positions (257,984 + the 4,096-row chunk) with the generator's seeded chunks
    (one 8,192-position chunk of the layer, later chunks rolled along the positions and
    scaled by 1 + c/64), then timed decodes at 262,080 and an 8-row prefill sample."""

    def __init__(self, threads=None):
        import oracle as orc
        from quantized_mixed_precision_qx_b200.synth import KVRecipe, Workload
        self.threads = threads or (os.cpu_count() or 1)
        self.wl = Workload(L_, B_, H_, HQ_, D_, FILL_CHUNK, KVRecipe("outlier"), seed=0)
        self.o = orc.Cache(1, B_, H_, HQ_, D_, CTX, K_FMT, V_FMT, T_FMT, W_, threads=self.threads)
        base_k = self.wl.kv_chunk(0, 0, FILL_CHUNK, "k")
        base_v = self.wl.kv_chunk(0, 0, FILL_CHUNK, "v")
        n = N_FILL + C_PF
        t0 = time.perf_counter()
        t, c = 0, 0
        while t < n:
            m = min(FILL_CHUNK, n - t)
            s = np.float32(1.0 + c / 64.0)
            self.o.append(0, np.ascontiguousarray(np.roll(base_k, 37 * c, axis=1)[:, :m] * s),
                          np.ascontiguousarray(np.roll(base_v, 91 * c, axis=1)[:, :m] * s))
            t += m
            c += 1
        self.fill_s = time.perf_counter() - t0
        self.n = n

    def decode_s(self, threads, step=0):
        q = self.wl.q_decode(0, step)
        self.o.threads = threads
        t0 = time.perf_counter()
        self.o.decode(0, q, 1.0)
        return time.perf_counter() - t0

    def prefill_rows_s(self, rows):
        q = self.wl.q_prefill(0, C_PF)
        self.o.threads = self.threads
        t0 = time.perf_counter()
        self.o.prefill(0, q, 1.0, rows=rows)
        return time.perf_counter() - t0


def oracle_baseline():
    """cpu_baseline object: the oracle (as it stands) on the sample above."""
    s = OracleSample()
    dbytes = decode_bytes(s.n)
    t_all = min(s.decode_s(s.threads, k) for k in range(2))
    t_one = s.decode_s(1)
    rows = [0, 2047, 2048, 4095, 511, 1023, 3071, 3583]
    t_pf = s.prefill_rows_s(rows)
    pf_flop = len(rows) * HQ_ * 4 * D_ * (N_FILL + np.mean(rows) + 1)
    return {"value": dbytes / t_all / 1e9, "unit": "GB/s", "cores": s.threads, "kind": "oracle",
            "value_1_thread": dbytes / t_one / 1e9, "cpu_model": cpu_model(),
            "append_mtok_s": s.n / s.fill_s / 1e6, "prefill_sample_gflops": pf_flop / t_pf / 1e9,
            "sample": (f"one layer of the workload filled to {s.n} positions (seeded chunks); decode of all 24 "
                       f"query heads at {s.n} timed at {s.threads} threads (best of 2) and at 1 thread; "
                       f"prefill of 8 chunk rows {rows} (all heads) at {s.threads} threads")}


def run_reference(args, rank):
    """The oracle arm: the CPU oracle times decodes of the headline shape (one layer at
    262,080 positions, all 24 query heads) on the machine's host cores, one decode per step."""
    if rank != 0:
        return
    s = OracleSample()
    dbytes = decode_bytes(s.n)
    for k in range(args.warmup):
        s.decode_s(s.threads, k)
    times = [s.decode_s(s.threads, args.warmup + k) for k in range(max(1, args.steps))]
    t = sum(times) / len(times)
    v = dbytes / t / 1e9
    desc = (f"one layer of the workload filled to {s.n} positions (seeded chunks), one decode of all 24 query "
            f"heads per step at {s.threads} threads")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": s.threads, "kind": "oracle", "sample": desc,
                             "cpu_model": cpu_model()},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
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
class Headline:
    """Device inputs, cache and events of the headline schedule on one GPU."""

    def __init__(self, dev, seed):
        import torch
        from quantized_mixed_precision_qx_b200 import kvq
        self.torch, self.kvq, self.dev = torch, kvq, dev
        gen = torch.Generator(device=dev)
        self.kf, self.vf, self.kc, self.vc, self.qp, self.kd, self.vd, self.qd = ([] for _ in range(8))
        for layer in range(L_):
            gen.manual_seed(1000 * seed + layer)
            scale = torch.ones(H_, D_, device=dev)
            for h in range(H_):
                scale[h, torch.randperm(D_, generator=gen, device=dev)[:8]] = 8.0
            self.kf.append(torch.randn(B_, N_FILL, H_, D_, device=dev, generator=gen) * scale)
            self.vf.append(torch.randn(B_, N_FILL, H_, D_, device=dev, generator=gen))
            self.kc.append(torch.randn(B_, C_PF, H_, D_, device=dev, generator=gen) * scale)
            self.vc.append(torch.randn(B_, C_PF, H_, D_, device=dev, generator=gen))
            self.qp.append(torch.randn(B_, C_PF, HQ_, D_, device=dev, generator=gen) / math.sqrt(D_))
            self.kd.append(torch.randn(N_DEC, B_, 1, H_, D_, device=dev, generator=gen) * scale)
            self.vd.append(torch.randn(N_DEC, B_, 1, H_, D_, device=dev, generator=gen))
            self.qd.append(torch.randn(N_DEC, B_, HQ_, D_, device=dev, generator=gen) / math.sqrt(D_))
        self.out_pf = torch.empty(B_, C_PF, HQ_, D_, device=dev)
        self.out_dec = torch.empty(N_DEC, L_, B_, HQ_, D_, device=dev)
        self.cache = kvq.KVCache(L_, B_, H_, HQ_, D_, CTX, K_FMT, V_FMT, T_FMT, W_, device=dev, ws_rows=C_PF)
        self.h = self.cache.handle
        self.ws = self.cache.ensure_workspace(C_PF)
        ev = lambda: torch.cuda.Event(enable_timing=True)   # noqa: E731
        self.ev_fill = [(ev(), ev()) for _ in range(L_)]
        self.ev_pf = [(ev(), ev()) for _ in range(L_)]
        self.ev_dec = [(ev(), ev()) for _ in range(N_DEC * L_)]

    def rebind(self, stream):
        self.kvq.kvq_cache_bind(self.h, self.cache.dev, self.cache.nbytes, stream)

    def device_step(self, stream):
        kvq, h, ws = self.kvq, self.h, self.ws
        self.rebind(stream)
        for layer in range(L_):
            e0, e1 = self.ev_fill[layer]
            e0.record(stream)
            for t, c in fill_plan():
                kvq.kvq_append(h, layer, self.kf[layer][:, t:t + c], self.vf[layer][:, t:t + c], c, stream)
            e1.record(stream)
        for layer in range(L_):
            kvq.kvq_append(h, layer, self.kc[layer], self.vc[layer], C_PF, stream)
            e0, e1 = self.ev_pf[layer]
            e0.record(stream)
            kvq.kvq_prefill_attention(h, layer, self.qp[layer], C_PF, 1.0, self.out_pf, ws, ws.numel(), stream)
            e1.record(stream)
        for s in range(N_DEC):
            for layer in range(L_):
                kvq.kvq_append(h, layer, self.kd[layer][s], self.vd[layer][s], 1, stream)
                e0, e1 = self.ev_dec[s * L_ + layer]
                e0.record(stream)
                kvq.kvq_decode_attention(h, layer, self.qd[layer][s], 1.0, self.out_dec[s, layer], ws, ws.numel(),
                                         stream)
                e1.record(stream)

    def step_times(self):
        fill = sum(a.elapsed_time(b) for a, b in self.ev_fill) / 1e3
        pf = sum(a.elapsed_time(b) for a, b in self.ev_pf) / 1e3
        dec = [a.elapsed_time(b) / 1e3 for a, b in self.ev_dec]
        return fill, pf, dec


class HostInputs:
    """Pinned host copies of the schedule's inputs and the device landing buffers of the
    end-to-end run. The fill appends cycle through 8 distinct pinned chunks per tensor (every
    append's input still crosses PCIe); the prompt chunk, its queries and the decode-step
    inputs are per layer."""

    def __init__(self, hl: Headline):
        torch = hl.torch
        self.hl = hl
        self.k = [hl.kf[0][:, i * FILL_CHUNK:(i + 1) * FILL_CHUNK].contiguous().cpu().pin_memory() for i in range(8)]
        self.v = [hl.vf[0][:, i * FILL_CHUNK:(i + 1) * FILL_CHUNK].contiguous().cpu().pin_memory() for i in range(8)]
        self.kc = [t.cpu().pin_memory() for t in hl.kc]
        self.vc = [t.cpu().pin_memory() for t in hl.vc]
        self.qp = [t.cpu().pin_memory() for t in hl.qp]
        self.kd = [t.cpu().pin_memory() for t in hl.kd]
        self.vd = [t.cpu().pin_memory() for t in hl.vd]
        self.qd = [t.cpu().pin_memory() for t in hl.qd]
        self.out_pf = [torch.empty(B_, C_PF, HQ_, D_).pin_memory() for _ in range(2)]
        self.out_dec = torch.empty(N_DEC, L_, B_, HQ_, D_).pin_memory()
        dev = hl.dev
        self.dk = [torch.empty(B_, FILL_CHUNK, H_, D_, device=dev) for _ in range(2)]
        self.dv = [torch.empty(B_, FILL_CHUNK, H_, D_, device=dev) for _ in range(2)]
        self.dq = [torch.empty(B_, C_PF, HQ_, D_, device=dev) for _ in range(2)]
        self.ddk = [torch.empty(B_, 1, H_, D_, device=dev) for _ in range(2)]
        self.ddv = [torch.empty(B_, 1, H_, D_, device=dev) for _ in range(2)]
        self.ddq = [torch.empty(B_, HQ_, D_, device=dev) for _ in range(2)]
        self.copy_stream = torch.cuda.Stream(device=dev)
        self.h2d = 0
        self.d2h = 0

    def e2e_step(self, stream):
        """The whole schedule with every input copied from pinned host memory (on a second
        stream, double-buffered, so copies overlap the kernels) and every output read back."""
        torch, kvq, hl = self.hl.torch, self.hl.kvq, self.hl
        h, ws, cs = hl.h, hl.ws, self.copy_stream
        ops = []
        for layer in range(L_):
            for i, (t, c) in enumerate(fill_plan()):
                ops.append(("fill", layer, i, c))
        for layer in range(L_):
            ops.append(("chunk", layer, 0, C_PF))
        for s in range(N_DEC):
            for layer in range(L_):
                ops.append(("dec", layer, s, 1))
        hl.rebind(stream)
        start = torch.cuda.Event()
        start.record(stream)
        cs.wait_event(start)
        consumed = [None, None]
        h2d = d2h = 0

        def issue(j):
            nonlocal h2d
            kind, layer, i, c = ops[j]
            b = j & 1
            with torch.cuda.stream(cs):
                if consumed[b] is not None:
                    cs.wait_event(consumed[b])
                if kind == "fill":
                    src_k, src_v = self.k[i % 8][:, :c], self.v[i % 8][:, :c]
                    dk, dv = self.dk[b][:, :c], self.dv[b][:, :c]
                    dk.copy_(src_k, non_blocking=True)
                    dv.copy_(src_v, non_blocking=True)
                    h2d += 2 * src_k.numel() * 4
                elif kind == "chunk":
                    self.dk[b][:, :c].copy_(self.kc[layer], non_blocking=True)
                    self.dv[b][:, :c].copy_(self.vc[layer], non_blocking=True)
                    self.dq[b].copy_(self.qp[layer], non_blocking=True)
                    h2d += (2 * self.kc[layer].numel() + self.qp[layer].numel()) * 4
                else:
                    self.ddk[b].copy_(self.kd[layer][i], non_blocking=True)
                    self.ddv[b].copy_(self.vd[layer][i], non_blocking=True)
                    self.ddq[b].copy_(self.qd[layer][i], non_blocking=True)
                    h2d += (2 * self.kd[layer][i].numel() + self.qd[layer][i].numel()) * 4
                e = torch.cuda.Event()
                e.record(cs)
                return e

        ready = issue(0)
        for j, (kind, layer, i, c) in enumerate(ops):
            nxt = issue(j + 1) if j + 1 < len(ops) else None
            b = j & 1
            stream.wait_event(ready)
            if kind == "fill":
                kvq.kvq_append(h, layer, self.dk[b][:, :c], self.dv[b][:, :c], c, stream)
            elif kind == "chunk":
                kvq.kvq_append(h, layer, self.dk[b][:, :c], self.dv[b][:, :c], C_PF, stream)
                kvq.kvq_prefill_attention(h, layer, self.dq[b], C_PF, 1.0, hl.out_pf, ws, ws.numel(), stream)
                self.out_pf[layer & 1].copy_(hl.out_pf, non_blocking=True)
                d2h += hl.out_pf.numel() * 4
            else:
                kvq.kvq_append(h, layer, self.ddk[b], self.ddv[b], 1, stream)
                kvq.kvq_decode_attention(h, layer, self.ddq[b], 1.0, hl.out_dec[i, layer], ws, ws.numel(), stream)
                self.out_dec[i, layer].copy_(hl.out_dec[i, layer], non_blocking=True)
                d2h += hl.out_dec[i, layer].numel() * 4
            ev = torch.cuda.Event()
            ev.record(stream)
            consumed[b] = ev
            ready = nxt
        self.h2d, self.d2h = h2d, d2h


def run_kvq(args, rank, world):
    import torch
    import torch.distributed as dist

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    hl = Headline(dev, seed=rank)
    acct = step_accounting()

    for _ in range(args.warmup):
        hl.device_step(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    t_step0 = torch.cuda.Event(enable_timing=True)
    t_step1 = torch.cuda.Event(enable_timing=True)
    fill_t = pf_t = dec_t = 0.0
    dec_calls = []
    torch.cuda.synchronize()
    t_step0.record(stream)
    for _ in range(args.steps):
        hl.device_step(stream)
        torch.cuda.synchronize()
        f, p, d = hl.step_times()
        fill_t += f
        pf_t += p
        dec_t += sum(d)
        dec_calls.extend(d)
    t_step1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clock_info = clocks.stop()
    step_ms = t_step0.elapsed_time(t_step1) / args.steps

    # ---- end to end: pinned host inputs, copies inside the timed region
    hi = HostInputs(hl)
    for _ in range(max(1, min(2, args.warmup))):
        hi.e2e_step(stream)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        hi.e2e_step(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_s = e0.elapsed_time(e1) / 1e3 / args.steps
    h2d, d2h = hi.h2d, hi.d2h
    assert h2d == hi_h2d() and d2h == hi_d2h(), (h2d, d2h)
    status = hl.kvq.kvq_device_status(hl.h)
    del hi, hl
    torch.cuda.empty_cache()

    # ---- max over ranks
    dec_t, fill_t, pf_t, e2e_s, step_ms = max_over_ranks([dec_t, fill_t, pf_t, e2e_s, step_ms], world, dev)
    if rank != 0:
        return
    peaks = read_peaks()
    peak = peaks["hbm_gbs"]
    K = args.steps
    value = whole_job_gbs(world, acct["decode_bytes"] * K, dec_t)
    per_call = acct["decode_bytes"] / (N_DEC * L_)
    avg_call = dec_t / (K * N_DEC * L_)
    achieved = per_call / avg_call / 1e9
    traffic = recorded_traffic()
    fill_gbs = acct["fill_bytes"] * K / fill_t / 1e9
    pf_tflops = acct["prefill_flop"] * K / pf_t / 1e12
    extra = None if args.no_extra else supplementary(dev, peaks)
    cpu = oracle_baseline() if world == 1 else None
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD,
                   "l2": "inputs larger than L2: each layer's cache is 404 MB and consecutive decodes read "
                         "different layers (no flush)",
                   "parallelism": f"replicas x{world}"},
        "decode_frac_of_peak": achieved / peak,
        "decode_call_us": {"mean": avg_call * 1e6, "median": statistics.median(dec_calls) * 1e6,
                           "max": max(dec_calls) * 1e6},
        "append_fill_mtok_s": world * acct["fill_positions"] * K / fill_t / 1e6,
        "append_fill_gbs": world * fill_gbs,
        "prefill_alg_tflops": world * pf_tflops,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "peak_source": peaks["source"] + " (hbm_gbs, copy bandwidth)",
                     "kernel": "decode call (ring pass + low-bit pass + merge) at 262,081..262,144 positions",
                     "algorithmic_bytes_per_launch": per_call},
        "roofline_append": {"bound": "hbm", "achieved": fill_gbs, "peak": peak, "unit": "GB/s",
                            "frac": fill_gbs / peak, "traffic": None,
                            "kernel": "append_kernel, fill appends of 8,192 positions",
                            "algorithmic_bytes_per_step": acct["fill_bytes"]},
        "roofline_prefill": {"bound": "tensor", "achieved": pf_tflops, "peak": peaks["bf16_tflops_sustained"],
                             "unit": "TFLOP/s", "frac": pf_tflops / peaks["bf16_tflops_sustained"], "traffic": None,
                             "peak_source": peaks["source"] + " (bf16_tflops_sustained; fp16 runs at the bf16 rate)",
                             "kernel": "prefill_tiles + prefill_staged + prefill_merge, 4,096 rows over 262,080 "
                                       "positions, algorithmic FLOP",
                             "algorithmic_flop_per_step": acct["prefill_flop"]},
        "cpu_baseline": cpu,
        "e2e": {"value": world * acct["decode_bytes"] / e2e_s / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "step_ms": e2e_s * 1e3,
                "note": "decode bytes / whole end-to-end step time (fill, prefill and decode through the C ABI "
                        "with every input copied from pinned host memory and every output read back)"},
        "gpu_launches": acct["launches"] * K,
        "device_status": "ok" if status == 0 else "a bounded device wait ran out",
        "clocks": clock_info,
        "workloads": extra,
    }
    print(json.dumps(line), flush=True)


def hi_h2d() -> int:
    """Bytes copied host -> device per end-to-end step: every fill append's K and V, the
    prompt chunk's K, V and queries, each decode step's K, V and query (all layers)."""
    fill = L_ * N_FILL * H_ * D_ * 4 * 2
    chunk = L_ * (2 * C_PF * H_ * D_ + C_PF * HQ_ * D_) * 4
    dec = L_ * N_DEC * (2 * H_ * D_ + HQ_ * D_) * 4
    return fill + chunk + dec


def hi_d2h() -> int:
    """Bytes read back per end-to-end step: every prefill and decode output."""
    return L_ * (C_PF + N_DEC) * HQ_ * D_ * 4


def supplementary(dev, peaks):
    """Figures on the other workloads (one GPU, device-generated seeded inputs; parity for
    these shapes is covered by the tests): config D's schedule (latency-bound: contexts of
    1.5-48 MB, L2 flushed before each decode), KVarN decode and fill, the asymmetric sweep,
    and the quality figure per format."""
    import torch
    from quantized_mixed_precision_qx_b200 import kvq
    peak = peaks["hbm_gbs"]
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

    # config D schedule: 32 appends of 1,024 to 32,768, decode after each (L2 flushed)
    c = kvq.KVCache(1, 1, H_, HQ_, D_, CD_CTX, K_FMT, V_FMT, T_FMT, W_, device=dev)
    gen.manual_seed(7)
    ks = [torch.randn(1, CD_CHUNK, H_, D_, device=dev, generator=gen) for _ in range(CD_CTX // CD_CHUNK)]
    vs = [torch.randn(1, CD_CHUNK, H_, D_, device=dev, generator=gen) for _ in range(CD_CTX // CD_CHUNK)]
    q = torch.randn(1, HQ_, D_, device=dev, generator=gen) / math.sqrt(D_)
    out = torch.empty_like(q)
    ws = c.ensure_workspace(1)
    dts, ats = [], []
    for rep in range(3):
        kvq.kvq_cache_bind(c.handle, c.dev, c.nbytes)
        for s in range(CD_CTX // CD_CHUNK):
            a0, a1, d0, d1 = (torch.cuda.Event(enable_timing=True) for _ in range(4))
            a0.record()
            c.append(0, ks[s], vs[s])
            a1.record()
            flush.fill_(s & 0xFF)
            d0.record()
            kvq.kvq_decode_attention(c.handle, 0, q, 1.0, out, ws, ws.numel())
            d1.record()
            torch.cuda.synchronize()
            if rep > 0:
                ats.append(a0.elapsed_time(a1) / 1e3)
                dts.append(d0.elapsed_time(d1) / 1e3)
    cd_bytes = 2 * sum(decode_bytes((s + 1) * CD_CHUNK, B=1, H=H_) for s in range(CD_CTX // CD_CHUNK))
    cd_app = 2 * sum(append_bytes(s * CD_CHUNK, CD_CHUNK, B=1, H=H_) for s in range(CD_CTX // CD_CHUNK))
    res["config_d_schedule"] = {
        "decode_gbs": cd_bytes / sum(dts) / 1e9, "decode_frac": cd_bytes / sum(dts) / 1e9 / peak,
        "decode_us_mean": sum(dts) / len(dts) * 1e6, "append_mtok_s": 2 * CD_CTX / sum(ats) / 1e6,
        "append_gbs": cd_app / sum(ats) / 1e9,
        "note": "latency-bound: contexts 1,024..32,768 are 1.5-48 MB; L2 flushed before each decode"}
    del c, ks, vs
    torch.cuda.empty_cache()

    # index-gather decode (QSA budget): one full-length layer, 2,048 listed positions per kv
    # head (the 16 newest, in the ring, and 2,032 seeded others), L2 flushed before each call
    n = N_FILL + C_PF
    c = kvq.KVCache(1, 1, H_, HQ_, D_, n, K_FMT, V_FMT, T_FMT, W_, device=dev)
    fill(c, 1, H_, D_, n)
    gen.manual_seed(11)
    k_list = 2048
    lists = []
    for h in range(H_):
        rest = torch.randperm(n - 16, generator=gen, device=dev)[:k_list - 16]
        lists.append(torch.cat([torch.arange(n - 16, n, device=dev), rest]))
    idx = torch.stack(lists)[None].to(torch.int32).contiguous()
    in_ring = (idx >= n - W_)
    gbytes = int(in_ring.sum()) * 2 * ROW_T + int((~in_ring).sum()) * (ROW_K + ROW_V) + 2 * HQ_ * D_ * 4
    q = torch.randn(1, HQ_, D_, device=dev, generator=gen) / math.sqrt(D_)
    out = torch.empty_like(q)
    ws = c.ensure_workspace(1)
    ts = []
    for i in range(13):
        flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        kvq.kvq_decode_attention_indexed(c.handle, 0, q, 1.0, idx, k_list, out, ws, ws.numel())
        e1.record()
        torch.cuda.synchronize()
        if i >= 3:
            ts.append(e0.elapsed_time(e1) / 1e3)
    tg = statistics.median(ts)
    res["index_gather_2048"] = {"us": tg * 1e6, "gathered_bytes": gbytes, "gbs": gbytes / tg / 1e9,
                                "context": n, "positions_per_kv_head": k_list,
                                "note": "latency-bound: 3.2 MB gathered per call"}

    # multi-query verify (MTP): chunks of 1, 2, 4 and 8 draft rows through the prefill entry
    # point over the same full-length layer (the last C positions are the chunk), L2 flushed
    # before each call; bytes = every stored row once (the algorithmic minimum: chunks of up to
    # 4 rows actually read the rows once per row) + q + out
    verify = {}
    for C in (1, 2, 4, 8):
        qv = torch.randn(1, C, HQ_, D_, device=dev, generator=gen) / math.sqrt(D_)
        ov = torch.empty_like(qv)
        wsv = c.ensure_workspace(C)
        tv = []
        for i in range(8):
            flush.fill_(i & 0xFF)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            kvq.kvq_prefill_attention(c.handle, 0, qv, C, 1.0, ov, wsv, wsv.numel())
            e1.record()
            torch.cuda.synchronize()
            if i >= 3:
                tv.append(e0.elapsed_time(e1) / 1e3)
        tm = statistics.median(tv)
        vbytes = decode_bytes(n) + 2 * (C - 1) * HQ_ * D_ * 4
        verify[f"C={C}"] = {"us": tm * 1e6, "gbs": vbytes / tm / 1e9, "frac": vbytes / tm / 1e9 / peak}
    res["multi_query_verify"] = dict(verify, note="on-the-fly tcgen05 prefill, key range split over the SMs; "
                                                  f"context {n}")
    del c, idx
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

    # per-channel K decode (CUDA-core path): 4 kv heads x 256, 65,536 positions, K q5_0 per
    # channel, V q5_0, no tail
    B, H, Hq, D, n = 1, 4, 24, 256, 65536
    c = kvq.KVCache(1, B, H, Hq, D, n, 6, 6, 14, 0, device=dev, k_per_channel=1)
    t_fill = fill(c, B, H, D, n)
    td = time_decode(c, B, Hq, D)
    dbytes = B * H * n * 2 * rows_bytes(6, D) + 2 * B * Hq * D * 4
    res["per_channel_k"] = {"decode_gbs": dbytes / td / 1e9, "decode_frac": dbytes / td / 1e9 / peak,
                            "decode_us": td * 1e6, "append_fill_mtok_s": n * B / t_fill / 1e6,
                            "note": "K q5_0 per channel (token-axis blocks), V q5_0, no tail; CUDA-core attention"}
    del c
    torch.cuda.empty_cache()
    res["quality_rel_l2_vs_fp32"] = quality(dev)
    return res


FMT_NAMES = ["q2_0", "q2_1", "q3_0", "q3_1", "q4_0", "q4_1", "q5_0", "q5_1", "q6_0", "q6_1", "q8_0", "q8_1"]


def quality(dev):
    """Relative L2 error of the decode output against softmax attention over the unquantized
    fp32 inputs (computed in float64), per format: K = V = the format, no tail; K-only rows
    (K = the format, V = q8_1, the most precise block format) and V-only rows (K = q8_1,
    V = the format); and the config D formats with their q8_0 tail. Batch 1, 4 KV heads x
    256, 24 query heads, 8192 positions with 8 outlier K channels per head (x8), 4 queries."""
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
    cases = [(name, f, f, kvq.NONE, 0, 0) for f, name in enumerate(FMT_NAMES)]
    cases += [(f"K-only {name}", f, kvq.Q8_1, kvq.NONE, 0, 0) for f, name in enumerate(FMT_NAMES)]
    cases += [(f"V-only {name}", kvq.Q8_1, f, kvq.NONE, 0, 0) for f, name in enumerate(FMT_NAMES)]
    cases.append(("q6_0/q5_0 + q8_0 tail 2048", K_FMT, V_FMT, T_FMT, W_, 0))
    # per-channel (token-axis) K against per-token K, V q8_1, without and with a 2,048 q8_0 tail
    for f in (kvq.Q4_0, kvq.Q5_0, kvq.Q6_0):
        for tf, W in ((kvq.NONE, 0), (kvq.Q8_0, W_)):
            tail = "no tail" if W == 0 else "q8_0 tail 2048"
            cases.append((f"K-only {FMT_NAMES[f]} per-token, {tail}", f, kvq.Q8_1, tf, W, 0))
            cases.append((f"K-only {FMT_NAMES[f]} per-channel, {tail}", f, kvq.Q8_1, tf, W, 1))
    res = {}
    for name, kf, vf, tf, W, kpc in cases:
        c = kvq.KVCache(1, B, H, Hq, D, n, kf, vf, tf, W, device=dev, k_per_channel=kpc)
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
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads' figures")
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
