#!/usr/bin/env python
"""Benchmark of the deterministic-reduction hot path on B200.

One step = one pass over every kernel of the path on seeded synthetic inputs
shaped like the pages' workloads:
  plan      stable sort of 4096 tokens by adapter id (8 adapters)
  shrink    segmented LoRA shrink, M=4096, K=4096, r=16, split-K 8:
            tree (deterministic), atomic, unsplit
  expand    segmented LoRA expand r=16 -> N=4096
  fused     shrink (tree, split-K 8) and expand in one launch, y on chip
  shrink16  LoRA shrink M=16, K=4096, r=16: tree s=8, atomic s=8, unsplit
  gemm      batch-invariant GEMM M=4096, N=4096, K=4096 (tcgen05)
  treegemm  TP-invariant tree GEMM M=2048, N=4096, K=16384, 8 emulated shards
  attn      decode attention, fixed-size KV split: 32 sequences x 2048 tokens,
            32 query heads over 8 kv heads, head size 128
  rmsnorm   4096 x 4096 bf16
  lsm       log_softmax 4096 x 151936 fp32
  mean      mean of the same 4096 x 151936 fp32 rows

The headline `value` is the deterministic split-K LoRA-shrink HBM GB/s on
the segmented workload (algorithmic bytes / kernel time, CUDA events on the
launch stream).  Every kernel's own time, throughput and roofline fraction
is listed under "kernels"; "roofline" describes the kernel with the largest
share of the step.  L2 is flushed before each kernel: 256 MiB written, then read back.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Det. split-K LoRA-shrink HBM GB/s; BI-GEMM TFLOP/s; % of roofline; Δ vs atomic"
WORKLOAD = ("segmented multi-adapter LoRA shrink M=4096 tokens, 8 adapters, K=4096, r=16, "
            "split-K 8 tree, inside one pass of the whole deterministic-reduction path")
L2_FLUSH_BYTES = 256 << 20

M4, K4, R4, NAD = 4096, 4096, 16, 8
PLAN_TILES = (M4 + 63) // 64 + NAD + 1


def shrink_bytes(M=M4, K=K4, r=R4, n_ad=NAD):
    """Algorithmic bytes of one segmented shrink: x, every adapter's A, y,
    and the plan's token ids and 16-byte tile headers."""
    return M * K * 2 + n_ad * r * K * 2 + M * r * 4 + 4 * M + 16 * ((M + 63) // 64 + n_ad + 1)


def expand_bytes(M=M4, N=4096, r=R4, n_ad=NAD):
    """y, every adapter's B, the fp32 out write and the token ids."""
    return M * r * 4 + n_ad * N * r * 2 + M * N * 4 + 4 * M


def fused_bytes(M=M4, K=K4, N=4096, r=R4, n_ad=NAD):
    """Fused shrink + expand: x, every adapter's A and B, the fp32 out
    write, the plan's token ids and tile headers (y never leaves the chip)."""
    return M * K * 2 + n_ad * r * K * 2 + n_ad * N * r * 2 + M * N * 4 + 4 * M + 16 * ((M + 63) // 64 + n_ad + 1)


# decode attention: 32 sequences of 2048 cached tokens, 32 query heads over
# 8 kv heads, head size 128 (a grouped-query decoder layer)
ATT_B, ATT_HQ, ATT_HKV, ATT_D, ATT_L = 32, 32, 8, 128, 2048


def attn_bytes(B, Hq, Hkv, D, lens):
    """K and V of every sequence's cached tokens, q, and the fp32 out."""
    return sum(lens) * Hkv * D * 2 * 2 + B * Hq * D * 2 + B * Hq * D * 4


SHRINK_BYTES = shrink_bytes()


# Nominal B200 figures (datasheet): the targets are stated against these.
NOMINAL_HBM_GBS = 8000.0
NOMINAL_BF16_TFLOPS = 2250.0


def peaks():
    """Roofline denominators.  Every kernel here is timed alone (its own
    graph, L2 flushed before it), so the tensor peak is the burst figure.
    The nominal datasheet figures are reported beside them."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    nominal = {"hbm_gbs_nominal": NOMINAL_HBM_GBS, "bf16_tflops_nominal": NOMINAL_BF16_TFLOPS}
    try:
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured (MEASURED_PEAKS.json: copy GB/s, cuBLAS bf16 burst TFLOP/s)", **nominal}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback (earlier measurement on this pool: 6.65 TB/s copy, 1.59 PFLOP/s burst)",
                **nominal}


# --------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling (every 20 ms) of SM clocks and throttle reasons.
    Started before the warm-up; only samples taken inside the timed window
    are summarised (the nearest ones if the window is shorter than one
    sampling period)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []
        self.window = (0.0, 0.0)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        t0, t1 = self.window
        inside = [ln for (t, ln) in self.lines if t0 <= t <= t1]
        if not inside and self.lines:
            inside = [min(self.lines, key=lambda tl: abs(tl[0] - 0.5 * (t0 + t1)))[1]]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in inside:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "window_s": round(t1 - t0, 3)}


# ------------------------------------------------------------------ workload

def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


class Workload:
    """Device-resident inputs and outputs of one step, and its kernel list."""

    def __init__(self, bi, synth, seed):
        self.bi = bi
        d = synth.lora_inputs(M4, K4, R4, n_adapters=NAD, N=4096, seed=seed)
        self.ids_host = d["ids"]
        self.x_host = d["x"]
        self.x = dev_bf16(d["x"])
        self.A = dev_bf16(d["at"])
        self.B = dev_bf16(d["bt"])
        self.ids = torch.from_numpy(d["ids"]).cuda()
        self.plan = torch.empty(bi.lora_plan_bytes(M4, NAD) // 4, dtype=torch.int32, device="cuda")
        self.y = torch.empty(M4, R4, dtype=torch.float32, device="cuda")
        self.y_at = torch.empty_like(self.y)
        self.y_un = torch.empty_like(self.y)
        self.out = torch.empty(M4, 4096, dtype=torch.float32, device="cuda")
        d1 = synth.lora_inputs(16, 4096, 16, seed=seed)
        self.x16, self.A16 = dev_bf16(d1["x"]), dev_bf16(d1["at"][0])
        self.y16 = torch.empty(16, 16, dtype=torch.float32, device="cuda")
        xr, wr = synth.rmsnorm_inputs(4096, 4096, seed=seed)
        self.xr, self.wr = dev_bf16(xr), dev_bf16(wr)
        self.yr = torch.empty_like(self.xr)
        self.logits = torch.from_numpy(synth.logits_inputs(4096, 151936, seed=seed)).cuda()
        self.lsm = torch.empty_like(self.logits)
        self.mean = torch.empty(4096, dtype=torch.float32, device="cuda")
        g = np.random.default_rng(seed)
        self.aq = torch.randn(ATT_B, ATT_HQ, ATT_D, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16).cuda()
        self.ak = torch.randn(ATT_B, ATT_HKV, ATT_L, ATT_D, generator=torch.Generator().manual_seed(seed + 1)).to(torch.bfloat16).cuda()
        self.av = torch.randn(ATT_B, ATT_HKV, ATT_L, ATT_D, generator=torch.Generator().manual_seed(seed + 2)).to(torch.bfloat16).cuda()
        self.alens = torch.full((ATT_B,), ATT_L, dtype=torch.int32, device="cuda")
        self.aout = torch.empty(ATT_B, ATT_HQ, ATT_D, dtype=torch.float32, device="cuda")
        self.aws = torch.empty(bi.attn_decode_ws_bytes(ATT_B, ATT_HQ, ATT_D, ATT_L), dtype=torch.uint8, device="cuda")
        del g
        self.flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        self.flush_f = self.flush.view(torch.float32)
        self.flush_sink = torch.empty((), dtype=torch.float32, device="cuda")
        self.kernels = self._kernels()

    def _kernels(self):
        """(name, fn, algorithmic bytes, flops, bound, our launches per call)"""
        bi = self.bi
        lsm_bytes = 4096 * 151936 * 8
        k = [
            ("plan", lambda: bi.lora_plan(self.ids, NAD, self.plan),
             4 * M4 + 4 * (M4 + NAD + 2) + 4 * M4 + 16 * PLAN_TILES, 0, "hbm", 1),
            ("shrink_tree_s8", lambda: bi.lora_shrink_segmented(self.x, self.A, self.plan, self.y, 8, "tree"),
             SHRINK_BYTES, 2 * M4 * K4 * R4, "hbm", 1),
            ("shrink_atomic_s8", lambda: bi.lora_shrink_segmented(self.x, self.A, self.plan, self.y_at, 8, "atomic"),
             SHRINK_BYTES, 2 * M4 * K4 * R4, "hbm", 1),
            ("shrink_unsplit", lambda: bi.lora_shrink_segmented(self.x, self.A, self.plan, self.y_un, 1, "unsplit"),
             SHRINK_BYTES, 2 * M4 * K4 * R4, "hbm", 1),
            ("expand", lambda: bi.lora_expand_segmented(self.y, self.B, self.plan, self.out),
             expand_bytes(), 2 * M4 * 4096 * R4, "hbm", 1),
            ("fused_shrink_expand", lambda: bi.lora_fused(self.x, self.A, self.B, self.plan, self.out, splits=8),
             fused_bytes(), 2 * M4 * K4 * R4 + 2 * M4 * 4096 * R4, "hbm", 1),
            ("shrink16_tree_s8", lambda: bi.lora_shrink(self.x16, self.A16, self.y16, 8, "tree"),
             16 * 4096 * 2 * 2 + 16 * 16 * 4, 2 * 16 * 4096 * 16, "hbm", 1),
            ("shrink16_atomic_s8", lambda: bi.lora_shrink(self.x16, self.A16, self.y16, 8, "atomic"),
             16 * 4096 * 2 * 2 + 16 * 16 * 4, 2 * 16 * 4096 * 16, "hbm", 1),
            ("shrink16_unsplit", lambda: bi.lora_shrink(self.x16, self.A16, self.y16, 1, "unsplit"),
             16 * 4096 * 2 * 2 + 16 * 16 * 4, 2 * 16 * 4096 * 16, "hbm", 1),
            ("attn_decode", lambda: bi.attn_decode(self.aq, self.ak, self.av, self.alens, self.aout, ws=self.aws),
             attn_bytes(ATT_B, ATT_HQ, ATT_HKV, ATT_D, [ATT_L] * ATT_B), 4 * ATT_B * ATT_HQ * ATT_L * ATT_D, "hbm", 2),
            ("rmsnorm", lambda: bi.rmsnorm(self.xr, self.wr, self.yr, 1e-6),
             4096 * 4096 * 4 + 4096 * 2, 0, "hbm", 1),
            ("log_softmax", lambda: bi.log_softmax(self.logits, self.lsm), lsm_bytes, 0, "hbm", 1),
            ("mean", lambda: bi.mean(self.logits, self.mean), 4096 * 151936 * 4 + 4096 * 4, 0, "hbm", 1),
        ]
        k += self._gemm_kernels()
        return k

    def _gemm_kernels(self):
        bi = self.bi
        out = []
        try:
            M, N, K = 4096, 4096, 4096
            import invariant_bi_lora_b200.synth as synth
            a, w = synth.gemm_inputs(M, N, K, seed=0)
            self.ga, self.gw = dev_bf16(a), dev_bf16(w)
            self.gc = torch.empty(M, N, dtype=torch.float32, device="cuda")
            bi.gemm(self.ga, self.gw, self.gc)
            out.append(("gemm", lambda: bi.gemm(self.ga, self.gw, self.gc), 2 * M * K + 2 * N * K + 4 * M * N,
                        2 * M * N * K, "tensor", 1))
        except bi.BiError:
            pass
        try:
            M, N, K, S = 2048, 4096, 16384, 8
            import invariant_bi_lora_b200.synth as synth
            a, w = synth.gemm_inputs(M, N, K, seed=1)
            self.ta, self.tw = dev_bf16(a), dev_bf16(w)
            self.tc = torch.empty(M, N, dtype=torch.float32, device="cuda")
            self.tws = torch.empty(bi.gemm_tree_ws_bytes(M, N, S), dtype=torch.uint8, device="cuda")
            bi.gemm_tree(self.ta, self.tw, self.tc, S, self.tws)
            out.append(("tree_gemm_s8", lambda: bi.gemm_tree(self.ta, self.tw, self.tc, S, self.tws),
                        2 * M * K + 2 * N * K + 4 * M * N, 2 * M * N * K, "tensor", 2))
        except bi.BiError:
            pass
        return out


KERNEL_REPS = 10      # reps per kernel graph in the per-kernel timing block

# DRAM bytes (read + write) of one launch, from dram__bytes_read.sum and
# dram__bytes_write.sum of an ncu capture of the same kernel, stored here
# because ncu does not run inside the bench.  Only kernels whose code is
# unchanged since their capture are listed; the JSON line says where the
# figure comes from.  log_softmax: captured at 256 of the 4096 rows (reads
# 155,611,904 B, writes 98,571,008 B); reads scale with the rows, writes are
# the whole output less the 57,011,456 B that the capture shows still in L2
# at exit (a residue that does not grow once the output exceeds L2).
_LSM256_READ, _LSM256_WRITE, _LSM256_OUT = 155611904, 98571008, 256 * 151936 * 4
MEASURED_TRAFFIC = {"log_softmax": 16 * _LSM256_READ + 16 * _LSM256_OUT - (_LSM256_OUT - _LSM256_WRITE)}
TRAFFIC_SOURCE = {"log_softmax": "ncu capture of this kernel at 256 rows: reads x 16, writes = output less the "
                                 "L2 residue the capture shows at exit"}


def capture(fn, stream):
    """Capture fn() into a CUDA graph on `stream`."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def run_ours(args, rank, world, device):
    from invariant_bi_lora_b200 import bi, synth
    wl = Workload(bi, synth, seed=0)
    pk = peaks()
    cs = torch.cuda.Stream()                       # capture / launch stream

    def flush_l2(i):
        # 256 MiB written, then read back: the write evicts every line the
        # last kernel left, the read-back makes the write-backs of that
        # buffer happen here, so the next kernel starts on a cold L2 holding
        # only clean lines and its DRAM traffic is its own
        wl.flush.fill_(i & 0xff)
        torch.sum(wl.flush_f, dim=0, out=wl.flush_sink)

    def step_body():
        for i, (name, fn, *_rest) in enumerate(wl.kernels):
            flush_l2(i)
            fn()

    # everything below runs with cs as the current stream: graph replays go to
    # the current stream, and the timing events must be on the same one
    cs.wait_stream(torch.cuda.current_stream())
    if args.eager_only:
        # profiler launch lists: the same kernels launched eagerly, no graphs,
        # no timing (ncu's replay of graph nodes does not take the cluster
        # launches here)
        with torch.cuda.stream(cs):
            for _ in range(args.warmup + args.steps):
                step_body()
            torch.cuda.synchronize()
        return {"note": "eager launches for a profiler launch list; not a measurement",
                "steps": args.steps, "warmup": args.warmup, "status": bi.get_device_status(cs)}
    with torch.cuda.stream(cs):
        # eager warm-up (TMA descriptors, kernel attributes, occupancy queries)
        for _ in range(args.warmup):
            step_body()
        torch.cuda.synchronize()
        if bi.get_device_status(cs) != 0:
            raise RuntimeError("device status set during warm-up")

        # one step = one replay of this graph: every kernel once, each after a flush
        g_step = capture(step_body, cs)
        # per-kernel graphs for the difference timing: R x (flush, kernel) and R x flush
        R = KERNEL_REPS
        def reps(fn):
            def body():
                for i in range(R):
                    flush_l2(i)
                    if fn is not None:
                        fn()
            return body
        g_flush = capture(reps(None), cs)
        g_kern = [capture(reps(fn), cs) for (name, fn, *_r) in wl.kernels]
        for _ in range(args.warmup):
            g_step.replay()
        torch.cuda.synchronize()

        ev = lambda: torch.cuda.Event(enable_timing=True)
        clocks = ClockSampler(device)
        clocks.start()
        time.sleep(0.3)
        # ---------------- timed region: exactly K steps
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        h0 = time.time()
        t0, t1 = ev(), ev()
        t0.record(cs)
        for _ in range(args.steps):
            g_step.replay()
        t1.record(cs)
        torch.cuda.synchronize()
        h1 = time.time()
        if world > 1:
            torch.distributed.barrier()
        clocks.mark(h0, h1)
        total_ms = t0.elapsed_time(t1)

        # ---------------- per-kernel durations: (R x [flush, kernel]) - (R x [flush]),
        # the flush-only graph timed right before and right after each kernel
        # graph (their mean is subtracted), five rounds, median
        def replay_ms(g):
            a, b = ev(), ev()
            a.record(cs); g.replay(); b.record(cs)
            torch.cuda.synchronize()
            return a.elapsed_time(b)
        per = {name: [] for (name, *_r) in wl.kernels}
        for _ in range(5):
            for (name, *_r), g in zip(wl.kernels, g_kern):
                f0 = replay_ms(g_flush)
                tk = replay_ms(g)
                f1 = replay_ms(g_flush)
                per[name].append(max(tk - 0.5 * (f0 + f1), 1e-6) / R)

        def time_kernel(fn):
            """The same difference timing for one more kernel (ms, median of 5)."""
            g = capture(reps(fn), cs)
            t = []
            for _ in range(5):
                f0 = replay_ms(g_flush)
                tk = replay_ms(g)
                f1 = replay_ms(g_flush)
                t.append(max(tk - 0.5 * (f0 + f1), 1e-6) / R)
            del g
            return statistics.median(t)

        sweep = None
        if not args.no_sweep:
            del g_kern
            sweep = Sweep(bi, synth, wl).run(time_kernel, pk)
        clk = clocks.stop()
    for k, v in per.items():
        sys.stderr.write(f"kernel {k}: {[round(t * 1e3, 2) for t in v]} us\n")
    per = {k: statistics.median(v) for k, v in per.items()}
    if world > 1:
        from invariant_bi_lora_b200.tp import max_over_ranks
        t = max_over_ranks([total_ms] + list(per.values()), device="cuda")
        total_ms = t[0]
        per = {k: t[j + 1] for j, k in enumerate(per)}
    status = bi.get_device_status(cs)

    kern = []
    for (name, fn, nbytes, flops, bound, launches) in wl.kernels:
        ms = per[name]
        gbs = nbytes / (ms * 1e-3) / 1e9
        tfl = flops / (ms * 1e-3) / 1e12 if flops else None
        kern.append({"name": name, "us": round(ms * 1e3, 3), "bytes": nbytes, "flops": flops,
                     "gbs": round(gbs, 1), "tflops": None if tfl is None else round(tfl, 2),
                     **roof(bound, gbs, tfl, pk), "launches": launches})
    by = {k["name"]: k for k in kern}
    dom = max(kern, key=lambda k: k["us"])
    tree = by["shrink_tree_s8"]
    value = world * tree["gbs"]
    gemm = by.get("gemm")
    e2e = measure_e2e(wl, bi, args) if rank == 0 else None
    atomic_var = atomic_variation(wl, bi) if rank == 0 else None
    stream16 = shrink16_stream(wl, bi, pk) if rank == 0 else None
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded numpy PCG64; shapes of the pages' workloads)",
        "config": {"workload": WORKLOAD, "global_batch": M4 * world, "seq_len": None,
                   "parallelism": f"dp{world} (independent replicas, no collective)",
                   "l2": "flushed before every kernel (256 MiB written, then read back: cold, clean L2)",
                   "timing": "step = one CUDA-graph replay of the whole path; per-kernel time = "
                             f"(graph of {R} x [flush, kernel]) - mean of the (graph of {R} x [flush]) "
                             "replays just before and after it, CUDA events, median of 5"},
        "roofline": {"kernel": dom["name"], "bound": dom["bound"], "achieved": dom["achieved"],
                     "peak": dom["peak"], "unit": dom["unit"], "frac": dom["frac"],
                     "traffic": MEASURED_TRAFFIC.get(dom["name"]),
                     "traffic_source": TRAFFIC_SOURCE.get(dom["name"]),
                     "peak_source": pk["source"], "peak_nominal": dom["peak_nominal"],
                     "frac_nominal": dom["frac_nominal"]},
        "shrink_roofline": {"bound": "hbm", "achieved": tree["gbs"], "peak": pk["hbm_gbs"], "unit": "GB/s",
                            "frac": tree["frac"], "peak_nominal": NOMINAL_HBM_GBS,
                            "frac_nominal": tree["frac_nominal"], "bytes_per_launch": SHRINK_BYTES},
        "delta_vs_atomic_pct": round(100.0 * (tree["us"] / by["shrink_atomic_s8"]["us"] - 1.0), 2),
        "speedup_vs_unsplit_pct": round(100.0 * (by["shrink_unsplit"]["us"] / tree["us"] - 1.0), 2),
        "bi_gemm_tflops": None if gemm is None else gemm["tflops"],
        "atomic_variation": atomic_var,
        "shrink16_cold_stream": stream16,
        "kernels": kern,
        "sweep": sweep,
        "kernel_sum_ms": round(sum(per.values()), 4),
        "gpu_launches": args.steps * sum(k["launches"] for k in kern),
        "device_status": status,
        "clocks": clk,
        "e2e": e2e,
    }
    return line


class Sweep:
    """The measurement rows of the configurations beside the step's (each
    timed alone like the step's kernels, outside the timed step region):
      d2  RMSNorm / log_softmax / mean on the first R of the 4096 rows,
          R in {1, 7, 64, 513, 4096} (R <= 64 is latency: read the us);
      d3  batch-invariant GEMM, K = 4096, N in {4096, 14336},
          M in {1, 16, 64, 256, 1024, 4096} (HBM-bound for M <= 64);
      d4  segmented shrink (tree / atomic s=8, unsplit) and expand at
          r in {8, 16, 64}, M = 4096, 8 adapters;
      d5  tree GEMM K = 16384, N = 4096, M in {1, 128, 2048},
          s in {1, 2, 4, 8} emulated shards (with the combine);
      N2  the cross-rank combine by peer pointers (bi_tree_combine_peers)
          over s separate partial buffers of M=2048 x N=4096 fp32, here all
          on this GPU (standing in for s ranks' buffers), s in {2, 4, 8}."""

    def __init__(self, bi, synth, wl):
        self.bi, self.rows = bi, []
        self.cases = []
        R_ALL = (1, 7, 64, 513, 4096)
        for R in R_ALL:
            n = 4096
            self.add("d2", f"rmsnorm R={R}", {"rows": R, "n": n}, "hbm", R * n * 4 + n * 2, 0,
                     lambda R=R: bi.rmsnorm(wl.xr[:R], wl.wr, wl.yr[:R], 1e-6))
            self.add("d2", f"log_softmax R={R}", {"rows": R, "n": 151936}, "hbm", R * 151936 * 8, 0,
                     lambda R=R: bi.log_softmax(wl.logits[:R], wl.lsm[:R]))
            self.add("d2", f"mean R={R}", {"rows": R, "n": 151936}, "hbm", R * 151936 * 4 + R * 4, 0,
                     lambda R=R: bi.mean(wl.logits[:R], wl.mean[:R]))
        a, w = synth.gemm_inputs(4096, 14336, 4096, seed=3)
        self.ga, self.gw = dev_bf16(a), dev_bf16(w)
        self.gc = torch.empty(4096, 14336, dtype=torch.float32, device="cuda")
        for N in (4096, 14336):
            for M in (1, 16, 64, 256, 1024, 4096):
                bound = "hbm" if M <= 64 else "tensor"
                A_, W_ = self.ga[:M], self.gw[:N]
                C_ = self.gc.view(-1)[:M * N].view(M, N)
                self.add("d3", f"gemm M={M} N={N}", {"M": M, "N": N, "K": 4096}, bound,
                         2 * M * 4096 + 2 * N * 4096 + 4 * M * N, 2 * M * N * 4096,
                         lambda A_=A_, W_=W_, C_=C_: bi.gemm(A_, W_, C_))
        for r in (8, 16, 64):
            d = synth.lora_inputs(M4, K4, r, n_adapters=NAD, N=4096, seed=0)
            X, A, B = dev_bf16(d["x"]), dev_bf16(d["at"]), dev_bf16(d["bt"])
            plan = bi.lora_plan(torch.from_numpy(d["ids"]).cuda(), NAD)
            y = torch.empty(M4, r, dtype=torch.float32, device="cuda")
            bi.lora_shrink_segmented(X, A, plan, y, 8, "tree")
            for mode, s in (("tree", 8), ("atomic", 8), ("unsplit", 1)):
                self.add("d4", f"shrink {mode} s={s} r={r}", {"M": M4, "K": K4, "r": r, "adapters": NAD, "splits": s},
                         "hbm", shrink_bytes(r=r), 2 * M4 * K4 * r,
                         lambda X=X, A=A, plan=plan, y=y, mode=mode, s=s: bi.lora_shrink_segmented(X, A, plan, y, s, mode))
            self.add("d4", f"expand r={r}", {"M": M4, "N": 4096, "r": r, "adapters": NAD}, "hbm",
                     expand_bytes(r=r), 2 * M4 * 4096 * r,
                     lambda y=y, B=B, plan=plan: bi.lora_expand_segmented(y, B, plan, wl.out))
            self.add("N4", f"fused shrink+expand s=8 r={r}", {"M": M4, "K": K4, "N": 4096, "r": r, "adapters": NAD},
                     "hbm", fused_bytes(r=r), 2 * M4 * K4 * r + 2 * M4 * 4096 * r,
                     lambda X=X, A=A, B=B, plan=plan: bi.lora_fused(X, A, B, plan, wl.out, splits=8))
        gen = torch.Generator().manual_seed(7)
        for Bq, L in ((1, 256), (1, 4096), (8, 16384), (32, 1024), (64, 4096)):
            q = torch.randn(Bq, 32, 128, generator=gen).to(torch.bfloat16).cuda()
            kk = torch.randn(Bq, 8, L, 128, generator=gen).to(torch.bfloat16).cuda()
            vv = torch.randn(Bq, 8, L, 128, generator=gen).to(torch.bfloat16).cuda()
            lens = torch.full((Bq,), L, dtype=torch.int32, device="cuda")
            out = torch.empty(Bq, 32, 128, dtype=torch.float32, device="cuda")
            ws = torch.empty(bi.attn_decode_ws_bytes(Bq, 32, 128, L), dtype=torch.uint8, device="cuda")
            self.add("N1", f"attn_decode B={Bq} L={L}", {"B": Bq, "Hq": 32, "Hkv": 8, "D": 128, "L": L}, "hbm",
                     attn_bytes(Bq, 32, 8, 128, [L] * Bq), 4 * Bq * 32 * L * 128,
                     lambda q=q, kk=kk, vv=vv, lens=lens, out=out, ws=ws: bi.attn_decode(q, kk, vv, lens, out, ws=ws))
        a, w = synth.gemm_inputs(2048, 4096, 16384, seed=1)
        self.ta, self.tw = dev_bf16(a), dev_bf16(w)
        self.tc = torch.empty(2048, 4096, dtype=torch.float32, device="cuda")
        self.tws = torch.empty(bi.gemm_tree_ws_bytes(2048, 4096, 8), dtype=torch.uint8, device="cuda")
        for M in (1, 128, 2048):
            for s in (1, 2, 4, 8):
                bound = "tensor" if M >= 2048 else "hbm"
                A_, C_ = self.ta[:M], self.tc[:M]
                self.add("d5", f"tree_gemm M={M} s={s}", {"M": M, "N": 4096, "K": 16384, "shards": s}, bound,
                         2 * M * 16384 + 2 * 4096 * 16384 + 4 * M * 4096, 2 * M * 4096 * 16384,
                         lambda A_=A_, C_=C_, s=s: bi.gemm_tree(A_, self.tw, C_, s, self.tws))
        count = 2048 * 4096
        self.peer_bufs = [torch.empty(count, dtype=torch.float32, device="cuda").normal_() for _ in range(8)]
        self.peer_out = torch.empty(count, dtype=torch.float32, device="cuda")
        for s_ in (2, 4, 8):
            ptrs = [b.data_ptr() for b in self.peer_bufs[:s_]]
            self.add("N2", f"tree_combine_peers s={s_}", {"count": count, "s": s_, "buffers": "local"}, "hbm",
                     4 * count * (s_ + 1), 0, lambda ptrs=ptrs: bi.tree_combine_peers(ptrs, self.peer_out))

    def add(self, row, name, cfg, bound, nbytes, flops, fn):
        self.cases.append((row, name, cfg, bound, nbytes, flops, fn))

    def run(self, time_kernel, pk):
        out = []
        for (row, name, cfg, bound, nbytes, flops, fn) in self.cases:
            try:
                fn()
                torch.cuda.synchronize()
                ms = time_kernel(fn)
            except Exception as e:                     # a shape the library rejects
                out.append({"row": row, "name": name, "config": cfg, "error": str(e)})
                continue
            gbs = nbytes / (ms * 1e-3) / 1e9
            tfl = flops / (ms * 1e-3) / 1e12 if flops else None
            out.append({"row": row, "name": name, "config": cfg, "us": round(ms * 1e3, 3),
                        "gbs": round(gbs, 1), "tflops": None if tfl is None else round(tfl, 2),
                        **roof(bound, gbs, tfl, pk)})
        return out


def roof(bound, gbs, tfl, pk):
    """achieved / peak / frac of one kernel: tensor-bound kernels against the
    burst bf16 figure, HBM-bound ones against the copy bandwidth; the same
    against the nominal datasheet figures in frac_nominal."""
    if bound == "tensor":
        ach, peak, nom, unit = tfl, pk["bf16_tflops"], pk["bf16_tflops_nominal"], "TFLOP/s"
    else:
        ach, peak, nom, unit = gbs, pk["hbm_gbs"], pk["hbm_gbs_nominal"], "GB/s"
    return {"bound": bound, "achieved": round(ach, 2), "peak": peak, "unit": unit, "frac": round(ach / peak, 4),
            "peak_nominal": nom, "frac_nominal": round(ach / nom, 4)}


def atomic_variation(wl, bi, replays=100):
    """Identical-input replays of the M=16 shrink (split-K 8): the fraction
    of replay pairs whose outputs differ anywhere and the fraction of
    elements that differ from replay 0, for the atomic and the tree mode.
    Outside the timed region."""
    out = {}
    for mode in ("atomic", "tree"):
        outs = []
        for _ in range(replays):
            bi.lora_shrink(wl.x16, wl.A16, wl.y16, 8, mode)
            outs.append(wl.y16.clone())
        torch.cuda.synchronize()
        h = torch.stack(outs).view(torch.int32).cpu().numpy().reshape(replays, -1)
        uniq = len({row.tobytes() for row in h})
        pairs_diff = 0
        for i in range(replays):
            pairs_diff += int(np.sum(np.any(h[i + 1:] != h[i], axis=1)))
        npairs = replays * (replays - 1) // 2
        out[mode] = {"replays": replays, "distinct_outputs": uniq,
                     "pairs_differing": round(pairs_diff / npairs, 4),
                     "elements_differing_vs_first": round(float(np.mean(h[1:] != h[0])), 4)}
    return out


def shrink16_stream(wl, bi, pk, l2_bytes=126 << 20):
    """The M=16 shrink as a cold stream: back-to-back calls in one CUDA graph,
    each on its own copy of x and A, the copies together three times the L2
    size, so every call reads from DRAM.  Per-call time (median of 5 graph
    replays / calls) and its HBM fraction; latency, not bandwidth, bounds a
    263 KB call.  Outside the timed region."""
    call_bytes = 16 * 4096 * 2 * 2 + 16 * 16 * 4
    copies = -(-3 * l2_bytes // call_bytes)
    xs = wl.x16.unsqueeze(0).expand(copies, -1, -1).contiguous()
    As = wl.A16.unsqueeze(0).expand(copies, -1, -1).contiguous()
    out = {"calls": copies, "bytes_per_call": call_bytes}
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        for mode, splits in (("tree", 8), ("atomic", 8), ("unsplit", 1)):
            bi.lora_shrink(xs[0], As[0], wl.y16, splits, mode)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=st):
                for i in range(copies):
                    bi.lora_shrink(xs[i], As[i], wl.y16, splits, mode)
            ts = []
            for _ in range(5):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(st); g.replay(); b.record(st)
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b) * 1e3 / copies)
            us = statistics.median(ts)
            gbs = call_bytes / us / 1e3
            out[mode] = {"us_per_call": round(us, 3), "gbs": round(gbs, 1), "frac": round(gbs / pk["hbm_gbs"], 4)}
            del g
    del xs, As
    return out


def measure_e2e(wl, bi, args):
    """Same metric through the public API with host buffers: every step
    copies x and the adapter ids from pinned host memory, builds the plan,
    runs the deterministic shrink and reads y back to the host."""
    x_h = torch.from_numpy(np.ascontiguousarray(wl.x_host).view(np.int16)).view(torch.bfloat16).pin_memory()
    ids_h = torch.from_numpy(wl.ids_host).pin_memory()
    y_h = torch.empty(M4, R4, dtype=torch.float32).pin_memory()
    x_d = torch.empty_like(wl.x)
    ids_d = torch.empty_like(wl.ids)
    stream = torch.cuda.current_stream()

    def one():
        x_d.copy_(x_h, non_blocking=True)
        ids_d.copy_(ids_h, non_blocking=True)
        bi.lora_plan(ids_d, NAD, wl.plan)
        bi.lora_shrink_segmented(x_d, wl.A, wl.plan, wl.y, 8, "tree")
        y_h.copy_(wl.y, non_blocking=True)

    for _ in range(max(3, args.warmup)):
        one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(args.steps, 10)
    a.record(stream)
    for _ in range(n):
        one()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / n
    return {"value": round(SHRINK_BYTES / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
            "h2d_bytes_per_step": x_h.numel() * 2 + ids_h.numel() * 4,
            "d2h_bytes_per_step": y_h.numel() * 4, "ms_per_step": round(ms, 4)}


# ------------------------------------------------------------ CPU oracle

def oracle_shrink_rate(seconds=10.0):
    """The oracle's fp64 shrink over the segmented workload (all 4096
    tokens, 8 adapters), repeated for about `seconds`; returns GB/s in the
    same algorithmic-bytes unit, threads used, passes."""
    import oracle
    from invariant_bi_lora_b200 import synth
    d = synth.lora_inputs(M4, K4, R4, n_adapters=NAD, seed=0)
    nt = oracle.max_threads()
    t0 = time.perf_counter()
    passes = 0
    while True:
        oracle.shrink_exact(d["x"], d["at"], d["ids"], nthreads=nt)
        passes += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return SHRINK_BYTES * passes / el / 1e9, nt, passes, el


def cpu_family_baselines(budget_s=12.0):
    """The oracle on the host cores for the other kernel families, each on a
    bounded sample of its configuration, in the GPU line's units:
    canonical-fp32 and fp64 paths of the row ops, the fp64 GEMM on sampled
    rows, the fp64 expand and the canonical tree combine.  About budget_s
    seconds in all."""
    import oracle
    from invariant_bi_lora_b200 import synth
    nt = oracle.max_threads()
    out = []
    per = budget_s / 9.0

    def timed(name, fn, unit_amount, unit, sample):
        t0 = time.perf_counter()
        n = 0
        while True:
            fn()
            n += 1
            el = time.perf_counter() - t0
            if el >= per:
                break
        out.append({"name": name, "value": round(unit_amount * n / el, 4), "unit": unit, "cores": nt,
                    "kind": "oracle", "sample": f"{n} x {sample} in {el:.2f} s"})

    xr, wr = synth.rmsnorm_inputs(1024, 4096, seed=0)
    b = 1024 * 4096 * 4 + 4096 * 2
    timed("rmsnorm canonical fp32", lambda: oracle.rmsnorm_canon(xr, wr, nthreads=nt), b / 1e9, "GB/s",
          "1024 rows x 4096")
    timed("rmsnorm fp64", lambda: oracle.rmsnorm_exact(xr, wr, nthreads=nt), b / 1e9, "GB/s", "1024 rows x 4096")
    lg = synth.logits_inputs(64, 151936, seed=0)
    timed("log_softmax canonical fp32", lambda: oracle.log_softmax_canon(lg, nthreads=nt),
          64 * 151936 * 8 / 1e9, "GB/s", "64 rows x 151936")
    timed("log_softmax fp64", lambda: oracle.log_softmax_exact(lg, nthreads=nt),
          64 * 151936 * 8 / 1e9, "GB/s", "64 rows x 151936")
    timed("mean canonical fp32", lambda: oracle.mean_canon(lg, nthreads=nt), 64 * 151936 * 4 / 1e9, "GB/s",
          "64 rows x 151936")
    timed("mean fp64", lambda: oracle.mean_exact(lg, nthreads=nt), 64 * 151936 * 4 / 1e9, "GB/s",
          "64 rows x 151936")
    a, w = synth.gemm_inputs(4096, 4096, 4096, seed=0)
    rows = np.arange(0, 4096, 256)
    timed("gemm fp64 (sampled rows)", lambda: oracle.gemm_exact(a, w, rows=rows, nthreads=nt),
          2 * rows.size * 4096 * 4096 / 1e12, "TFLOP/s", f"{rows.size} of 4096 rows, N=K=4096")
    d = synth.lora_inputs(512, 64, 16, n_adapters=NAD, N=4096, seed=0)
    yv = np.random.default_rng(0).standard_normal((512, 16)).astype(np.float32)
    timed("expand fp64", lambda: oracle.expand_exact(yv, d["bt"], d["ids"], nthreads=nt),
          expand_bytes(M=512) / 1e9, "GB/s", "512 tokens, N=4096, r=16, 8 adapters")
    parts = np.random.default_rng(1).standard_normal((8, 1 << 20)).astype(np.float32)
    timed("tree combine canonical fp32", lambda: oracle.tree_combine(parts, nthreads=nt), 9 * 4 * (1 << 20) / 1e9,
          "GB/s", "8 partials of 2^20")
    return out


def cpu_baseline_entry(seconds):
    v, nt, passes, el = oracle_shrink_rate(seconds)
    return {"value": round(v, 3), "unit": "GB/s", "cores": nt, "kind": "oracle",
            "sample": f"{passes} full passes of the oracle's fp64 shrink over the segmented "
                      f"workload (4096 tokens x 4096 x r=16, 8 adapters) in {el:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle
    from invariant_bi_lora_b200 import synth
    d = synth.lora_inputs(M4, K4, R4, n_adapters=NAD, seed=0)
    nt = oracle.max_threads()
    for _ in range(args.warmup):
        oracle.shrink_exact(d["x"][:256], d["at"], d["ids"][:256], nthreads=nt)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.shrink_exact(d["x"], d["at"], d["ids"], nthreads=nt)
    el = time.perf_counter() - t0
    v = SHRINK_BYTES * args.steps / el / 1e9
    return {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * el / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": M4, "seq_len": None, "parallelism": "cpu"},
            "cpu_baseline": {"value": round(v, 3), "unit": "GB/s", "cores": nt, "kind": "oracle",
                             "sample": f"{args.steps} full passes of the oracle's fp64 segmented shrink"},
            "e2e": {"value": round(v, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------- one-op cases (ncu)

CASES = ("plan", "shrink", "shrink_segmented", "expand_segmented", "fused", "gemm", "addmm", "tree_gemm",
         "attn_decode", "rmsnorm", "log_softmax", "mean")
CASE_DEFAULTS = {"M": 16384, "K": 4096, "N": 4096, "r": 16, "adapters": 8, "splits": 8, "mode": "tree",
                 "shards": 8, "rows": 4096, "n": 151936, "B": 32, "L": 2048, "Hq": 32, "Hkv": 8, "D": 128}


def run_case(a):
    """One library operation on seeded inputs, --iters times back to back
    (no timing): the command line of the ncu summaries.  Inputs are drawn
    once and stay on the device."""
    from invariant_bi_lora_b200 import bi, synth
    torch.cuda.set_device(0)
    op = a.case
    if op in ("plan", "shrink", "shrink_segmented", "expand_segmented", "fused"):
        d = synth.lora_inputs(a.M, a.K, a.r, n_adapters=a.adapters,
                              N=a.N if op in ("expand_segmented", "fused") else 0, seed=0)
        X, A = dev_bf16(d["x"]), dev_bf16(d["at"])
        y = torch.empty(a.M, a.r, dtype=torch.float32, device="cuda")
        ids = torch.from_numpy(d["ids"]).cuda()
        plan = bi.lora_plan(ids, a.adapters)
        if op == "plan":
            run = lambda: bi.lora_plan(ids, a.adapters, plan)
        elif op == "shrink":
            A0 = A[0].contiguous()
            run = lambda: bi.lora_shrink(X, A0, y, a.splits, a.mode)
        elif op == "shrink_segmented":
            run = lambda: bi.lora_shrink_segmented(X, A, plan, y, a.splits, a.mode)
        elif op == "fused":
            B = dev_bf16(d["bt"])
            out = torch.empty(a.M, a.N, dtype=torch.float32, device="cuda")
            run = lambda: bi.lora_fused(X, A, B, plan, out, splits=a.splits)
        else:
            B = dev_bf16(d["bt"])
            out = torch.empty(a.M, a.N, dtype=torch.float32, device="cuda")
            bi.lora_shrink_segmented(X, A, plan, y, a.splits, "tree")
            run = lambda: bi.lora_expand_segmented(y, B, plan, out)
    elif op in ("gemm", "addmm", "tree_gemm"):
        g_a, g_w = synth.gemm_inputs(a.M, a.N, a.K, seed=0)
        GA, GW = dev_bf16(g_a), dev_bf16(g_w)
        C = torch.empty(a.M, a.N, dtype=torch.float32, device="cuda")
        if op == "gemm":
            run = lambda: bi.gemm(GA, GW, C)
        elif op == "addmm":
            bias = dev_bf16(synth.normal_bf16((a.N,), 1.0, seed=0, tag=9))
            run = lambda: bi.addmm(bias, GA, GW, C)
        else:
            ws = torch.empty(max(1, bi.gemm_tree_ws_bytes(a.M, a.N, a.shards)), dtype=torch.uint8, device="cuda")
            run = lambda: bi.gemm_tree(GA, GW, C, a.shards, ws)
    elif op == "attn_decode":
        gen = torch.Generator().manual_seed(0)
        q = torch.randn(a.B, a.Hq, a.D, generator=gen).to(torch.bfloat16).cuda()
        kk = torch.randn(a.B, a.Hkv, a.L, a.D, generator=gen).to(torch.bfloat16).cuda()
        vv = torch.randn(a.B, a.Hkv, a.L, a.D, generator=gen).to(torch.bfloat16).cuda()
        lens = torch.full((a.B,), a.L, dtype=torch.int32, device="cuda")
        out = torch.empty(a.B, a.Hq, a.D, dtype=torch.float32, device="cuda")
        ws = torch.empty(bi.attn_decode_ws_bytes(a.B, a.Hq, a.D, a.L), dtype=torch.uint8, device="cuda")
        run = lambda: bi.attn_decode(q, kk, vv, lens, out, ws=ws)
    elif op == "rmsnorm":
        x, w = synth.rmsnorm_inputs(a.rows, a.n, seed=0)
        X, W = dev_bf16(x), dev_bf16(w)
        Y = torch.empty_like(X)
        run = lambda: bi.rmsnorm(X, W, Y)
    elif op in ("log_softmax", "mean"):
        X = torch.from_numpy(synth.logits_inputs(a.rows, a.n, seed=0)).cuda()
        if op == "log_softmax":
            O = torch.empty_like(X)
            run = lambda: bi.log_softmax(X, O)
        else:
            O = torch.empty(a.rows, dtype=torch.float32, device="cuda")
            run = lambda: bi.mean(X, O)
    else:
        raise SystemExit(f"unknown case {op}; one of {', '.join(CASES)}")
    for _ in range(a.iters):
        run()
    torch.cuda.synchronize()
    st = bi.get_device_status()
    if st != 0:
        raise SystemExit(f"device status {st}")
    print(f"{op}: {a.iters} runs ok")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--eager-only", action="store_true",
                    help="launch the step's kernels eagerly and exit (for ncu launch lists)")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the per-configuration measurement rows (d2-d5)")
    ap.add_argument("--case", default=None,
                    help="run one library operation on seeded inputs --iters times and exit "
                         "(for profiler captures): " + ", ".join(CASES))
    ap.add_argument("--iters", type=int, default=3)
    for k, v in CASE_DEFAULTS.items():
        ap.add_argument(f"--{k}", type=type(v), default=v)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.case:
        run_case(args)
        return

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    # CPU baselines first (rank 0, N=1 only), before any GPU work.
    cpu, cpu_families = None, None
    if rank == 0 and world == 1 and not args.eager_only:
        cpu = cpu_baseline_entry(args.cpu_seconds)
        cpu_families = cpu_family_baselines(min(12.0, 1.2 * args.cpu_seconds))

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    try:
        line = run_ours(args, rank, world, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if rank == 0:
        line["cpu_baseline"] = cpu
        line["cpu_baselines_other"] = cpu_families
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
