#!/usr/bin/env python3
"""Benchmark of the CSA + HCA decode hot path at 1M context on B200.

Workload (default ``decode_b4_1m``): batch 4, one query token per sequence at
position 1,048,575; one CSA layer (FP4 indexer over 262,144 compressed
entries, exact top-1024, attention over 1,024 entries + 128 window tokens)
and one HCA layer (dense attention over 8,192 entries + 128 window tokens),
H = 64, d = 512.  A step is one pass of the whole hot path: index scores,
top-k, CSA attention (split-K + log-sum-exp combine), HCA attention.

Metric: query tokens per second (whole job: all ranks' query tokens / max
over ranks of the device time).  Inputs are synthetic (hca_inputs recipes)
and resident in HBM before the timed region; the decode step is one CUDA
graph per replica, and four independently built replicas rotate so that the
bytes one pass touches are out of L2 (126 MB) when the replica comes back.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_b4_1m|decode_b16_64k|prefill_4096_131k|stack61_b32_256k]

Multi-GPU: one process per GPU under torchrun; each rank runs its own
replicas (the decode batch shards over sequences with no data exchange), so
scaling is weak.  ``--impl reference`` times the CPU oracle on the host cores
(rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import hca_inputs as inp  # noqa: E402

MEASURED = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
NOMINAL_HBM_GBS = 8000.0


def peaks():
    try:
        with open(MEASURED) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {
        "hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
        "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
        "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
        "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
        "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown",
    }

    def __init__(self, index: int):
        self.samples, self.ok, self._stop = [], False, threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:      # timed region shorter than one poll: nearest samples around it
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
        mhz = sorted(s[1] for s in inside)
        reasons = set()
        for s in inside:
            for name, attr in self.REASONS.items():
                if s[2] & getattr(self.nv, attr, 0):
                    reasons.add(name)
        return {"sm_mhz": mhz[len(mhz) // 2] if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(inside)}


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
        pg = dist
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local, pg


def max_over_ranks(value: float, pg) -> float:
    if pg is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg):
    if pg is not None:
        pg.barrier()


# ------------------------------------------------------------------ measured DRAM traffic
# dram__bytes_read.sum + dram__bytes_write.sum of one launch of a kernel, taken
# with ncu on the same workload, valid only while the kernel's source file is
# the one that was captured (first 16 hex digits of its sha256); otherwise the
# bench reports null.
MEASURED_TRAFFIC = {
    # dram__bytes_read.sum + dram__bytes_write.sum of one launch on decode_b4_1m
    # (1-pass ncu capture, caches flushed, 4 launches): 20.65 MB + 0 B, and
    # 71.36 MB + 0.04-1.34 MB (the indexer's scores mostly stay in L2; median taken)
    "hca_attn": {"bytes": 20650000, "workload": "decode_b4_1m",
                 "source": "long_context_attention_hca_b200/csrc/attention_tc.cu", "sha256_16": "060c4543b74c857b"},
    "indexer": {"bytes": 71440000, "workload": "decode_b4_1m",
                "source": "long_context_attention_hca_b200/csrc/indexer.cu", "sha256_16": "d1a1a7570f1b9597"},
}


def measured_traffic(kernel: str, workload: str):
    """The captured DRAM bytes of one launch, or None: another workload, or the
    kernel's source changed since the capture."""
    import hashlib
    e = MEASURED_TRAFFIC.get(kernel)
    if e is None or e["workload"] != workload:
        return None
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), e["source"])
    try:
        h = hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    return e["bytes"] if h == e["sha256_16"] else None


# ------------------------------------------------------------------ tensor peaks measured in this run
def gemm_peaks(n=8192, reps=20):
    """Dense GEMM throughput of this GPU in TFLOP/s, measured here with torch
    (cuBLAS / cuBLASLt): bf16 and fp16 n x n x n matmuls and an e4m3 x e4m3
    scaled matmul (fp32 scales, bf16 out).  A short burst after warm-up, CUDA
    events on the current stream; the denominators of the prefill fractions."""
    out = {}
    dev = torch.device("cuda")
    a = torch.randn((n, n), device=dev)
    b = torch.randn((n, n), device=dev)
    flop = 2.0 * n * n * n

    def timeit(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return flop * reps / (e0.elapsed_time(e1) * 1e-3) / 1e12

    for name, dt in (("bf16", torch.bfloat16), ("fp16", torch.float16)):
        x, y = a.to(dt), b.to(dt)
        out[name] = timeit(lambda: torch.matmul(x, y))
        del x, y
    try:
        x8 = a.to(torch.float8_e4m3fn)
        y8 = b.to(torch.float8_e4m3fn).t().contiguous().t()       # column-major second operand
        one = torch.ones((), device=dev)
        out["fp8_e4m3"] = timeit(lambda: torch._scaled_mm(x8, y8, scale_a=one, scale_b=one,
                                                          out_dtype=torch.bfloat16))
        del x8, y8
    except Exception as ex:                     # reported, not hidden
        out["fp8_e4m3"] = None
        out["fp8_error"] = str(ex)[:200]
    del a, b
    torch.cuda.empty_cache()
    out["how"] = f"torch matmul / _scaled_mm, {n}x{n}x{n}, {reps} reps after 3 warm-up, CUDA events"
    return out


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


# ------------------------------------------------------------------ algorithmic bytes (decode)
def decode_bytes(wl):
    """Algorithmic HBM bytes of one decode step of a CSA + HCA layer pair:
    FP4 indexer keys of every eligible CSA entry (64 B codes + 4 B scales),
    the k selected CSA entries and every HCA entry (448 B FP8 + 28 B scales
    + 128 B bf16 RoPE = 604 B), the 128-token bf16 windows, queries in and
    outputs out.  Scores and split partials stay on chip / in L2."""
    dn = wl.d - wl.d_rope
    entry = dn + 4 * (dn // wl.g) + 2 * wl.d_rope
    ikey = wl.c // 2 + wl.c // 32
    T = wl.t + 1
    nc, nh = T // 4, T // 128
    qo = wl.H * wl.d * 2 * 2
    per_seq = {
        "indexer": nc * ikey + wl.Hi * (wl.c // 2 + wl.c // 32 + 4),
        "csa_attn": min(wl.k, nc) * entry + wl.W * wl.d * 2 + qo + min(wl.k, nc) * 4,
        "hca_attn": nh * entry + wl.W * wl.d * 2 + qo,
        "topk": nc * 4 + wl.k * 4 + 8,          # scores read (they stay in L2 at this size), indices written
    }
    return {k: v * wl.B for k, v in per_seq.items()}


def step_bytes_of(algo) -> int:
    """HBM bytes one decode step must move: the indexer's key stream plus
    both attention calls.  The scores the top-k reads and the split-K
    partials stay in L2 and are not counted."""
    return algo["indexer"] + algo["csa_attn"] + algo["hca_attn"]


# ------------------------------------------------------------------ CPU oracle timings
def oracle_decode_sample(wl, seq_fraction=1.0, seed_offset=0):
    """Build the inputs of one decode sequence on the CPU (seeded CPU draws;
    HCA entries pooled by the oracle itself, untimed) and return a closure
    that runs the oracle's decode of that sequence: index scores over the
    first `seq_fraction` of the CSA entries, top-k, CSA attention, HCA
    attention over the same fraction of HCA entries."""
    import numpy as np
    import oracle
    T = wl.t + 1
    nc = int((T // 4) * seq_fraction)
    nh = max(1, int((T // 128) * seq_fraction))
    d, dr, g = wl.d, wl.d_rope, wl.g
    gen = lambda name, shape, std=1.0: inp.normal_bf16(shape, std, wl.seed + 1000 + seed_offset, name)
    qb = inp.bf16_bits(gen("q", (wl.H, d)))
    win = inp.bf16_bits(gen("win", (wl.W, d)))
    # HCA entries: pool nh blocks of 128 raw tokens with the oracle (setup)
    xr = inp.bf16_bits(gen("x", (1, nh * 128, d)))
    gr = inp.bf16_bits(gen("gate", (1, nh * 128, d)))
    b128 = inp.normal_f32((128, d), 0.5, wl.seed + 1000, "b128").numpy()
    hc, hs, hr, _ = oracle.compress(xr, gr, b128, 128, nh, dr, g)
    # CSA entries: only the selected ones are ever read; pool them on demand
    x4 = inp.bf16_bits(gen("x4", (1, 4 * 2048, d)))
    g4 = inp.bf16_bits(gen("g4", (1, 4 * 2048, d)))
    b4 = inp.normal_f32((4, d), 0.5, wl.seed + 1000, "b4").numpy()
    cc, cs, cr, _ = oracle.compress(x4, g4, b4, 4, 2048, dr, g)
    qc = inp.uniform_bytes((1, 1, wl.Hi, wl.c // 2), wl.seed + 1000, "iq").numpy()
    qs = inp.ue8m0_scales((1, 1, wl.Hi, wl.c // 32), wl.seed + 1000, "iqs").numpy()
    w = inp.uniform_f32((1, 1, wl.Hi), wl.seed + 1000, "iw").numpy()
    kc = inp.uniform_bytes((1, nc, wl.c // 2), wl.seed + 1000, "ik").numpy()
    ks = inp.ue8m0_scales((1, nc, wl.c // 32), wl.seed + 1000, "iks").numpy()
    pos = np.array([[4 * nc - 1]], np.int32)

    def run():
        s, _ = oracle.index_scores(qc, qs, w, kc, ks, pos, 4)
        idx, cnt = oracle.topk(s[0], pos[0], 4, wl.k)
        ent = idx[0, :cnt[0]] % 2048          # selected entries mapped onto the pooled sample
        oracle.attend(qb, cc[0], cs[0], cr[0], ent, win, wl.softmax_scale, g)
        oracle.attend(qb, hc[0], hs[0], hr[0], np.arange(nh), win, wl.softmax_scale, g)
    return run


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def run_reference(args, wl):
    """--impl reference: the CPU oracle, as it stands, on the host cores."""
    import oracle
    oracle.build()
    threads = oracle.set_threads(cpu_cores())
    frac = 1.0
    run = oracle_decode_sample(wl, frac)
    t0 = time.perf_counter(); run(); t_one = time.perf_counter() - t0
    budget = 150.0
    if t_one * (args.steps + args.warmup) > budget:
        frac = max(1e-3, budget / ((args.steps + args.warmup) * t_one))
        run = oracle_decode_sample(wl, frac)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = (time.perf_counter() - t0) / args.steps
    value = frac / dt
    sample = (f"one query token (sequence) of {wl.name}: FP4 index scores over {100 * frac:.3g}% of its "
              f"{(wl.t + 1) // 4} CSA entries, exact top-{wl.k}, CSA attention over {wl.k}+{wl.W} keys, "
              f"HCA attention over {100 * frac:.3g}% of its {(wl.t + 1) // 128} entries + {wl.W} window tokens; "
              f"C oracle (fp64 attention) at {threads} threads; value = sampled fraction / time per step")
    line = {"metric": "1M-ctx CSA+HCA decode query-tok/s", "impl": "reference", "value": value,
            "unit": "query-tok/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "global_batch": wl.B, "seq_len": wl.t + 1, "parallelism": "none"},
            "cpu_baseline": {"value": value, "unit": "query-tok/s", "cores": threads, "kind": "oracle",
                             "cpu_model": cpu_model(), "sample": sample},
            "e2e": {"value": value, "unit": "query-tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm: decode
def bench_decode(args, wl, world, rank, pg):
    import long_context_attention_hca_b200 as hca
    from hca_workloads import build_decode
    from long_context_attention_hca_b200.pipeline import DecodeRunner, packed_indexer_query

    dev = torch.device("cuda")
    n_rep = args.replicas
    reps = []
    for r in range(n_rep):
        dw = build_decode(wl)
        runner = DecodeRunner(dw.layers, wl.B, wl.H, wl.k, wl.t, wl.softmax_scale, dense_budget=args.dense_budget,
                              sparse_budget=args.sparse_budget, index_budget=args.index_budget)
        reps.append((dw, runner))
    main = torch.cuda.current_stream()

    # per replica: the step as one graph (timed), and a second graph with external
    # timing events around each kernel class (replayed once, untimed, for the
    # per-kernel breakdown: event nodes between kernels would cost time and break
    # the programmatic launch edges of the timed graph)
    graphs, graphs_ev, evs = [], [], []
    for dw, runner in reps:
        s = torch.cuda.Stream()
        s.wait_stream(main)
        with torch.cuda.stream(s):
            for _ in range(2):
                runner.step(dw.q, dw.iq)
        main.wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            runner.step(dw.q, dw.iq)
        graphs.append(g)
        g2 = torch.cuda.CUDAGraph()
        ev = {}
        with torch.cuda.graph(g2):
            runner.step(dw.q, dw.iq, events=ev)
        graphs_ev.append(g2)
        evs.append(ev)
    # the timed graph: one whole step per replica, in order; each step joins its two
    # streams before the next one forks, so the steps do not overlap, and only the
    # launch gaps between separate graph replays go
    g_all = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_all):
        for dw, runner in reps:
            runner.step(dw.q, dw.iq)
    torch.cuda.synchronize()

    for i in range(args.warmup):
        graphs[i % n_rep].replay()
    g_all.replay()
    torch.cuda.synchronize()
    n_all, n_rest = divmod(args.steps, n_rep)

    clocks = ClockSampler(torch.cuda.current_device()).start()
    time.sleep(0.02)
    barrier(pg)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.perf_counter()
    e0.record()
    for _ in range(n_all):
        g_all.replay()
    for i in range(n_rest):
        graphs[i].replay()
    e1.record()
    torch.cuda.synchronize()
    t_wall1 = time.perf_counter()
    barrier(pg)
    time.sleep(0.01)
    clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    ms_max = max_over_ranks(ms, pg)

    # per-kernel durations from one (untimed) replay of each replica's evented graph
    for g in graphs_ev:
        g.replay()
    torch.cuda.synchronize()
    kern = {}
    for ev in evs:
        for name, (a, b) in ev.items():
            kern.setdefault(name, []).append(a.elapsed_time(b))
    kern_ms = {k: sum(v) / len(v) for k, v in kern.items()}

    # ---------------- end to end through the public API: host q / indexer q in, outputs out
    dw, runner = reps[0]
    h_q = [t.to("cpu").pin_memory() for t in dw.q]
    # each layer's indexer query packed in one buffer, host and device: one copy
    h_iq = [None if t is None else packed_indexer_query(t, device="cpu", pin=True) for t in dw.iq]
    # the outputs back to back in pinned memory, as the runner's device outputs are: one copy
    h_out = list(torch.empty((len(runner.out),) + tuple(runner.out[0].shape), dtype=runner.out[0].dtype,
                             pin_memory=True).unbind(0))
    d_q = [t.clone() for t in dw.q]
    d_iq = [None if t is None else packed_indexer_query(t) for t in dw.iq]
    h2d = sum(t.numel() * t.element_size() for t in h_q) + sum(
        sum(x.numel() * x.element_size() for x in t) for t in h_iq if t is not None)
    d2h = sum(t.numel() * t.element_size() for t in h_out)

    def e2e_step():
        for a, b in zip(d_q, h_q):
            a.copy_(b, non_blocking=True)
        for a, b in zip(d_iq, h_iq):
            if a is not None:
                for x, y in zip(a, b):
                    x.copy_(y, non_blocking=True)
        runner.step(d_q, d_iq)
        for a, b in zip(h_out, runner.out):
            a.copy_(b, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    n_e2e = max(10, min(args.steps, 200))
    barrier(pg)
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(n_e2e):
        e2e_step()
    f1.record()
    torch.cuda.synchronize()
    barrier(pg)
    e2e_eager_ms = max_over_ranks(f0.elapsed_time(f1) / n_e2e, pg)

    # the same step as one CUDA graph, as a decode loop runs it, through
    # DecodeRunner.step_host: query copies overlap the indexer, outputs stream
    # out as each layer finishes
    def e2e_step_host():
        runner.step_host(h_q, h_iq, h_out, d_q, d_iq)

    s_cap = torch.cuda.Stream()
    s_cap.wait_stream(main)
    with torch.cuda.stream(s_cap):
        e2e_step_host()
    main.wait_stream(s_cap)
    torch.cuda.synchronize()
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e):
        e2e_step_host()
    for _ in range(3):
        g_e2e.replay()
    torch.cuda.synchronize()
    barrier(pg)
    torch.cuda.synchronize()
    f0.record()
    for _ in range(n_e2e):
        g_e2e.replay()
    f1.record()
    torch.cuda.synchronize()
    barrier(pg)
    e2e_py_ms = max_over_ranks(f0.elapsed_time(f1) / n_e2e, pg)
    del g_e2e

    # the same step through the C ABI's host-to-host call (hca_decode_step_host:
    # the library issues the copies and the kernels on two streams), as one graph
    plan = runner.capi_plan(d_q, d_iq, packed=3)

    def e2e_step_capi():
        runner.step_host_capi(plan, h_q, h_iq, h_out)

    s_cap = torch.cuda.Stream()
    s_cap.wait_stream(main)
    with torch.cuda.stream(s_cap):
        e2e_step_capi()
    main.wait_stream(s_cap)
    torch.cuda.synchronize()
    g_capi = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_capi):
        e2e_step_capi()
    for _ in range(3):
        g_capi.replay()
    torch.cuda.synchronize()
    barrier(pg)
    torch.cuda.synchronize()
    f0.record()
    for _ in range(n_e2e):
        g_capi.replay()
    f1.record()
    torch.cuda.synchronize()
    barrier(pg)
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / n_e2e, pg)
    del g_capi

    # ---------------- roofline of the dominant kernel
    # Each candidate kernel alone: one graph launches it once per replica (inputs
    # rotate, more bytes than L2 holds), replayed; CUDA events on the launching stream.
    hbm, bf16, bf16s, src = peaks()
    algo = decode_bytes(wl)
    solo_ms = {}
    for name in ("indexer", "csa_attn", "hca_attn"):
        calls = []
        for dw, runner in reps:
            for li, L in enumerate(dw.layers):
                if name == "indexer" and L.ratio == 4:
                    qc, qs, w = dw.iq[li]
                    calls.append(lambda dw=dw, runner=runner, li=li, L=L, qc=qc, qs=qs, w=w: hca.lightning_index(
                        qc, qs, w, L.k_codes, L.k_sf, runner.q_pos, 4, scores=runner.scores[li]))
                elif name == "csa_attn" and L.ratio == 4:
                    calls.append(lambda dw=dw, runner=runner, li=li, L=L: hca.compressed_attn_decode(
                        dw.q[li], L.cache, runner.count[li], min(runner.k, L.n_entries), L.window, runner.scale,
                        idx=runner.idx[li], out=runner.out[li], ws=runner.ws[li]))
                elif name == "hca_attn" and L.ratio == 128:
                    # the kernel alone takes every SM (the library default split plan), with a
                    # workspace sized for that plan
                    ws_solo = torch.empty(max(hca.decode_workspace_size(wl.B, wl.H, L.cache.layout, L.n_entries,
                                                                        L.window.shape[1]), 16),
                                          dtype=torch.uint8, device=dev)
                    calls.append(lambda dw=dw, runner=runner, li=li, L=L, ws_solo=ws_solo: hca.compressed_attn_decode(
                        dw.q[li], L.cache, runner.n_dense[li], L.n_entries, L.window, runner.scale,
                        out=runner.out[li], ws=ws_solo))
        if not calls:
            continue
        s = torch.cuda.Stream()
        s.wait_stream(main)
        with torch.cuda.stream(s):
            for f in calls:
                f()
            s.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                for f in calls:
                    f()
            g.replay()
            s.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            n_rep_solo = 20
            a.record(s)
            for _ in range(n_rep_solo):
                g.replay()
            b.record(s)
            s.synchronize()
        solo_ms[name] = a.elapsed_time(b) / (n_rep_solo * len(calls))
        del g
    dominant = max(solo_ms, key=solo_ms.get) if solo_ms else None
    roof = None
    if dominant is not None:
        ach = algo[dominant] / (solo_ms[dominant] * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": dominant, "achieved": ach, "peak": hbm, "unit": "GB/s",
                "frac": ach / hbm, "peak_source": f"{src} (burst copy)", "traffic": measured_traffic(dominant, wl.name),
                "algorithmic_bytes": algo[dominant], "avg_launch_us": solo_ms[dominant] * 1e3,
                "timing": "the kernel alone, CUDA events, inputs rotating over replicas (L2-cold)",
                "solo_us": {k: v * 1e3 for k, v in solo_ms.items()}}
    step_bytes = step_bytes_of(algo)

    value = world * wl.B / (ms_max * 1e-3)
    line = {
        "metric": "1M-ctx CSA+HCA decode query-tok/s", "value": value, "unit": "query-tok/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp16/fp32 (FP8/FP4 storage)",
        "data": "synthetic",
        "config": {"workload": wl.name, "global_batch": wl.B * world, "seq_len": wl.t + 1,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"inputs larger than L2: {n_rep} rotating replicas, {n_rep * step_bytes / 1e6:.0f} MB touched per cycle",
                   "graph": f"one CUDA graph of {n_rep} whole steps (one per replica, each joined before the next "
                            f"forks), replayed {n_all} times, then {n_rest} single-step graphs"},
        "step_hbm": {"algorithmic_bytes": step_bytes, "achieved_gbs": step_bytes / (ms_max * 1e-3) / 1e9,
                     "frac_of_measured": step_bytes / (ms_max * 1e-3) / 1e9 / hbm,
                     "frac_of_8tbs": step_bytes / (ms_max * 1e-3) / 1e9 / NOMINAL_HBM_GBS},
        "kernels_us": {k: v * 1e3 for k, v in kern_ms.items()},
        "roofline": roof,
        "clocks": clocks.summary(t_wall0, t_wall1),
        "e2e": {"value": world * wl.B / (e2e_ms * 1e-3), "unit": "query-tok/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "how": "hca_decode_step_host (the C ABI's host-to-host decode step: "
                "pinned host queries in, pinned host outputs out, copies and kernels queued by the library on two "
                "streams) captured as one CUDA graph and replayed",
                "python_step_host_value": world * wl.B / (e2e_py_ms * 1e-3),
                "eager_value": world * wl.B / (e2e_eager_ms * 1e-3)},
        "gpu_launches": reps[0][1].kernels_per_step * args.steps,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    for g in graphs:
        del g


def prefill_flops(wl):
    """Algorithmic work of one prefill chunk: attention 4*H*d flop per
    (query, key) pair over each query's CSA keys (min(k, eligible) + window)
    and HCA keys (eligible entries + window); indexer 2*Hi*c int ops per
    (query, eligible CSA entry)."""
    p0, Tq, W = wl.t, wl.Tq, wl.W
    att = ind = 0
    for p in range(p0, p0 + Tq):
        e4, e128 = (p + 1) // 4, (p + 1) // 128
        win = min(W, p + 1)
        att += min(wl.k, e4) + win + e128 + win
        ind += e4
    return 4 * wl.H * wl.d * att, 2 * wl.Hi * wl.c * ind


def prefill_attn_flops(wl):
    """Algorithmic flops of each prefill attention launch: 4*H*d per (query, key)."""
    p0, Tq, W = wl.t, wl.Tq, wl.W
    csa = hca_ = 0
    for p in range(p0, p0 + Tq):
        win = min(W, p + 1)
        csa += min(wl.k, (p + 1) // 4) + win
        hca_ += (p + 1) // 128 + win
    f = 4 * wl.H * wl.d
    return {"csa_attn": f * csa, "hca_attn": f * hca_}


def oracle_prefill_sample(wl, rows):
    """Host inputs for `rows` prefill queries of the workload, drawn on the CPU
    (seeded), and a closure running the oracle's whole path for them: index
    scores over every eligible CSA entry, top-k, CSA attention, HCA attention.
    The compressed entries are pooled by the oracle itself (setup, untimed);
    only a pool of 2048 CSA entries is built, and selected indices map onto it."""
    import numpy as np
    import oracle
    d, dr, g = wl.d, wl.d_rope, wl.g
    seed = wl.seed + 2000
    gen = lambda name, shape, std=1.0: inp.bf16_bits(inp.normal_bf16(shape, std, seed, name))
    nh = (wl.t + wl.Tq) // 128
    x = gen("x", (1, nh * 128, d)); gt = gen("gate", (1, nh * 128, d))
    b128 = inp.normal_f32((128, d), 0.5, seed, "b128").numpy()
    hc, hs, hr, _ = oracle.compress(x, gt, b128, 128, nh, dr, g)
    x4 = gen("x4", (1, 4 * 2048, d)); g4 = gen("g4", (1, 4 * 2048, d))
    b4 = inp.normal_f32((4, d), 0.5, seed, "b4").numpy()
    cc, cs, cr, _ = oracle.compress(x4, g4, b4, 4, 2048, dr, g)
    nc = (wl.t + wl.Tq) // 4
    kc = inp.uniform_bytes((1, nc, wl.c // 2), seed, "ik").numpy()
    ks = inp.ue8m0_scales((1, nc, wl.c // 32), seed, "iks").numpy()
    qb = gen("q", (len(rows), wl.H, d))
    win = gen("win", (wl.W, d))
    qc = inp.uniform_bytes((1, len(rows), wl.Hi, wl.c // 2), seed, "iq").numpy()
    qs = inp.ue8m0_scales((1, len(rows), wl.Hi, wl.c // 32), seed, "iqs").numpy()
    w = inp.uniform_f32((1, len(rows), wl.Hi), seed, "iw").numpy()

    def run():
        for j, i in enumerate(rows):
            p = wl.t + i
            pos = np.array([[p]], np.int32)
            sc, _ = oracle.index_scores(qc[:, j:j + 1], qs[:, j:j + 1], w[:, j:j + 1], kc, ks, pos, 4)
            idx, cnt = oracle.topk(sc[0], pos[0], 4, wl.k)
            ent128, w0, w1 = oracle.causal_keys(p, 128, wl.W)
            oracle.attend(qb[j], cc[0], cs[0], cr[0], idx[0, :cnt[0]] % 2048, win, wl.softmax_scale, g)
            oracle.attend(qb[j], hc[0], hs[0], hr[0], ent128, win, wl.softmax_scale, g)
    return run


def bench_prefill(args, wl, world, rank, pg):
    import long_context_attention_hca_b200 as hca
    from hca_workloads import build_prefill
    from long_context_attention_hca_b200.pipeline import PrefillRunner
    pw = build_prefill(wl)
    runner = PrefillRunner(pw.state, wl.t, wl.Tq, wl.H, wl.k, wl.W, wl.softmax_scale)
    args_step = (pw.raw_chunk, pw.gate_chunk, pw.raw_window, pw.q, pw.iq)
    main = torch.cuda.current_stream()
    # warm-up eagerly, then one CUDA graph per chunk step (the inputs, 0.3 GB of
    # queries alone, are larger than L2)
    s = torch.cuda.Stream()
    s.wait_stream(main)
    with torch.cuda.stream(s):
        runner.step(*args_step)
    main.wait_stream(s)
    torch.cuda.synchronize()
    # the timed graph has no timing events; a second one with them gives the
    # per-kernel breakdown (replayed once, untimed)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        runner.step(*args_step)
    g_ev = torch.cuda.CUDAGraph()
    ev = {}
    with torch.cuda.graph(g_ev):
        runner.step(*args_step, events=ev)
    for _ in range(max(3, args.warmup)):
        g.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device()).start()
    time.sleep(0.02)
    barrier(pg)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    e0.record()
    for _ in range(args.steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    barrier(pg)
    clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, pg)
    g_ev.replay()
    torch.cuda.synchronize()
    kern_ms = {k: a.elapsed_time(b) for k, (a, b) in ev.items()}
    del g, g_ev

    # each attention launch alone (CUDA events on the launching stream)
    st = pw.state
    solo = {}
    calls = {
        "hca_attn": lambda: hca.compressed_attn_prefill(pw.q, wl.t, 128, st.hca, pw.raw_window, wl.W,
                                                        wl.softmax_scale, out=runner.out_hca, stream=s2),
        "csa_attn": lambda: hca.compressed_attn_prefill(pw.q, wl.t, 4, st.csa, pw.raw_window, wl.W,
                                                        wl.softmax_scale, idx=runner.idx, count=runner.count,
                                                        out=runner.out_csa, stream=s2),
    }
    s2 = torch.cuda.Stream()
    s2.wait_stream(main)
    for name, fn in calls.items():
        with torch.cuda.stream(s2):
            fn()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            n_solo = 3
            a.record(s2)
            for _ in range(n_solo):
                fn()
            b.record(s2)
            s2.synchronize()
        solo[name] = a.elapsed_time(b) / n_solo
    fl = prefill_attn_flops(wl)
    fl_att, op_ind = prefill_flops(wl)
    gp = gemm_peaks()
    hbm, bf16, bf16s, src = peaks()
    dominant = max(solo, key=solo.get)
    ach = fl[dominant] / (solo[dominant] * 1e-3) / 1e12
    fp16_peak = gp["fp16"]
    roof = {"bound": "tensor", "kernel": dominant, "achieved": ach, "peak": fp16_peak, "unit": "TFLOP/s",
            "frac": ach / fp16_peak, "peak_source": "fp16 dense GEMM measured in this run (cuBLAS, burst)",
            "frac_of_fp8_measured": (ach / gp["fp8_e4m3"]) if gp.get("fp8_e4m3") else None,
            "frac_of_bf16_measured": ach / gp["bf16"], "traffic": None,
            "algorithmic_flops": fl[dominant], "avg_launch_us": solo[dominant] * 1e3,
            "timing": "the kernel alone, CUDA events on its stream, 3 launches after one warm-up",
            "solo_us": {k: v * 1e3 for k, v in solo.items()},
            "solo_tflops": {k: fl[k] / (solo[k] * 1e-3) / 1e12 for k in solo}}

    # end to end through the public API: the chunk's inputs from pinned host memory,
    # both attention outputs back to pinned host memory, every step
    h_in = [t.to("cpu").pin_memory() for t in (pw.raw_chunk, pw.gate_chunk, pw.raw_window, pw.q)]
    h_iq = [t.to("cpu").pin_memory() for t in pw.iq]
    d_in = [t.clone() for t in (pw.raw_chunk, pw.gate_chunk, pw.raw_window, pw.q)]
    d_iq = [t.clone() for t in pw.iq]
    h_out = [torch.empty_like(runner.out_csa, device="cpu").pin_memory(),
             torch.empty_like(runner.out_hca, device="cpu").pin_memory()]
    h2d = sum(t.numel() * t.element_size() for t in h_in + h_iq)
    d2h = sum(t.numel() * t.element_size() for t in h_out)

    def e2e_step():
        for a_, b_ in zip(d_in + d_iq, h_in + h_iq):
            a_.copy_(b_, non_blocking=True)
        oc, oh = runner.step(d_in[0], d_in[1], d_in[2], d_in[3], tuple(d_iq))
        h_out[0].copy_(oc, non_blocking=True)
        h_out[1].copy_(oh, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    n_e2e = max(3, min(args.steps, 20))
    barrier(pg)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(n_e2e):
        e2e_step()
    f1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / n_e2e, pg)

    line = {"metric": "prefill tokens/s", "value": world * wl.Tq / (ms * 1e-3), "unit": "tok/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp16/fp32 (FP8/FP4 storage)", "data": "synthetic",
            "config": {"workload": wl.name, "chunk": wl.Tq, "p0": wl.t,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "inputs larger than L2 (queries alone 268 MB per chunk)"},
            "tflops": {"attention": fl_att / (ms * 1e-3) / 1e12, "indexer_int": op_ind / (ms * 1e-3) / 1e12,
                       "total": (fl_att + op_ind) / (ms * 1e-3) / 1e12,
                       "frac_of_fp16_measured": (fl_att + op_ind) / (ms * 1e-3) / 1e12 / gp["fp16"],
                       "frac_of_fp8_measured": ((fl_att + op_ind) / (ms * 1e-3) / 1e12 / gp["fp8_e4m3"])
                       if gp.get("fp8_e4m3") else None},
            "gemm_peaks_tflops": gp,
            "kernels_us": {k: v * 1e3 for k, v in kern_ms.items()},
            "roofline": roof,
            "clocks": clocks.summary(t0, t1),
            "e2e": {"value": world * wl.Tq / (e2e_ms * 1e-3), "unit": "tok/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "how": "PrefillRunner.step from pinned host inputs (chunk raw KV "
                    "and gates, window, queries, indexer queries) to pinned host outputs (CSA and HCA), eager"},
            "gpu_launches": runner.kernels_per_step * args.steps}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        threads = oracle.set_threads(cpu_cores())
        rows = [0, 1000, 2047, 4095]
        run = oracle_prefill_sample(wl, rows)
        run()
        tt = time.perf_counter()
        run()
        dt = time.perf_counter() - tt
        line["cpu_baseline"] = {"value": len(rows) / dt, "unit": "tok/s", "cores": threads, "kind": "oracle",
                                "cpu_model": cpu_model(),
                                "sample": f"{len(rows)} query positions of {wl.name} ({rows}) through the oracle: "
                                          "index scores over every eligible CSA entry, exact top-k, CSA and HCA "
                                          f"attention in fp64, at {threads} threads"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def bench_stack(args, wl, world, rank, pg):
    from hca_workloads import build_decode
    from long_context_attention_hca_b200.pipeline import (DecodeRunner, gqa_bf16_bytes, kv_resident_bytes,
                                                           pro_layer_ratios)
    dw = build_decode(wl)
    runner = DecodeRunner(dw.layers, wl.B, wl.H, wl.k, wl.t, wl.softmax_scale, dense_budget=args.dense_budget)
    main = torch.cuda.current_stream()
    s = torch.cuda.Stream()
    s.wait_stream(main)
    with torch.cuda.stream(s):
        runner.step(dw.q, dw.iq)
    main.wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        runner.step(dw.q, dw.iq)
    g_ev = torch.cuda.CUDAGraph()        # with per-kernel timing events, replayed once untimed
    ev = {}
    with torch.cuda.graph(g_ev):
        runner.step(dw.q, dw.iq, events=ev)
    for _ in range(max(1, args.warmup)):
        g.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device()).start()
    barrier(pg)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    e0.record()
    for _ in range(args.steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    barrier(pg)
    clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, pg)
    g_ev.replay()
    torch.cuda.synchronize()
    per = {k: a.elapsed_time(b) * 1e3 for k, (a, b) in ev.items()}
    ratios = pro_layer_ratios(wl.layers)
    resident = kv_resident_bytes(wl.B, wl.t + 1, ratios)
    gqa = gqa_bf16_bytes(wl.B, wl.t + 1, wl.layers)
    line = {"metric": "61-layer decode step", "value": world * wl.B / (ms * 1e-3), "unit": "query-tok/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp16/fp32 (FP8/FP4 storage)",
            "data": "synthetic", "config": {"workload": wl.name, "global_batch": wl.B, "seq_len": wl.t + 1,
                                            "layers": wl.layers, "parallelism": "single GPU"},
            "kv_resident_bytes": resident, "gqa8_bf16_bytes": gqa, "kv_ratio": resident / gqa,
            "kernels_us_untimed_replay": per, "dense_budget_ctas": runner.dense_budget,
            "clocks": clocks.summary(t0, t1)}
    if rank == 0:
        print(json.dumps(line), flush=True)


def bench_select_variants(args, wl, rank):
    """The note's indexer variants on the decode workload's shapes: 4 or 64
    indexer heads (section 7 parameters: n_h^I = 64), fp32 or BF16 index
    scores (section 9: the top-k selector on BF16 scores, reported 2x faster
    at 99.7% KV recall).  Times the fused index + top-k call alone (one CUDA
    graph over 4 rotating replicas of the keys and queries, CUDA events), and
    measures the recall of the BF16 top-k sets against the exact fp32 ones."""
    import dataclasses
    import long_context_attention_hca_b200 as hca
    dev = torch.device("cuda")
    T = wl.t + 1
    nc = T // 4
    n_rep = 4
    out = {"metric": "decode index + top-k variants", "unit": "us", "config": {"workload": wl.name, "B": wl.B,
           "entries": nc, "k": wl.k}, "variants": {}, "recall_bf16_vs_fp32": {}}
    pos = torch.full((wl.B,), wl.t, dtype=torch.int32, device=dev)
    sets = {}
    for Hi in (4, 64):
        w2 = dataclasses.replace(wl, Hi=Hi)
        reps = []
        for r in range(n_rep):
            kc, ks = inp.indexer_keys(w2, wl.B, nc, layer=100 + r, device=dev)
            qc, qs, w = inp.indexer_queries(w2, wl.B, layer=100 + r, device=dev)
            reps.append((qc.view(wl.B, 1, Hi, -1), qs.view(wl.B, 1, Hi, -1), w.view(wl.B, 1, Hi), kc, ks))
        for bf in (False, True):
            sdt = torch.bfloat16 if bf else torch.float32
            bufs = []
            for (qc, qs, w, kc, ks) in reps:
                need = hca.topk_workspace_size(wl.B, nc, wl.k, bf)
                bufs.append((torch.empty((wl.B, 1, nc), dtype=sdt, device=dev),
                             torch.empty((wl.B, wl.k), dtype=torch.int32, device=dev),
                             torch.empty((wl.B,), dtype=torch.int32, device=dev),
                             torch.empty(max(need, 16), dtype=torch.uint8, device=dev)))

            def run(st):
                for (qc, qs, w, kc, ks), (sc, idx, cnt, ws) in zip(reps, bufs):
                    hca.lightning_index_topk(qc, qs, w, kc, ks, pos, 4, wl.k, scores=sc, idx=idx, count=cnt, ws=ws,
                                             stream=st, score_bf16=bf)
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):
                run(s)
                s.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=s):
                    run(s)
                for _ in range(3):
                    g.replay()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                n_it = 20
                a.record(s)
                for _ in range(n_it):
                    g.replay()
                b.record(s)
                s.synchronize()
            us = a.elapsed_time(b) * 1e3 / (n_it * n_rep)
            key = f"h{Hi}_{'bf16' if bf else 'fp32'}"
            out["variants"][key] = {"us": us, "key_bytes": wl.B * nc * 68, "gbs": wl.B * nc * 68 / (us * 1e-6) / 1e9}
            sets[key] = [set_rows(buf[1]) for buf in bufs]
            del g
        rec = []
        for r in range(n_rep):
            for a_, b_ in zip(sets[f"h{Hi}_fp32"][r], sets[f"h{Hi}_bf16"][r]):
                rec.append(len(a_ & b_) / max(len(a_), 1))
        out["recall_bf16_vs_fp32"][f"h{Hi}"] = {"mean": sum(rec) / len(rec), "min": min(rec), "rows": len(rec)}
        out["variants"][f"h{Hi}_bf16"]["speedup_vs_fp32"] = (out["variants"][f"h{Hi}_fp32"]["us"] /
                                                             out["variants"][f"h{Hi}_bf16"]["us"])
    out["pages"] = "BF16 index scores: 2x faster top-k, 99.7% KV recall (note section 9; trained model, no workload given)"
    if rank == 0:
        print(json.dumps(out), flush=True)


def set_rows(idx):
    h = idx.to("cpu").numpy()
    return [set(int(v) for v in row if v >= 0) for row in h]


def cpu_baseline(wl):
    """The oracle on the host cores: one query token of the workload (see
    oracle_decode_sample), at all cores and at one thread."""
    import oracle
    oracle.build()
    threads = oracle.set_threads(cpu_cores())
    run = oracle_decode_sample(wl, 1.0)
    run()
    t0 = time.perf_counter()
    n = 0
    while n < 5 and time.perf_counter() - t0 < 15.0:
        run()
        n += 1
    dt = (time.perf_counter() - t0) / n
    oracle.set_threads(1)
    t1 = time.perf_counter()
    run()
    dt1 = time.perf_counter() - t1
    oracle.set_threads(threads)
    return {"value": 1.0 / dt, "unit": "query-tok/s", "cores": threads, "kind": "oracle",
            "cpu_model": cpu_model(), "single_thread_value": 1.0 / dt1,
            "sample": f"one query token (sequence) of {wl.name} through the oracle: index scores over all "
                      f"{(wl.t + 1) // 4} CSA entries, exact top-{wl.k}, CSA and HCA attention in fp64; "
                      f"{n} repetitions at {threads} threads (OpenMP over entries and heads), 1 at one thread"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode_b4_1m",
                    choices=["decode_b4_1m", "decode_b16_64k", "prefill_4096_131k", "stack61_b32_256k"])
    ap.add_argument("--replicas", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dense-budget", type=int, default=None,
                    help="CTA cap of the step's dense (HCA) attention (default: the SMs that the top-k select leaves, at least half; "
                         "0: the library default, every SM)")
    ap.add_argument("--sparse-budget", type=int, default=0, help="CTA cap of the sparse decode attention (0: none)")
    ap.add_argument("--index-budget", type=int, default=0, help="CTA cap of the fused decode indexer (0: none)")
    ap.add_argument("--select-variants", action="store_true",
                    help="time the fused index + top-k with 4 / 64 indexer heads and fp32 / BF16 scores, and the "
                         "recall of BF16 top-k sets (decode workloads)")
    args = ap.parse_args()
    wl = inp.WORKLOADS[args.workload]
    world, rank, local, pg = dist_setup(args.gpus)
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, wl)
        if pg is not None:
            pg.destroy_process_group()
        return
    if args.select_variants:
        bench_select_variants(args, wl, rank)
    elif wl.prefill:
        bench_prefill(args, wl, world, rank, pg)
    elif wl.layers > 1:
        bench_stack(args, wl, world, rank, pg)
    else:
        bench_decode(args, wl, world, rank, pg)
    if pg is not None:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
