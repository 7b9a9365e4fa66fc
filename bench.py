#!/usr/bin/env python
"""Throughput of the packed Delta-rule state decode step on B200.

One step = one stq_decode_step over every (request, head) of the workload: restore
the packed state, gated delta update, float32 readout, refit, packed write-back.
Default workload: GDN, B = 512 requests x H = 48 heads, d = 128, nominal 6-bit
allocation ({4,6,8} bits at 0.2/0.5/0.3 of the heads plus 2% FP16 pivot heads),
lognormal row influence, x10 row/column outliers; states built by 256 FP32 warm-up
steps from zero.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl stq|reference]

Under torchrun each rank runs its own B requests on its own GPU (weak scaling, no
collective on the data path); rank 0 prints one JSON line. `--impl reference` times
the CPU oracle on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import tempfile
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from quantized_linear_attention_02_b200 import workload as W  # noqa: E402

D = 128
METRIC = "head-state decode steps/s and HBM GB/s (% of B200 peak), B=512 6-bit"
UNIT = "head-state steps/s"

# Peaks: MEASURED_PEAKS.json when present, else the pool's earlier measurement.
FALLBACK_HBM_GBS = 6650.0
SMS = 148
FP32_LANES_PER_SM = 128

# ncu dram bytes (read + write) per launch of decode_kernel on the default workload
# (GDN B = 512, dual-axis refit), and the sha256 of the kernel sources they were taken
# with (a changed kernel voids them).
TRAFFIC = {"bytes": 2 * (193_410_048 + 124_321_280),
           "kernel_sha256": "b81b69fa4e87e99547ed6ec1e1a71ed6942a634497f4d33ed93c64c47273bd1f",
           "source": "profiles/decode_kernel_gdn_b256_h48_nominal6.md: dram read + write of one "
                     "B = 256 launch, doubled for B = 512 (traffic grows with B)"}


def issue_rates(stream, reps=3):
    """Measured lane-operation rates (TFLOP/s-like units: 1e12 lane operations per second)
    of packed and of scalar FP32 FMA (the FMA pipe) and of LOP3 (the ALU pipe) on this
    GPU: the library's
    issue-rate probe at full occupancy, timed with CUDA events on `stream`, best of `reps`
    launches after one warm-up launch."""
    import torch
    from quantized_linear_attention_02_b200 import stq
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    blocks, iters = 4 * n_sm, 20000           # 2,048 threads per SM
    out = torch.empty(blocks * stq.PROBE_THREADS, device="cuda")
    rates = {}
    for mode, name in ((0, "ffma2"), (1, "ffma"), (2, "lop3")):
        stq.issue_rate_probe(mode, blocks, iters, out, stream)
        best = 0.0
        for _ in range(reps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            ops = stq.issue_rate_probe(mode, blocks, iters, out, stream)
            e1.record(stream)
            e1.synchronize()
            best = max(best, ops / (e0.elapsed_time(e1) * 1e-3) / 1e12)
        rates[name] = best
    return rates


def kernel_sha():
    """sha256 over the code (comments and blank lines dropped) of the sources the decode
    kernel is compiled from: a comment edit keeps the counters, a code edit voids them."""
    import re
    h = hashlib.sha256()
    for f in ("stq_device.cuh", "stq_kernels.cu", "stq_internal.h"):
        src = open(os.path.join(ROOT, "quantized_linear_attention_02_b200", "csrc", f)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update("\n".join(ln.rstrip() for ln in src.splitlines() if ln.strip()).encode())
    return h.hexdigest()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return float(j["hbm_gbs"]), float(j.get("sm_max_mhz", 1965.0)), "measured"
    return FALLBACK_HBM_GBS, 1965.0, "fallback"


# ---------------------------------------------------------------------------------
# algorithmic counts per step
# ---------------------------------------------------------------------------------
def algorithmic_bytes(w, B, scale_bits=32):
    """Bytes a decode step must move: every head's packed codes (or FP16 pivot rows)
    read and written, its scales r[128], c[128] read and written (heads with any
    quantised row; 4 or 2 bytes each), q, k, v, gate, beta read and o written."""
    rb = W.row_bits(w).astype(np.int64)
    per_req = 0
    for h in range(w.H):
        piv = rb[h] == 16
        codes = int((D * rb[h][~piv] // 8).sum()) + int(piv.sum()) * D * 2
        scales = 2 * D * (scale_bits // 8) if (~piv).any() else 0
        per_req += 2 * (codes + scales)
        per_req += 3 * D * 4 + (4 if w.kind == "gdn" else D * 4) + 4 + D * 4
    return per_req * B


def algorithmic_flops(w, B, scheme="stepquant"):
    """float32 operations the rule prescribes per step (each rounded IEEE operation
    of the oracle's definition): per quantised element 31 for GDN (restore 2, k^T S 2,
    update 2, readout 2, |S| row sum 1, y 1, column max 1, least-squares step one 7,
    step two 9 with the clamp, final code 4), one more for KDA's per-row 1/qmax in
    the column max; 13 with the row-absmax quantiser (restore, k^T S, update, readout
    8, row max 1, code 4); per FP16 pivot element 7 (decay, k^T S, update, readout)."""
    rb = W.row_bits(w)
    if scheme == "row_absmax":
        per_q = 13
    else:
        per_q = 31 + (1 if w.kind == "kda" else 0)
    nq = int((rb != 16).sum()) * D
    npv = int((rb == 16).sum()) * D
    return B * (per_q * nq + 7 * npv)


# ---------------------------------------------------------------------------------
# multi-rank timing: every rank times its own work; the job's time is the slowest rank
# ---------------------------------------------------------------------------------
def max_over_ranks(ms, world, device):
    """Largest of the ranks' times (ms); a no-op for one rank."""
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step, world, ms_per_step):
    """Units all ranks process per second (weak scaling: every rank does the same work)."""
    return units_per_rank_step * world / (ms_per_step * 1e-3)


# ---------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(os.environ.get("STQ_CLOCKS_DIR", tempfile.gettempdir()),
                                 f"stq_clocks_{os.getpid()}_gpu{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------------
# CPU oracle timing (reported baseline only)
# ---------------------------------------------------------------------------------
def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _oracle_worker(args):
    """One process of the all-cores oracle timing: decode steps of one request over a
    shard of the heads for about budget_s seconds (one BLAS thread)."""
    widx, heads, budget_s, scheme = args
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=1)
    except Exception:  # pragma: no cover
        pass
    from oracle import stq_oracle as O
    w = W.WORKLOADS[widx]
    sub = np.asarray(heads)
    rb, om = W.row_bits(w)[sub], W.omega(w)[sub]
    rng = np.random.default_rng(int(sub[0]))
    S = (rng.standard_normal((1, sub.size, D, D)) * 0.1).astype(np.float32)
    u, r, c, piv = O.refit(S, om, rb)
    n, t0, calls = 0, time.perf_counter(), 0
    while True:
        x = W.step_inputs(w, "decode", calls, 0, 1)
        u, r, c, piv, o, X = O.decode_step(u, r, c, piv, rb, om, x.q[:, sub], x.k[:, sub], x.v[:, sub],
                                           O.gate_rows(x.gate[:, sub], w.kind, D), x.beta[:, sub],
                                           scheme=scheme)
        n += sub.size
        calls += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            return n, el


def oracle_rate_all_cores(w, budget_s=10.0, scheme="stepquant"):
    """Head-state steps/s of the oracle on every host core: one spawned process per core,
    each on its own shard of one request's heads (processes are spawned, never forked
    from a process that has used the GPU)."""
    import multiprocessing as mp
    cores = len(os.sched_getaffinity(0))
    n = max(1, min(cores, w.H))
    shards = [list(range(w.H))[i::n] for i in range(n)]
    ctx = mp.get_context("spawn")
    with ctx.Pool(n) as pool:
        res = pool.map(_oracle_worker, [(w.index, sh, budget_s, scheme) for sh in shards])
    heads = sum(r[0] for r in res)
    el = max(r[1] for r in res)
    return heads / el, {"cores": n, "sample": f"{n} processes, each one request x {len(shards[0])} "
                                               f"heads of {w.name}, {el:.1f} s"}


def oracle_quantize_rate(w, budget_s=3.0):
    """Head-states/s of the oracle's quantiser alone (one thread)."""
    from oracle import stq_oracle as O
    rb, om = W.row_bits(w), W.omega(w)
    S = (np.random.default_rng(1).standard_normal((1, w.H, D, D)) * 0.1).astype(np.float32)
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        O.refit(S, om, rb)
        n += w.H
    return n / (time.perf_counter() - t0)


def oracle_rate(w, budget_s=10.0, reqs=1, scheme="stepquant"):
    """Head-state steps/s of the CPU oracle on one thread, timed on a sample of the
    workload (`reqs` requests x all heads per call) for about budget_s seconds."""
    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(limits=1)
    except Exception:  # pragma: no cover
        limiter = None
    from oracle import stq_oracle as O
    rb, om = W.row_bits(w), W.omega(w)
    rng = np.random.default_rng(0)
    S = (rng.standard_normal((reqs, w.H, D, D)) * 0.1).astype(np.float32)
    u, r, c, piv = O.refit(S, om, rb)
    heads, t0, calls = 0, time.perf_counter(), 0
    while True:
        x = W.step_inputs(w, "decode", calls, 0, reqs)
        u, r, c, piv, o, X = O.decode_step(u, r, c, piv, rb, om, x.q, x.k, x.v,
                                           O.gate_rows(x.gate, w.kind, D), x.beta, scheme=scheme)
        heads += reqs * w.H
        calls += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    if limiter is not None:
        limiter.unregister()
    return heads / el, {"kind": "oracle", "cores": 1,
                        "sample": f"{calls} oracle decode steps of {reqs} request(s) x {w.H} heads "
                                  f"of {w.name} in {el:.1f} s, one thread"}


def measure_drift(pool, slots, S_fp32, w, B, gen, dev, steps):
    """Chain `steps` decode steps on a copy of the packed state and on the FP32 state
    with the same inputs; report the relative L2 distance of the dequantised packed
    state from the FP32 state, and of the readouts, at the end (reported, not gated)."""
    import torch
    from quantized_linear_attention_02_b200 import stq
    sub = min(B, 64)                       # a sub-batch keeps the FP32 copy small
    idx = slots[:sub].contiguous()
    S = S_fp32[:sub].clone()
    pool.quantize_init(idx, S)
    o_q = torch.empty((sub, w.H, D), device=dev)
    o_f = torch.empty_like(o_q)
    g2 = torch.Generator(device=dev).manual_seed(4242)
    for _ in range(steps):
        q, k, v, g, b = W.torch_step_inputs(w, sub, g2, dev)
        pool.decode_step(idx, q, k, v, g, b, o_q)
        stq.fp32_decode_step(w.kind, S, q, k, v, g, b, o_f)
    Sq = torch.empty_like(S)
    pool.dequantize(idx, Sq)
    pool.check()
    rel_s = float(torch.linalg.vector_norm(Sq - S) / torch.linalg.vector_norm(S))
    rel_o = float(torch.linalg.vector_norm(o_q - o_f) / torch.linalg.vector_norm(o_f))
    return {"steps": steps, "requests": sub, "state_rel_l2_vs_fp32": rel_s, "readout_rel_l2_vs_fp32": rel_o}


def reference_arm(args, rank, world):
    w = W.WORKLOADS[args.workload]
    if rank != 0:
        return
    # size each step's sample so that warmup + steps take about args.ref_budget seconds
    from oracle import stq_oracle as O
    rb, om = W.row_bits(w), W.omega(w)
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=1)
    except Exception:  # pragma: no cover
        pass
    rng = np.random.default_rng(0)
    S = (rng.standard_normal((1, w.H, D, D)) * 0.1).astype(np.float32)
    u0, r0, c0, p0 = O.refit(S, om, rb)
    x = W.step_inputs(w, "decode", 0, 0, 1)
    t0 = time.perf_counter()
    O.decode_step(u0, r0, c0, p0, rb, om, x.q, x.k, x.v, O.gate_rows(x.gate, w.kind, D), x.beta)
    per_head = (time.perf_counter() - t0) / w.H
    n_steps = args.steps + args.warmup
    heads = int(max(1, min(w.H, args.ref_budget / max(n_steps, 1) / per_head)))
    sub = slice(0, heads)
    rbs, oms = rb[sub], om[sub]
    u, r, c, p = u0[:, sub], r0[:, sub], c0[:, sub], p0[:, sub]

    def step(t):
        nonlocal u, r, c, p
        x = W.step_inputs(w, "decode", t, 0, 1)
        u, r, c, p, o, X = O.decode_step(u, r, c, p, rbs, oms, x.q[:, sub], x.k[:, sub], x.v[:, sub],
                                         O.gate_rows(x.gate[:, sub], w.kind, D), x.beta[:, sub])

    for t in range(args.warmup):
        step(t)
    t0 = time.perf_counter()
    for t in range(args.steps):
        step(args.warmup + t)
    el = time.perf_counter() - t0
    value = heads * args.steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "d": D, "sample_heads_per_step": heads},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"each step: oracle decode of 1 request x {heads} heads of {w.name}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------
# the CUDA arm
# ---------------------------------------------------------------------------------
def stq_arm(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from quantized_linear_attention_02_b200 import build, stq
    build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = W.WORKLOADS[args.workload]
    B, H = (args.batch or w.B), w.H
    ub, om = W.unit_bits(w), W.omega(w)
    if args.compact_slots:       # profiling captures: one slot per request, smaller pool
        n_slots = B
        slot_ids = list(range(B))
    else:
        n_slots = W.n_slots(B)
        slot_ids = [W.slot_of_request(b) for b in range(B)]
    pool = stq.Pool(w.kind, n_slots, ub, om, device=dev, scheme=args.scheme, scale_bits=args.scale_bits)
    slots = torch.tensor(slot_ids, dtype=torch.int32, device=dev)
    gen = torch.Generator(device=dev).manual_seed(1000 * args.workload + rank)

    # initial states: FP32 warm-up steps from zero on the GPU, outlier rows, quantise
    S = torch.zeros((B, H, D, D), device=dev)
    out = torch.empty((B, H, D), device=dev)
    warm = w.warmup_steps if args.warm_steps < 0 else args.warm_steps
    for t in range(warm):
        q, k, v, g, b = W.torch_step_inputs(w, B, gen, dev)
        stq.fp32_decode_step(w.kind, S, q, k, v, g, b, out)
    W.torch_scale_outlier_rows(S, w)
    pool.quantize_init(slots, S)
    pool.check()
    drift = None
    if args.drift_steps > 0:
        drift = measure_drift(pool, slots, S, w, B, gen, dev, args.drift_steps)
    del S
    torch.cuda.empty_cache()

    n_sets = 8
    inputs = [W.torch_step_inputs(w, B, gen, dev) for _ in range(n_sets)]
    stream = torch.cuda.current_stream()

    def step(i):
        q, k, v, g, b = inputs[i % n_sets]
        pool.decode_step(slots, q, k, v, g, b, out, stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    clocks = ClockSampler(local_rank)
    clocks.start()
    # untimed steps under the sampler for at least args.soak_s seconds, so that the
    # clock record covers the same load however short the timed region is
    s0 = time.perf_counter()
    i = 0
    while time.perf_counter() - s0 < args.soak_s:
        for _ in range(50):
            step(i)
            i += 1
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    clk = clocks.stop()
    clk["covers"] = f"{args.soak_s:.2f} s of untimed steps, then the timed region"
    pool.check()

    ms_max = max_over_ranks(ms, world, dev)
    ms_step = ms_max / args.steps
    heads_per_step = B * H * world
    value = whole_job_rate(B * H, world, ms_step)

    # end to end through the host-buffer entry point: pinned inputs in, readout out
    e2e = None
    if args.e2e_steps > 0:
        n_e = args.e2e_steps
        pin = [[x.cpu().pin_memory() for x in s] for s in inputs[:2]]
        h_out = torch.empty((B, H, D), dtype=torch.float32).pin_memory()
        staging = torch.empty(pool.host_staging_bytes(B), dtype=torch.uint8, device=dev)
        for i in range(3):
            pool.decode_step_host(slots, *pin[i % 2], h_out, staging, stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for i in range(n_e):
            pool.decode_step_host(slots, *pin[i % 2], h_out, staging, stream)
        f1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        te = max_over_ranks(f0.elapsed_time(f1), world, dev)
        h2d = sum(x.numel() * 4 for x in pin[0])
        serial = {"value": whole_job_rate(B * H, world, te / n_e), "unit": UNIT,
                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": B * H * D * 4, "steps": n_e,
                  "form": "stq_decode_step_host: copies in, step, copy out on one stream"}

        # The same steps through the library's pipelined host-buffer call: inside the
        # C ABI, step i's inputs go up on an upload stream while step i-1 decodes and its
        # readout comes down on a download stream while step i+1 decodes; each call
        # returns once the previous step's readout is on the host.
        pipe = pool.pipeline(B)
        h_outs = [torch.empty((B, H, D), dtype=torch.float32).pin_memory() for _ in range(2)]
        for i in range(3):
            pipe.step(slots, *pin[i % 2], h_outs[i % 2], stream)
        pipe.finish(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        p0 = torch.cuda.Event(enable_timing=True)
        p1 = torch.cuda.Event(enable_timing=True)
        w0 = time.perf_counter()
        p0.record(stream)
        for i in range(n_e):
            pipe.step(slots, *pin[i % 2], h_outs[i % 2], stream)
        pipe.finish(stream)                       # the last readout is on the host
        p1.record(stream)
        torch.cuda.synchronize()
        wall_ms = (time.perf_counter() - w0) * 1e3
        pipe.close()
        if world > 1:
            dist.barrier()
        tp = max_over_ranks(p0.elapsed_time(p1), world, dev)
        e2e = {"value": whole_job_rate(B * H, world, tp / n_e), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": B * H * D * 4, "steps": n_e,
               "form": "stq_pipeline_step (C ABI): host-buffer decode steps, copies pipelined two "
                       "deep inside the library (H2D, step and D2H on three streams)",
               "host_wall_ms_per_step": wall_ms / n_e,
               "serial": serial}

    # the FP32-state step on the same shapes (the pages' comparison point for the
    # state-update speed-up), timed the same way; per rank, no collective
    fp32_ms = None
    if args.fp32_steps > 0:
        S32 = torch.zeros((B, H, D, D), device=dev)
        for i in range(3):
            q_, k_, v_, g_, b_ = inputs[i % n_sets]
            stq.fp32_decode_step(w.kind, S32, q_, k_, v_, g_, b_, out, stream)
        torch.cuda.synchronize()
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for i in range(args.fp32_steps):
            q_, k_, v_, g_, b_ = inputs[i % n_sets]
            stq.fp32_decode_step(w.kind, S32, q_, k_, v_, g_, b_, out, stream)
        g1.record(stream)
        torch.cuda.synchronize()
        fp32_ms = g0.elapsed_time(g1) / args.fp32_steps
        del S32
        torch.cuda.empty_cache()

    if rank != 0:
        return
    hbm_peak, smax, which = peaks()
    nbytes = algorithmic_bytes(w, B, args.scale_bits)
    flops = algorithmic_flops(w, B, args.scheme)
    sec = ms_step * 1e-3                 # one launch per step: the step time is the launch time
    hbm_ach = nbytes / sec / 1e9
    alu_peak = SMS * FP32_LANES_PER_SM * smax * 1e6 / 1e12
    alu_ach = flops / sec / 1e12
    traffic = None      # counters exist for the default workload and the current kernel only
    if (TRAFFIC["kernel_sha256"] == kernel_sha() and w.index == 3 and B == 512
            and args.scheme == "stepquant" and args.scale_bits == 32):
        traffic = TRAFFIC["bytes"]
    hbm = {"bound": "hbm", "achieved": hbm_ach, "peak": hbm_peak, "unit": "GB/s",
           "frac": hbm_ach / hbm_peak, "traffic": traffic, "peak_source": which,
           "algorithmic_bytes_per_launch": nbytes}
    alu = {"bound": "alu", "achieved": alu_ach, "peak": alu_peak, "unit": "TFLOP/s",
           "frac": alu_ach / alu_peak, "traffic": traffic,
           "peak_source": f"{SMS} SMs x {FP32_LANES_PER_SM} FP32 lanes x {smax:.0f} MHz",
           "algorithmic_flops_per_launch": flops}
    # the derived peak checked against the GPU: the issue-rate probe's packed-FMA rate
    # (the same lane count per SM and clock if the derivation holds) and its LOP3 rate
    rates = issue_rates(stream)
    fma_peak = max(rates["ffma2"], rates["ffma"])
    alu["peak_measured"] = {"value": fma_peak, "unit": "TFLOP/s",
                            "how": "stq_issue_rate_probe, the faster of mode 0 (fma.rn.f32x2) and mode 1 "
                                   "(fma.rn.f32) chains at 2,048 threads per SM, CUDA events, best of 3",
                            "ffma2": rates["ffma2"], "ffma": rates["ffma"], "alu_pipe_lop3": rates["lop3"]}
    alu["frac_of_measured"] = alu_ach / fma_peak
    roofline = alu if alu["frac"] >= hbm["frac"] else hbm
    other = hbm if roofline is alu else alu
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "kind": w.kind, "scheme": args.scheme, "scale_bits": args.scale_bits,
                   "B": B, "H": H, "d": D,
                   "global_batch": B * world, "bits": {str(b): int((ub == b).sum()) for b in sorted(set(ub.tolist()))},
                   "n_slots": n_slots, "l2": "inputs larger than L2 (packed state of the active slots "
                   f"{pool.sizes['slot_code_bytes'] * B / 1e9:.2f} GB, 8 rotating input sets)",
                   "parallelism": f"dp{world}"},
        "hbm_gbs": hbm_ach, "hbm_frac": hbm["frac"],
        "roofline": roofline, "roofline_other": other,
        "clocks": clk, "e2e": e2e, "gpu_launches": args.steps,
    }
    if drift is not None:
        line["drift"] = drift
    if fp32_ms is not None:
        line["fp32_state_step"] = {
            "ms_per_step": fp32_ms, "steps": args.fp32_steps,
            "packed_speedup_vs_fp32": fp32_ms / ms_step,
            "note": "FP32-state gated delta step (fp32_step_kernel) on the same shapes and inputs"}
    if world == 1 and not args.no_cpu_baseline:
        rate, info = oracle_rate(w, budget_s=args.cpu_budget, scheme=args.scheme)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, **info, "cpu": cpu_model()}
        if not args.no_cpu_all_cores:
            rate_all, info_all = oracle_rate_all_cores(w, budget_s=args.cpu_budget, scheme=args.scheme)
            line["cpu_baseline"]["all_cores"] = {"value": rate_all, "unit": UNIT, **info_all}
        if args.scheme == "stepquant":
            line["cpu_baseline"]["quantize_only"] = {"value": oracle_quantize_rate(w), "unit": "head-states/s",
                                                     "cores": 1}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["stq", "reference"], default="stq")
    ap.add_argument("--workload", type=int, default=3, help="index into the workload list (3 = GDN B=512 6-bit)")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--scheme", choices=["stepquant", "row_absmax"], default="stepquant",
                    help="requantisation rule (row_absmax: the pages' uniform baseline)")
    ap.add_argument("--scale-bits", type=int, choices=[32, 16], default=32,
                    help="storage of the scales r, c (16: the compact binary16 layout)")
    ap.add_argument("--soak-s", type=float, default=0.6,
                    help="seconds of untimed steps under the clock sampler before the timed region")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--ref-budget", type=float, default=90.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-cpu-all-cores", action="store_true", help="skip the all-cores oracle timing")
    ap.add_argument("--fp32-steps", type=int, default=200,
                    help="time this many FP32-state steps on the same shapes (0: skip)")
    ap.add_argument("--drift-steps", type=int, default=0,
                    help="after timing, chain this many steps on 64 requests against the FP32 state")
    ap.add_argument("--batch", type=int, default=0, help="override B (profiling captures only)")
    ap.add_argument("--compact-slots", action="store_true", help="B slots instead of 5B+1 (profiling captures only)")
    ap.add_argument("--warm-steps", type=int, default=-1, help="override the FP32 warm-up length (profiling only)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        stq_arm(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
