#!/usr/bin/env python
"""Throughput of the chunkwise gated delta-rule forward on B200 GPUs.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload I] [--chunk C]
                [--inverse exact|neumann] [--impl ours|reference]

One step = one gdr_chunk_fwd pass over the whole workload (all sequences, all
chunks) with inputs resident in HBM.  Prints ONE JSON line on rank 0.

* value: tokens/s (B*T per step) over all ranks; N>1 runs one process per GPU,
  each rank processing its own copy of the workload (independent sequences, no
  collective on the data path: weak scaling); time = max over ranks of the
  CUDA-event time of K steps between barriers.
* e2e: the same metric through gdr_chunk_fwd_host with pinned host buffers
  (host->device copies of every input and device->host copies of o and
  S_final inside the timed region).
* roofline: algorithmic bytes (or flops) of one launch / its average duration,
  against the measured peaks in MEASURED_PEAKS.json.
* cpu_baseline: the fp64 oracle timed on this host's cores on a bounded sample
  of the same workload (rank 0, N = 1 only).
* --impl reference: the oracle alone on the host cores (a bounded sample per
  step), the only comparison arm this method has.
* --pass backward / --momentum MU: the same line for gdr_chunk_bwd (seeded
  upstream gradients) or gdr_chunk_fwd_momentum (seeded per-chunk kappa), both
  CUDA-core kernels; their roofline is fp32 FMA issue ("alu").
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from gated_delta_rule_141_b200 import workloads as W  # noqa: E402

METRIC = "tokens/s and TFLOP/s (% of bf16 TC peak) for chunkwise gated-delta fwd, 1 B200"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# fp32 FMA issue on the CUDA cores: 148 SMs x 128 lanes x 2 FLOP x 1965 MHz (max SM clock)
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=4,
                    help="workload index (default 4: long_strong_decay_bf16, the largest)")
    ap.add_argument("--chunk", type=int, default=0)
    ap.add_argument("--T", type=int, default=0,
                    help="tokens per sequence instead of the workload's own (reduced-size "
                         "profiling captures; the JSON config records it)")
    ap.add_argument("--inverse", default="exact", choices=["exact", "neumann", "neumann1"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--kernel", default="auto", choices=["auto", "tc", "tc2", "tc2w", "simt", "simt2"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--epilogue", action="store_true",
                    help="add the readout epilogue (output gate times per-value-head RMSNorm, "
                         "unit weight) to every step, device-timed and end to end")
    ap.add_argument("--pass", dest="which", default="forward", choices=["forward", "backward"],
                    help="backward: time gdr_chunk_bwd (exact inverse; seeded upstream gradients)")
    ap.add_argument("--momentum", type=float, default=None,
                    help="time gdr_chunk_fwd_momentum with this mu (seeded 0/1 kappa per chunk)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# algorithmic work of one pass (per token and key head, summed over the workload)
def algorithmic(w: W.Workload, chunk: int, inverse: str, order=4, resid=1):
    C, dk, Dv, G = chunk, w.dk, w.R * w.dv, w.G
    s_in = 4 if w.in_dtype == "f32" else 2
    s_out = s_in
    if inverse == "exact":
        inv = C * C / 3.0
    elif inverse == "neumann1":
        # 16 x 16 diagonal blocks (triangular solves) and two triangular-times-dense
        # 16 x 16 products per block pair below them, per token of the chunk
        nb = (C + 15) // 16
        inv = (2.0 * nb * 16 ** 3 / 3.0 + nb * (nb - 1) * 16 ** 3) / C
    else:
        inv = (order - 1 + 2 * resid) * C * C / 3.0
    flop_tok = 3 * C * dk + 2 * C * Dv + 6 * dk * Dv + inv
    byte_tok = 2 * dk * s_in + Dv * s_in + Dv * s_out + 4 * G + 4
    units = w.B * w.Hk * w.T
    state = w.B * w.Hk * dk * Dv * 4 * (2 if w.s0_std > 0 else 1)
    return flop_tok * units, byte_tok * units + state


def roofline(flop: float, byts: float, ms: float, peaks: dict) -> dict:
    """The bound (HBM or tensor) whose time at peak is the larger for this work,
    the achieved rate against it, and both fractions."""
    s = ms * 1e-3
    hbm_frac = (byts / s) / (peaks["hbm_gbs"] * 1e9)
    tc_frac = (flop / s) / (peaks["bf16_tflops"] * 1e12)
    if byts / (peaks["hbm_gbs"] * 1e9) >= flop / (peaks["bf16_tflops"] * 1e12):
        roof = {"bound": "hbm", "achieved": byts / s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": hbm_frac}
    else:
        roof = {"bound": "tensor", "achieved": flop / s / 1e12, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": tc_frac}
    roof["hbm_frac"], roof["tc_frac"] = hbm_frac, tc_frac
    return roof


def rank_seed(workload_index: int, rank: int) -> int:
    """Each rank draws its own copy of the workload (weak scaling, independent
    sequences); rank 0 uses the standard seed."""
    return 1000 + workload_index + 7919 * rank


def max_over_ranks(ms: float, dist, device) -> float:
    """Slowest rank's time: the whole job is done when the last rank is."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_rank_step: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes its own tokens each step."""
    return world * tokens_per_rank_step / (ms_per_step * 1e-3)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def files_fingerprint(files):
    h = hashlib.sha1()
    for name in files:
        with open(os.path.join(ROOT, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:12]


def recorded_traffic(workload_name: str, chunk: int, inverse: str, kernel: str):
    """DRAM bytes per step (all of the step's launches) from a committed ncu summary
    (profiles/traffic.json), or None if there is none or the kernels' source files
    changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get("%s/C%d/%s/%s" % (workload_name, chunk, inverse, kernel))
    if not e:
        return None
    try:
        if files_fingerprint(e["files"]) != e["fingerprint"]:
            return None
    except OSError:
        return None
    return e.get("bytes_per_launch")


# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, flag in zip(names, parts[5:9]):
                if flag.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        loaded = [s for s in sm if s > 0.5 * (mx or max(sm))] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
def oracle_sample(w: W.Workload, x: dict, chunk: int, inverse: str, budget_s: float = 12.0):
    """Time the fp64 oracle on a bounded sample of the workload's sequences on
    all host cores: a prefix of each sequence's tokens (the oracle's cost per token
    does not depend on the position), grown towards the time budget, then more
    sequences.  Returns (tokens/s equivalent, threads, description, seconds)."""
    import oracle
    threads = max(1, oracle.max_threads())
    total = w.B * w.Hv

    def run(n, tl):
        seqs = [(s // w.Hv, s % w.Hv) for s in range(n)]
        xs = {}
        for name in ("q", "k", "g", "beta"):
            xs[name] = np.ascontiguousarray(np.stack([x[name][b, hv // w.R, :tl] for b, hv in seqs])[:, None])
        xs["v"] = np.ascontiguousarray(np.stack([x["v"][b, hv, :tl] for b, hv in seqs])[:, None])
        xs["S0"] = None if x["S0"] is None else np.stack([x["S0"][b, hv] for b, hv in seqs])[:, None]
        t0 = time.perf_counter()
        if inverse == "exact":
            oracle.recurrent(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], xs["S0"],
                             nthreads=threads)
        else:
            oracle.chunked(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], xs["S0"],
                           chunk=chunk, inverse=inverse, nthreads=threads)
        return time.perf_counter() - t0

    n = min(total, threads)
    tl = min(w.T, 2048)
    dt = run(n, tl)
    if tl < w.T and dt < budget_s:    # longer prefixes (whole chunks) towards the budget
        tl2 = min(w.T, max(tl, int(tl * budget_s / max(dt, 1e-3)) // 128 * 128))
        if tl2 > tl:
            tl = tl2
            dt = run(n, tl)
    if tl == w.T and dt < budget_s:   # then more sequences (multiples of the thread count)
        want = int(n * max(1.0, budget_s / max(dt, 1e-3)))
        n2 = min(total, max(n, (want // threads) * threads))
        if n2 > n:
            dt = run(n2, tl)
            n = n2
    tokens = n * tl / w.Hv             # value-head sequences -> tokens of B*T
    kind = "recurrent" if inverse == "exact" else "chunked-" + inverse
    desc = "%d of %d (batch, value-head) sequences, the first %d of their %d tokens, fp64 %s" % (
        n, total, tl, w.T, kind)
    return tokens / dt, threads, desc, dt


# ---------------------------------------------------------------------------
def run_reference(args, w, chunk, rank):
    if rank != 0:
        return 0
    x = W.make_inputs(w, rank_seed(args.workload, 0))
    times, rate_list = [], []
    desc, threads = "", 1
    variant = args.which == "backward" or args.momentum is not None
    up, kappa = None, None
    if variant:   # the same seeded upstream gradients / kappa as the GPU arm's rank 0
        rng = np.random.default_rng(7200 + args.workload)
        if args.which == "backward":
            up = (rng.standard_normal((w.B, w.Hv, w.T, w.dv)).astype(np.float32), None)
        else:
            kappa = (rng.random((w.B, (w.T + chunk - 1) // chunk)) >= 0.125).astype(np.int32)
    for step in range(args.warmup + args.steps):
        if variant:
            t0 = time.perf_counter()
            rate, threads, desc = oracle_variant_sample(w, x, chunk, up, args.momentum, kappa,
                                                        budget_s=2.0)
            dt = time.perf_counter() - t0
        else:
            rate, threads, desc, dt = oracle_sample(w, x, chunk, args.inverse, budget_s=2.0)
        if step >= args.warmup:
            rate_list.append(rate)
            times.append(dt)
    value = statistics.median(rate_list)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.median(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": (dict(config_dict(w, chunk, "exact", args.gpus),
                        which=("backward" if args.which == "backward" else "momentum mu=%g" % args.momentum))
                   if variant else config_dict(w, chunk, args.inverse, args.gpus)),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": desc + " per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(w, chunk, inverse, world):
    in_bytes = (w.B * w.T * (2 * w.Hk * w.dk + w.Hv * w.dv) * (2 if w.in_dtype == "bf16" else 4)
                + w.B * w.Hk * w.T * (w.G + 1) * 4)
    return {"workload": w.name, "B": w.B, "T": w.T, "Hk": w.Hk, "Hv": w.Hv, "dk": w.dk,
            "dv": w.dv, "G": w.G, "chunk": chunk, "inverse": inverse,
            "in_dtype": w.in_dtype, "S0": w.s0_std > 0,
            "parallelism": "replicas" if world > 1 else "single",
            "l2": ("inputs larger than L2" if in_bytes >= L2_BYTES
                   else "L2 flushed between steps")}


def oracle_variant_sample(w, x, chunk, up, mu, kappa, budget_s=12.0, t_cap=256):
    """The oracle on a bounded sample for the backward (recurrent_grad over whole key
    heads, the first t_cap tokens: it keeps every token's state) or for momentum
    (the chunked form with momentum, whole sequences).  Returns (tokens/s, threads,
    description)."""
    import oracle
    threads = max(1, oracle.max_threads())

    def run(n):
        heads = [(s // w.Hk, s % w.Hk) for s in range(n)]
        vh = lambda b, hk: [x_ for x_ in range(hk * w.R, (hk + 1) * w.R)]
        T = min(w.T, t_cap) if up is not None else w.T
        key = lambda name: np.stack([x[name][b, hk, :T] for b, hk in heads])[:, None]
        val = lambda arr: np.stack([arr[b, vh(b, hk), :T] for b, hk in heads])
        q, k, g, beta = key("q"), key("k"), key("g"), key("beta")
        v = val(x["v"])
        S0 = None if x["S0"] is None else np.stack([x["S0"][b, vh(b, hk)] for b, hk in heads])
        t0 = time.perf_counter()
        if up is not None:
            oracle.recurrent_grad(q, k, v, g, beta, S0, val(up[0]), None, nthreads=threads)
        else:
            kap = None if kappa is None else np.stack([kappa[b] for b, _ in heads])
            oracle.chunked(q, k, v, g, beta, S0, chunk=chunk, mu=mu, kappa=kap, nthreads=threads)
        return time.perf_counter() - t0, T

    total = w.B * w.Hk
    n = min(total, threads)
    dt, T = run(n)
    want = int(n * max(1.0, budget_s / max(dt, 1e-3)))
    n2 = min(total, max(n, (want // threads) * threads))
    if n2 > n:
        (dt, T), n = run(n2), n2
    tokens = n * T / w.Hk
    what = ("fp64 recurrent_grad (reverse sweep), first %d tokens" % T if up is not None
            else "fp64 chunked form with momentum, all %d tokens" % T)
    return tokens / dt, threads, "%d of %d (batch, key-head) sequences with their %d value heads, %s" % (
        n, total, w.R, what)


def run_variant(args, w, chunk, rank, world, local):
    """--pass backward (gdr_chunk_bwd) or --momentum MU (gdr_chunk_fwd_momentum): the
    same timing rules and JSON line as the forward, for these CUDA-core paths."""
    import torch
    from gated_delta_rule_141_b200 import gdr
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    backward = args.which == "backward"
    x = W.make_inputs(w, rank_seed(args.workload, rank))
    dt_in = torch.bfloat16 if w.in_dtype == "bf16" else torch.float32
    dev = {n: torch.from_numpy(x[n]).to("cuda").to(dt_in) for n in ("q", "k", "v")}
    dev["g"] = torch.from_numpy(x["g"]).cuda()
    dev["beta"] = torch.from_numpy(x["beta"]).cuda()
    dev["S0"] = None if x["S0"] is None else torch.from_numpy(x["S0"]).cuda()
    rng = np.random.default_rng(7200 + args.workload + 7919 * rank)
    up, kappa = None, None
    if backward:   # upstream gradients ~ N(0, 1)
        up = (rng.standard_normal((w.B, w.Hv, w.T, w.dv)).astype(np.float32),
              rng.standard_normal((w.B, w.Hv, w.dk, w.dv)).astype(np.float32))
        dev["dO"], dev["dS_final"] = torch.from_numpy(up[0]).cuda(), torch.from_numpy(up[1]).cuda()
    else:          # kappa: 0 with probability 1/8 per chunk (a document reset inside it)
        kappa = (rng.random((w.B, (w.T + chunk - 1) // chunk)) >= 0.125).astype(np.int32)
        dev["kappa"] = torch.from_numpy(kappa).cuda()
    # the backward runs on the CUDA cores; momentum on the two-pass tensor-core path when
    # it applies (bf16, dk = 128, chunk 64), else on the CUDA cores
    vkernel = "simt" if backward else ("auto" if args.kernel == "auto" else args.kernel)
    shape = gdr.make_shape(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv,
                           gdr.BF16 if w.in_dtype == "bf16" else gdr.F32,
                           gdr.BF16 if w.in_dtype == "bf16" else gdr.F32, kernel=vkernel)
    gm = gdr.gate_mode_for(w.G, w.dk)
    ws = None
    if backward:
        nb = gdr.bwd_workspace_bytes(shape, chunk, gm)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda") if nb else None
    on_tc2 = False
    if not backward and vkernel != "simt":
        tc2_shape = gdr.make_shape(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv, gdr.BF16 if w.in_dtype == "bf16"
                                   else gdr.F32, gdr.BF16 if w.in_dtype == "bf16" else gdr.F32,
                                   kernel="tc2")
        on_tc2 = (w.in_dtype == "bf16" and w.dk == 128 and chunk == 64 and w.dv % 64 == 0)
        if on_tc2:
            nb = gdr.workspace_bytes(tc2_shape, chunk, gm)
            ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    in_bytes = sum(t.numel() * t.element_size() for t in dev.values() if t is not None)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda") if in_bytes < L2_BYTES else None
    stream = torch.cuda.current_stream()
    out = {}

    def call(d):
        if backward:
            out["g"] = gdr.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d["dO"],
                                     d["dS_final"], chunk=chunk, gate_mode=gm, kernel="simt",
                                     workspace=ws, stream=stream)
        else:
            out["o"] = gdr.chunk_fwd_momentum(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"],
                                              mu=args.momentum, kappa=d["kappa"], chunk=chunk,
                                              gate_mode=gm, kernel="tc2" if on_tc2 else "simt",
                                              workspace=ws, stream=stream)

    step_events = []

    def step(timed=False):
        if flush is not None:
            flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call(dev)
        e1.record(stream)
        if timed:
            step_events.append((e0, e1))

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    sampler = ClockSampler(local)
    with sampler:
        barrier()
        for _ in range(args.steps):
            step(timed=True)
        barrier()
    ms_step = max_over_ranks(sum(a.elapsed_time(b) for a, b in step_events), dist,
                             torch.device("cuda", local)) / args.steps
    tokens_step = w.B * w.T
    value = job_tokens_per_s(world, tokens_step, ms_step)
    flop, byts = algorithmic(w, chunk, "exact")
    if backward:   # the forward recomputed once, its chunk products run backwards twice
        flop *= 3
        byts = 2 * byts + 4 * w.B * w.Hv * w.T * w.dv * 2 + 4 * w.B * w.Hk * w.T * (2 * w.dk + w.G + 1)
    achieved = flop / (ms_step * 1e-3) / 1e12
    if on_tc2:   # the forward's roofline: the same algorithmic work, the same two passes
        peaks, peak_src = measured_peaks()
        roof = roofline(flop, byts, ms_step, peaks)
        roof.update(peak_source=peak_src + " (burst)", traffic=None, kernel="tc2",
                    tflops=achieved)
    else:
        roof = {"bound": "alu", "achieved": achieved, "peak": FP32_ALU_TFLOPS, "unit": "TFLOP/s",
                "frac": achieved / FP32_ALU_TFLOPS, "traffic": None,
                "peak_source": "fp32 FMA on the CUDA cores from unit counts and the max SM clock",
                "kernel": "simt", "hbm_gbs": byts / (ms_step * 1e-3) / 1e9}
    # kernels launched per step: backward = forward recompute, 4 zero fills, the backward;
    # momentum on the two-pass path: pass 1 and the state pass
    launches = 6 if backward else (2 if on_tc2 else 1)

    e2e = None
    if not args.no_e2e:
        host = {n: (None if t is None else t.cpu().pin_memory()) for n, t in dev.items()}
        dbuf = {n: (None if t is None else torch.empty_like(t)) for n, t in dev.items()}
        h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
        if backward:
            res = {n: torch.empty(tuple(t.shape), dtype=torch.float32).pin_memory()
                   for n, t in gdr.chunk_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"],
                                             dev["S0"], dev["dO"], dev["dS_final"], chunk=chunk,
                                             gate_mode=gm, kernel="simt", workspace=ws,
                                             stream=stream).items() if t is not None}
        else:
            res = {"o": torch.empty((w.B, w.Hv, w.T, w.dv), dtype=dt_in).pin_memory(),
                   "S_final": torch.empty((w.B, w.Hv, w.dk, w.dv), dtype=torch.float32).pin_memory()}
        d2h = sum(t.numel() * t.element_size() for t in res.values())

        def e2e_step():
            with torch.cuda.stream(stream):
                for n in dev:
                    if host[n] is not None:
                        dbuf[n].copy_(host[n], non_blocking=True)
                call(dbuf)
                got = out["g"] if backward else dict(zip(("o", "S_final"), out["o"]))
                for n, t in res.items():
                    t.copy_(got[n], non_blocking=True)

        for _ in range(2):
            e2e_step()
        barrier()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, min(args.steps, 10))
        ev0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        ev1.record(stream)
        barrier()
        ms_e2e = max_over_ranks(ev0.elapsed_time(ev1), dist, torch.device("cuda", local)) / n_e2e
        e2e = {"value": job_tokens_per_s(world, tokens_step, ms_e2e), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, threads, desc = oracle_variant_sample(w, x, chunk, up, args.momentum, kappa)
        cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    what = "backward (gdr_chunk_bwd)" if backward else "forward with momentum mu=%g" % args.momentum
    line = {
        "metric": "tokens/s of the chunkwise gated-delta %s, %s" % (
            what, "two-pass tensor-core path" if on_tc2 else "CUDA-core kernels"),
        "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if on_tc2 else "f32",
        "data": "synthetic (seeded numpy PCG64, distributions of the workload)",
        "config": dict(config_dict(w, chunk, "exact", world), which=what,
                       kernel="tc2" if on_tc2 else "simt"),
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": args.steps * launches, "clocks": sampler.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = W.WORKLOADS[args.workload]
    if args.T:
        w = w.scaled(T=args.T)
    chunk = args.chunk or w.chunk
    if args.impl == "reference":
        return run_reference(args, w, chunk, rank)
    if args.which == "backward" or args.momentum is not None:
        return run_variant(args, w, chunk, rank, world, local)

    import torch
    from gated_delta_rule_141_b200 import gdr
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    x = W.make_inputs(w, rank_seed(args.workload, rank))
    dt_in = torch.bfloat16 if w.in_dtype == "bf16" else torch.float32
    dev = {n: torch.from_numpy(x[n]).to("cuda").to(dt_in) for n in ("q", "k", "v")}
    dev["g"] = torch.from_numpy(x["g"]).cuda()
    dev["beta"] = torch.from_numpy(x["beta"]).cuda()
    dev["S0"] = None if x["S0"] is None else torch.from_numpy(x["S0"]).cuda()
    o = torch.empty((w.B, w.Hv, w.T, w.dv), dtype=dt_in, device="cuda")
    Sf = torch.empty((w.B, w.Hv, w.dk, w.dv), dtype=torch.float32, device="cuda")
    in_bytes = sum(t.numel() * t.element_size() for t in dev.values() if t is not None)
    flush = None
    if in_bytes < L2_BYTES:
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    shape_run = gdr.make_shape(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv,
                               gdr.BF16 if w.in_dtype == "bf16" else gdr.F32,
                               gdr.BF16 if w.in_dtype == "bf16" else gdr.F32, kernel=args.kernel)
    gm_run = gdr.gate_mode_for(w.G, w.dk)
    ws_bytes = gdr.workspace_bytes(shape_run, chunk, gm_run, args.inverse)
    workspace = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda") if ws_bytes else None
    kern = gdr.select_kernel(shape_run, chunk, gm_run, args.inverse)
    # the two-pass path: pass 1, then one state pass, or three when segmented
    two_pass = kern in (gdr.KERNEL_TC2, gdr.KERNEL_TC2W)
    nseg = gdr.state_segments(shape_run, chunk, gm_run, args.inverse) if two_pass else 0
    # Neumann at chunk 128 on the two-pass path adds the pair kernel after pass 1
    pair = two_pass and args.inverse in ("neumann", "neumann1") and chunk == 128
    launches_per_step = ((1 + (1 if nseg == 1 else 3) + (1 if pair else 0)) if two_pass
                         else 2 if kern == gdr.KERNEL_SIMT2 else 1)
    zgate = None
    if args.epilogue:   # output-gate logits z ~ N(0, 1), seeded apart from the workload's draws
        zr = np.random.default_rng(7000 + args.workload).standard_normal(tuple(o.shape)).astype(np.float32)
        zgate = torch.from_numpy(zr).cuda().to(o.dtype)
        launches_per_step += 1
    # with an L2 flush between steps, only the launches themselves are timed
    step_events = []

    def step(timed=False):
        if flush is not None:
            flush.zero_()
        if timed and flush is not None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        gdr.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"],
                      chunk=chunk, inverse=args.inverse, o=o, S_final=Sf, kernel=args.kernel,
                      workspace=workspace, stream=stream)
        if zgate is not None:
            gdr.output_gate_rmsnorm(o, zgate, None, eps=1e-6, stream=stream)
        if timed and flush is not None:
            e1.record(stream)
            step_events.append((e0, e1))

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    if gdr.device_status(stream) != gdr.OK:
        raise RuntimeError("device status reported a timeout during warm-up")

    sampler = ClockSampler(local)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with sampler:
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            step(timed=True)
        ev1.record(stream)
        barrier()
    ms_total = ev0.elapsed_time(ev1)
    if step_events:
        ms_total = sum(a.elapsed_time(b) for a, b in step_events)
    ms_total = max_over_ranks(ms_total, dist, torch.device("cuda", local))
    ms_step = ms_total / args.steps
    tokens_step = w.B * w.T
    value = job_tokens_per_s(world, tokens_step, ms_step)

    # kernel-only launch time, for the roofline (no L2 flush between launches
    # when the inputs exceed L2 anyway)
    flop, byts = algorithmic(w, chunk, args.inverse)
    if args.epilogue:   # the epilogue reads o and z and writes o once more
        byts += 3 * o.numel() * o.element_size()
    peaks, peak_src = measured_peaks()
    roof = roofline(flop, byts, ms_step, peaks)
    roof["peak_source"] = peak_src + " (burst)"
    roof["traffic"] = recorded_traffic(w.name, chunk, args.inverse,
                                       gdr.KERNEL_NAMES.get(kern, str(kern)))
    roof["tflops"] = flop / (ms_step * 1e-3) / 1e12
    roof["kernel"] = gdr.KERNEL_NAMES.get(kern, str(kern))
    roof["launches_per_step"] = launches_per_step

    # end to end through the host-buffer entry point
    e2e = None
    if not args.no_e2e:
        host = {n: (None if t is None else t.cpu().pin_memory()) for n, t in dev.items()}
        host["o"] = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        host["S_final"] = torch.empty(Sf.shape, dtype=torch.float32).pin_memory()
        dbuf = {n: (None if t is None else torch.empty_like(t)) for n, t in dev.items()}
        dbuf["o"], dbuf["S_final"] = torch.empty_like(o), torch.empty_like(Sf)
        shape, gm = shape_run, gm_run
        h2d = sum(t.numel() * t.element_size() for n, t in host.items()
                  if t is not None and n not in ("o", "S_final"))
        d2h = host["o"].numel() * host["o"].element_size() + host["S_final"].numel() * 4
        e2e_steps = max(3, min(args.steps, 20))
        if zgate is not None:
            host["z"], dbuf["z"] = zgate.cpu().pin_memory(), torch.empty_like(zgate)
            h2d += host["z"].numel() * host["z"].element_size()

        def e2e_step():
            if zgate is None:
                gdr.chunk_fwd_host(host, dbuf, shape, chunk, gm, args.inverse, workspace, stream)
                return
            # with the epilogue: the same copies around the device entry points
            with torch.cuda.stream(stream):
                for n in dev:
                    if host[n] is not None:
                        dbuf[n].copy_(host[n], non_blocking=True)
                dbuf["z"].copy_(host["z"], non_blocking=True)
                gdr.chunk_fwd(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["g"], dbuf["beta"], dbuf["S0"],
                              chunk=chunk, inverse=args.inverse, o=dbuf["o"], S_final=dbuf["S_final"],
                              kernel=args.kernel, workspace=workspace, stream=stream)
                gdr.output_gate_rmsnorm(dbuf["o"], dbuf["z"], None, eps=1e-6, stream=stream)
                host["o"].copy_(dbuf["o"], non_blocking=True)
                host["S_final"].copy_(dbuf["S_final"], non_blocking=True)

        for _ in range(2):
            e2e_step()
        barrier()
        ev0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        ev1.record(stream)
        barrier()
        ms_e2e = max_over_ranks(ev0.elapsed_time(ev1), dist, torch.device("cuda", local))
        e2e = {"value": job_tokens_per_s(world, tokens_step, ms_e2e / e2e_steps), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, threads, desc, _ = oracle_sample(w, x, chunk, args.inverse)
        cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc}

    kchunk = gdr.kernel_chunk(shape_run, chunk, gm_run, args.inverse)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.in_dtype == "bf16" else "f32",
        "data": "synthetic (seeded numpy PCG64, distributions of the workload)",
        "config": dict(config_dict(w, chunk, args.inverse, world), kernel_chunk=kchunk,
                       state_segments=nseg, epilogue=bool(args.epilogue)),
        "tflops": roof["tflops"], "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": args.steps * launches_per_step, "kernel": gdr.KERNEL_NAMES.get(kern, str(kern)),
        "clocks": sampler.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
