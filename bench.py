#!/usr/bin/env python
"""Benchmark of the gated-delta-rule library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl gdn|reference]

One step = one ``gdn_forward`` call over the long-sequence workload (bf16
q/k/v, float32 gates and state, B=1, H=16, T=65536, dk=dv=128, chunk=64,
slow-decay gates) with inputs resident in HBM.  The single-token decode path
(B=64, H=16, d=128, state 134 MB) is timed in its own region and reported in
the same line under ``decode``.  Under torchrun every rank runs its own
independent replica (the (batch, head) problems are independent: weak
scaling, no collective on the data path); times are device times (CUDA
events on the launching stream), max over ranks.

The JSON line also carries ``e2e`` (the same metric through the C ABI with
pinned host buffers, copies inside the timed region), ``kernels`` (device
time, share and algorithmic rates of each kernel kind of the forward, from
CUDA events the library records around each launch inside the timed
region), ``roofline`` of the dominant one, ``clocks`` sampled with
nvidia-smi during the run, and ``cpu_baseline`` (the float64 oracle on a
bounded sample, host cores).
``--impl reference`` times the float64 CPU oracle as the reference arm.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gdn_inputs import (WORKLOADS, as_f32_numpy, decode_inputs, forward_inputs, length_mix, raw_inputs,  # noqa: E402
                        varlen_inputs)

FWD_WORKLOAD = "fwd_bf16_b1h16_t64k_d128"
# the serving decode workload at batch 64 (state 67 MB, 134 MB read and written per step, partly served by
# the 126 MB L2) and one whose state (268 MB, 537 MB per step) is twice L2, so that its HBM fraction is not
# helped by the cache
DEC_WORKLOADS = ("decode_bf16_b64h16_d128_x1024", "decode_bf16_b256h16_d128_x256")
METRIC = "gated-delta forward tokens/s & TFLOP/s vs BF16 roofline; decode GB/s vs HBM peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- unit counts
def fwd_flop_per_token_head(dk, dv, C):
    """Full-tile contractions of the chunkwise method per token and head:
    K K^T, Q K^T, T.(beta gamma K), T.(beta V), P.U  (2C(3dk + 2dv))
    and W S^T, Q S^T, U^T Ktil (6 dk dv)."""
    return 2 * C * (3 * dk + 2 * dv) + 6 * dk * dv


def fwd_bytes(B, T, H, dk, dv, es, s0, s_final):
    """Compulsory HBM bytes of one forward: q, k, v, out, two float32 gates, and the states."""
    per_tok_head = (2 * dk + 2 * dv) * es + 8
    return B * T * H * per_tok_head + (int(s0) + int(s_final)) * B * H * dv * dk * 4


def decode_bytes_per_head_step(dk, dv, es):
    return 2 * dk * dv * 4 + (2 * dk + 2 * dv) * es + 8


# Counted FLOP of each kernel kind per token-head: the method's contractions assigned to the kernel
# that performs them.  The prep kernel forms K K^T, Q K^T (one [Q;K] K^T product) and W = T diag(beta
# gamma) K; the chain kernel forms Ut = T diag(beta) V, P U, W S^T, Q S^T and U^T Ktil.  They sum to
# fwd_flop_per_token_head.  The transfer and prefix kernels exist only to cut long sequences into
# segments: their arithmetic is overhead and earns no count.
def counted_flop_per_token_head(kind, dk, dv, C):
    if kind == "prep":
        return 6 * C * dk
    if kind == "chain":
        return 4 * C * dv + 6 * dk * dv
    if kind == "fused":
        return fwd_flop_per_token_head(dk, dv, C)
    return 0


def source_sha(relpath):
    """First 16 hex digits of the sha256 of a source file of the repository."""
    import hashlib
    with open(os.path.join(ROOT, relpath), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def measured_traffic(profile):
    """DRAM bytes (read + write) per unit that an ncu capture recorded for each kernel kind, from the
    machine-readable lines of a summary under profiles/:
        traffic <kind> <source file> <sha256[:16] of that file at capture time> <bytes per unit>
    A kind whose source has changed since the capture is left out (its traffic is unknown)."""
    path = os.path.join(ROOT, "profiles", profile)
    out = {}
    if not os.path.exists(path):
        return out
    with open(path) as f:
        for line in f:
            m = re.match(r"\s*traffic\s+(\S+)\s+(\S+)\s+([0-9a-f]{16})\s+([0-9.eE+]+)\s*$", line)
            if m and os.path.exists(os.path.join(ROOT, m.group(2))) and source_sha(m.group(2)) == m.group(3):
                out[m.group(1)] = float(m.group(4))
    return out


FWD_TRAFFIC_PROFILE = "fwd_traffic_b1h16_t16k_d128.md"
DECODE_TRAFFIC_PROFILE = "decode_traffic_d128.md"


def kernel_units(kind, w, nseg):
    """Units one launch of a kernel kind processes, the unit its measured traffic is quoted per:
    token-heads (prep, chain, fused), segment boundaries times heads (transfer, prefix)."""
    nth = w.B * w.T * w.H
    if kind in ("prep", "chain", "fused"):
        return nth
    if kind in ("transfer", "prefix"):
        # a transfer CTA runs only as many chunks as its segment's decay makes necessary (the whole
        # segment when the gates barely decay), so its work is counted per segment boundary
        return w.B * w.H * max(nseg - 1, 0)
    return 0


def kernel_design_bytes(kind, w, es, nseg):
    """HBM bytes ONE launch of a kernel kind moves by this design (inputs, outputs and the two-kernel
    forward's per-chunk workspace: P and T diag(beta) at 2C bytes per token each, W^T at 2 dk, the
    gate record at 528 B per chunk).  This is the design's own traffic, not the algorithmic bytes:
    the compulsory bytes of the step are fwd_bytes."""
    C, dk, dv = w.chunk, w.dk, w.dv
    nth = w.B * w.T * w.H
    tile = 2 * C + 2 * C + 2 * dk + 528.0 / C
    if kind == "prep":
        return nth * (2 * dk * es + 8 + tile)
    if kind == "chain":
        return nth * ((2 * dk + 2 * dv) * es + tile)
    if kind == "transfer":
        return None  # data-dependent: the chunks a segment's decay requires (its measured traffic is reported)
    if kind == "prefix":
        return kernel_units(kind, w, nseg) * 3 * dv * dk * 4
    if kind == "fused":
        return nth * ((2 * dk + 2 * dv) * es + 8)
    return 0


# ---------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks/throttle sampling in the background (read-only queries)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: torch.device):
        try:
            self.dev = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.dev = str(device.index or 0)
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = max((float(r[2]) for r in rows if r[2].replace(".", "").isdigit()), default=None)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        loaded = [x for x in sm if smax and x > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(rows)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_info():
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return model, len(os.sched_getaffinity(0))


def fwd_config(w, raw, world):
    """The `config` object of the forward line, shared by the GPU arm and the reference arm so that
    both describe the same workload in the same words."""
    es = 2 if w.dtype == "bf16" else 4
    nbytes = fwd_bytes(w.B, w.T, w.H, w.dk, w.dv, es, w.s0_std is not None, True)
    return {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv, "chunk": w.chunk,
            "input_dtype": w.dtype, "state_dtype": "f32",
            "input_stage": "fused (raw q, k and gate logits)" if raw else "none (unit q, k; gates)",
            "parallelism": "replicas" if world > 1 else "single",
            "l2": "inputs larger than L2 (%.2f GB read+written per step)" % (nbytes / 1e9)}


# ---------------------------------------------------------------- oracle timing
def oracle_forward_sample(w, budget_s: float):
    """Float64 oracle on a bounded prefix of the forward workload (all heads of batch row 0,
    the first T' tokens), sized from a short calibration run to take about `budget_s`.
    Returns (tokens/s, cores, description)."""
    import oracle
    _, cores = cpu_info()
    threads = min(cores, w.B * w.H)  # the oracle parallelises over (b, h) only

    def run(Tp):
        inp = forward_inputs(1, Tp, w.H, w.dk, w.dv, w.dtype, seed=w.seed, alpha_mu=w.alpha_mu)
        args = [as_f32_numpy(inp[n]) for n in ("q", "k", "v", "log_alpha", "beta")]
        t0 = time.perf_counter()
        oracle.forward(*args, None, nthreads=threads)
        return time.perf_counter() - t0

    probe = 128
    dt = max(run(probe), 1e-4)
    Tp = int(max(probe, min(w.T, probe * budget_s / dt)))
    dt = run(Tp)
    return Tp / dt, threads, "oracle float64, batch row 0 of %s: H=%d, first %d of %d tokens, %d threads" % (
        w.name, w.H, Tp, w.T, threads), Tp, dt


# ---------------------------------------------------------------- reference arm
def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    model, cores = cpu_info()
    for _ in range(args.warmup):
        oracle_forward_sample(w, 0.5)
    times, toks = [], []
    for _ in range(args.steps):
        tps, threads, desc, Tp, dt = oracle_forward_sample(w, args.ref_step_seconds)
        times.append(dt)
        toks.append(Tp)
    value = sum(toks) / sum(times)
    sample = desc + "; CPU: " + model
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * statistics.mean(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": fwd_config(w, False, int(os.environ.get("WORLD_SIZE", "1"))),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "host_cores": cores,
                         "oracle_threads": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm
def time_region(fn, steps, stream, world):
    barrier(world)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return start.elapsed_time(end)  # ms


def time_decode(gdn, wd, dev, stream, world, rank, warmup, peaks, peak_kind):
    """Times wd.steps consecutive gdn_decode_step launches (replayed from a CUDA graph) on a decode
    workload whose inputs are all resident in HBM; returns its object of the JSON line."""
    dsteps = wd.steps
    di = decode_inputs(dsteps, wd.B, wd.H, wd.dk, wd.dv, wd.dtype, seed=wd.seed + 1000 * rank, s0_std=wd.s0_std)
    dd = {k: v.to(dev) for k, v in di.items()}
    del di
    S = dd["S"].clone()
    dout = torch.empty((dsteps, wd.B, wd.H, wd.dv), dtype=dd["q"].dtype, device=dev)

    def dec_run():
        for t in range(dsteps):
            gdn.decode_step(dd["q"][t], dd["k"][t], dd["v"][t], dd["log_alpha"][t], dd["beta"][t], S,
                            out=dout[t], stream=stream)

    for _ in range(max(1, warmup // 3)):
        dec_run()
    # The launches (each still one gdn_decode_step call through the C ABI) are captured once in a CUDA
    # graph and replayed: a Python call costs about as long as one decode kernel, and host overhead
    # must not leave the GPU idle inside the timed region.
    replay = dec_run
    graph = None
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            cap = torch.cuda.current_stream()
            for t in range(dsteps):
                gdn.decode_step(dd["q"][t], dd["k"][t], dd["v"][t], dd["log_alpha"][t], dd["beta"][t], S,
                                out=dout[t], stream=cap)
        graph.replay()
        torch.cuda.synchronize()
        replay = graph.replay
    except RuntimeError:
        torch.cuda.synchronize()
    dms = time_region(replay, 1, stream, world) / dsteps
    dms = max_over_ranks(dms, world)
    des = 2 if wd.dtype == "bf16" else 4
    dbytes = wd.B * wd.H * decode_bytes_per_head_step(wd.dk, wd.dv, des)
    dgbs = dbytes / (dms / 1e3) / 1e9
    tr_unit = measured_traffic(DECODE_TRAFFIC_PROFILE).get("decode_b%d" % wd.B)
    res = {"workload": wd.name, "steps": dsteps, "us_per_step": dms * 1e3,
           "state_bytes": wd.B * wd.H * wd.dv * wd.dk * 4,
           "launch": "cuda_graph" if replay is not dec_run else "eager",
           "tokens_per_s": world * wd.B / (dms / 1e3), "GB_per_s": dgbs,
           "roofline": {"bound": "hbm", "achieved": dgbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": dgbs / peaks["hbm_gbs"],
                        "traffic": None if tr_unit is None else tr_unit * wd.B * wd.H,
                        "traffic_source": "profiles/" + DECODE_TRAFFIC_PROFILE,
                        "peak_kind": peak_kind, "bytes_per_launch": dbytes},
           "launches": dsteps}
    del dd, S, dout, graph, replay
    torch.cuda.empty_cache()
    return res


def run_decode_only(args, world, rank):
    """One decode workload alone (for profiler captures of the decode kernel)."""
    import gated_delta_rule_142_b200 as gdn
    gdn.load()
    peaks, peak_kind = load_peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    res = time_decode(gdn, WORKLOADS[args.decode_only], dev, torch.cuda.current_stream(dev), world, rank,
                      args.warmup, peaks, peak_kind)
    if rank == 0:
        print(json.dumps({"decode": res}), flush=True)
    return 0


def run_gdn(args, world, rank, local):
    import gated_delta_rule_142_b200 as gdn
    from gated_delta_rule_142_b200 import build as gdn_build
    if not os.path.exists(gdn.LIBRARY):
        gdn_build.build()
    gdn.load()
    peaks, peak_kind = load_peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    sampler = ClockSampler(dev)
    sampler.start()

    # ---- forward, inputs resident in HBM ----
    w = WORKLOADS[args.workload]
    if args.tokens:
        # a shorter sequence of the same workload, for profiler captures that must stay small
        w = dataclasses.replace(w, T=args.tokens, name="%s_first%d" % (w.name, args.tokens))
    es = 2 if w.dtype == "bf16" else 4
    if args.raw:
        # the layer's raw projections: q, k unnormalised, gate logits in place of the gates; the
        # step then includes the input stage
        r = raw_inputs((w.B, w.T, w.H), w.dk, w.dv, w.dtype, seed=w.seed + 1000 * rank,
                       s0_shape=(w.B, w.H, w.dv, w.dk), s0_std=w.s0_std, alpha_mu=w.alpha_mu)
        inp = {"q": r["q"], "k": r["k"], "v": r["v"], "log_alpha": r["x_alpha"], "beta": r["x_beta"], "S0": r["S0"]}
    else:
        inp = forward_inputs(w.B, w.T, w.H, w.dk, w.dv, w.dtype, seed=w.seed + 1000 * rank, s0_std=w.s0_std,
                             alpha_mu=w.alpha_mu)
    w_cfg = w  # the workload as the reference arm names it (the raw flag goes into the config)
    fwd = gdn.forward_raw if args.raw else gdn.forward
    d = {k: (None if v is None else v.to(dev)) for k, v in inp.items()}
    out = torch.empty((w.B, w.T, w.H, w.dv), dtype=d["q"].dtype, device=dev)
    Sf = torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device=dev)

    def fwd_step():
        fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], chunk=w.chunk, out=out,
                    S_final=Sf, stream=stream)

    for _ in range(args.warmup):
        fwd_step()
    # per-kernel device times: every launch inside the timed region is bracketed by CUDA events on
    # the launching stream (host-side records only)
    gdn.timing_start()
    ms = time_region(fwd_step, args.steps, stream, world)
    ktimes = gdn.timing_stop()
    ms_step = max_over_ranks(ms / args.steps, world)
    tokens = w.B * w.T
    value = world * tokens / (ms_step / 1e3)
    flop = w.B * w.T * w.H * fwd_flop_per_token_head(w.dk, w.dv, w.chunk)
    nbytes = fwd_bytes(w.B, w.T, w.H, w.dk, w.dv, es, w.s0_std is not None, True)
    tflops = flop / (ms_step / 1e3) / 1e12
    gbs = nbytes / (ms_step / 1e3) / 1e9
    scratch_bytes, launches_per_fwd = gdn.forward_plan(w.B, w.T, w.H, w.dk, w.dv, w.chunk, d["q"].dtype)
    chunks = -(-w.T // w.chunk)
    ws_tiles = w.B * w.H * chunks * (32768 + 528)
    nseg = 1 + max(0, scratch_bytes - ws_tiles) // (3 * w.B * w.H * w.dv * w.dk * 4) if "prep" in ktimes else 1
    traffic_unit = measured_traffic(FWD_TRAFFIC_PROFILE)
    kernels = {}
    step_traffic = 0.0
    for kind, (kms, n) in ktimes.items():
        per = kms / n
        cf = counted_flop_per_token_head(kind, w.dk, w.dv, w.chunk)
        kflop = w.B * w.T * w.H * cf
        by = kernel_design_bytes(kind, w, es, nseg)
        units = kernel_units(kind, w, nseg)
        tr = traffic_unit[kind] * units if kind in traffic_unit else None
        kernels[kind] = {"launches_per_step": n / args.steps, "ms_per_launch": per, "share": kms / (ms * 1.0),
                         "counted_flop_per_token_head": cf, "counted_flop_per_launch": kflop,
                         "counted_tflops": kflop / (per / 1e3) / 1e12,
                         "design_bytes_per_launch": by,
                         "design_gb_per_s": None if by is None else by / (per / 1e3) / 1e9,
                         "traffic_per_launch": tr}
        step_traffic = None if (step_traffic is None or tr is None) else step_traffic + tr * n / args.steps
    top = max(kernels, key=lambda k: ktimes[k][0]) if kernels else None
    # roofline of the whole step: the counted FLOP of the chunkwise method over the step's
    # device time against the measured dense bf16 peak (burst: the step is timed as a short burst of
    # launches), and the compulsory bytes against the measured copy bandwidth beside it.
    roof = {"bound": "tensor", "kernel": "forward step (%d launches)" % launches_per_fwd,
            "achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": tflops / peaks["bf16_tflops"], "peak_kind": peak_kind + " bf16 burst",
            "flop_per_step": flop, "flop_per_token_head": fwd_flop_per_token_head(w.dk, w.dv, w.chunk),
            "hbm": {"achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                    "compulsory_bytes_per_step": nbytes},
            "traffic": step_traffic,
            "traffic_over_compulsory": None if step_traffic is None else step_traffic / nbytes,
            "traffic_source": "profiles/" + FWD_TRAFFIC_PROFILE,
            "dominant_kernel": top}

    # ---- decode: consecutive single-token steps, each its own launch ----
    decs = [time_decode(gdn, WORKLOADS[n], dev, stream, world, rank, args.warmup, peaks, peak_kind)
            for n in ([] if args.no_decode else DEC_WORKLOADS)]
    dec = decs[0] if decs else None
    clocks = sampler.stop()

    # ---- e2e: same forward through the C ABI with pinned host buffers ----
    e2e = None
    if not args.no_e2e:
        h = {k: (None if v is None else v.pin_memory()) for k, v in inp.items()}
        hout = torch.empty((w.B, w.T, w.H, w.dv), dtype=h["q"].dtype).pin_memory()
        hSf = torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32).pin_memory()

        def e2e_step():
            fwd(h["q"], h["k"], h["v"], h["log_alpha"], h["beta"], h["S0"], chunk=w.chunk, out=hout,
                        S_final=hSf, stream=stream)

        e2e_step()
        torch.cuda.synchronize()
        ke = max(1, min(args.steps, 10))
        ems = max_over_ranks(time_region(e2e_step, ke, stream, world) / ke, world)
        h2d = sum(t.numel() * t.element_size() for k, t in h.items() if t is not None)
        d2h = hout.numel() * hout.element_size() + hSf.numel() * hSf.element_size()
        e2e = {"value": world * tokens / (ems / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems, "steps": ke,
               "host_link_gb_per_s": (h2d + d2h) / (ems / 1e3) / 1e9,
               "bound": "host link: every step moves its inputs in and its outputs out over PCIe"}

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only) ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        model, host_cores = cpu_info()
        tps, threads, desc, _, _ = oracle_forward_sample(w, args.cpu_seconds)
        cpu = {"value": tps, "unit": "tokens/s", "cores": threads, "host_cores": host_cores,
               "oracle_threads": threads, "kind": "oracle", "sample": desc + "; CPU: " + model}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": fwd_config(w_cfg, args.raw, world),
            "tflops": tflops, "gb_per_s": gbs,
            "roofline": roof, "kernels": kernels, "segments": nseg,
            "decode": dec, "decode_large_state": decs[1] if len(decs) > 1 else None, "e2e": e2e, "cpu_baseline": cpu, "clocks": clocks,
            "gpu_launches": args.steps * launches_per_fwd, "forward_launches_per_step": launches_per_fwd,
            "forward_scratch_bytes": scratch_bytes,
        }
        print(json.dumps(line), flush=True)
    return 0


def run_varlen(args, world, rank):
    """Packed prefill: args.varlen sequences with lengths drawn log-uniformly from [256, 8192]
    (seeded), H = 16, d = 128, bf16, one gdn_forward_varlen call per step, inputs in HBM.  With
    --varlen-long L the first sequence has L tokens instead (one long sequence among short ones,
    gates of the long-context workloads: x_alpha ~ N(-3, 1))."""
    import gated_delta_rule_142_b200 as gdn
    gdn.load()
    peaks, peak_kind = load_peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    lengths = length_mix(args.varlen, 256, 8192, seed=rank)
    alpha_mu = 0.0
    if args.varlen_long:
        lengths = [args.varlen_long] + lengths[1:]
        alpha_mu = -3.0
    H, d = 16, 128
    inp = varlen_inputs(lengths, H, d, d, "bf16", seed=1000 + rank, s0_std=0.02, alpha_mu=alpha_mu)
    dd = {n: inp[n].to(dev) for n in ("q", "k", "v", "log_alpha", "beta", "S0")}
    T = sum(lengths)
    out = torch.empty((T, H, d), dtype=torch.bfloat16, device=dev)
    Sf = torch.empty((len(lengths), H, d, d), dtype=torch.float32, device=dev)

    def step():
        gdn.forward_varlen(dd["q"], dd["k"], dd["v"], dd["log_alpha"], dd["beta"], inp["cu_seqlens"], dd["S0"],
                           chunk=64, out=out, S_final=Sf, stream=stream)

    sampler = ClockSampler(dev)
    sampler.start()
    for _ in range(args.warmup):
        step()
    gdn.timing_start()
    ms = time_region(step, args.steps, stream, world)
    ktimes = gdn.timing_stop()
    clocks = sampler.stop()
    ms_step = max_over_ranks(ms / args.steps, world)
    nth = T * H
    work = {"prep": (nth * 6 * 64 * d, nth * (2 * d * 2 + 8 + 2 * 64 + 2 * 64 + 2 * d + 8)),
            "chain": (nth * (6 * d * d + 4 * 64 * d), nth * (4 * d * 2 + 2 * 64 + 2 * 64 + 2 * d + 8))}
    kernels = {}
    for kind, (kms, n) in ktimes.items():
        per = kms / n
        flop, by = work.get(kind, (0, 0))
        kernels[kind] = {"launches_per_step": n / args.steps, "ms_per_launch": per, "share": kms / ms,
                         "tflops": flop / (per / 1e3) / 1e12, "gb_per_s": by / (per / 1e3) / 1e9}
    top = max(kernels, key=lambda k: ktimes[k][0]) if kernels else None
    roof = None
    if top in work:
        kt = kernels[top]
        tf, gb = kt["tflops"] / peaks["bf16_tflops"], kt["gb_per_s"] / peaks["hbm_gbs"]
        roof = ({"bound": "tensor", "achieved": kt["tflops"], "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                 "frac": tf} if tf >= gb else
                {"bound": "hbm", "achieved": kt["gb_per_s"], "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gb})
        roof.update({"kernel": top, "traffic": None, "peak_kind": peak_kind})
    if rank == 0:
        line = {"metric": "gated-delta packed prefill tokens/s", "value": world * T / (ms_step / 1e3),
                "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": {"workload": "varlen_bf16_n%d%s_h16_d128" % (
                               args.varlen, "_long%d" % args.varlen_long if args.varlen_long else ""),
                           "sequences": len(lengths), "alpha_mu": alpha_mu,
                           "tokens": T, "min_len": min(lengths), "max_len": max(lengths), "H": H, "dk": d, "dv": d,
                           "chunk": 64, "parallelism": "replicas" if world > 1 else "single"},
                "roofline": roof, "kernels": kernels, "clocks": clocks,
                "gpu_launches": sum(int(n) for _, n in ktimes.values())}
        print(json.dumps(line), flush=True)
    return 0


# float32 FMA peak of the CUDA cores, derived from unit counts and the clock: 148 SMs x 128 FP32
# lanes x 2 FLOP per FMA x 1.965 GHz (the backward runs on the CUDA cores in float32)
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def run_backward(args, world, rank):
    """gdn_backward over the chosen forward workload (inputs, grad_out and grad_S_final in HBM); one
    call per step.  Counted work: twice the forward's counted FLOP per token-head (the usual
    backward-to-forward ratio of the dense contractions).  The tensor-core reverse mode (two backward
    launches per call) is reported against the measured bf16 tensor peak, the CUDA-core one against
    the float32 CUDA-core peak."""
    import gated_delta_rule_142_b200 as gdn
    gdn.load()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    w = WORKLOADS[args.workload]
    if args.tokens:
        w = dataclasses.replace(w, T=args.tokens, name="%s_first%d" % (w.name, args.tokens))
    inp = forward_inputs(w.B, w.T, w.H, w.dk, w.dv, w.dtype, seed=w.seed + 1000 * rank, s0_std=w.s0_std,
                         alpha_mu=w.alpha_mu)
    d = {k: (None if v is None else v.to(dev)) for k, v in inp.items()}
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed + 77)
    g_out = torch.randn((w.B, w.T, w.H, w.dv), generator=g).to(d["q"].dtype).to(dev)
    g_Sf = torch.randn((w.B, w.H, w.dv, w.dk), generator=g).to(dev)

    def step():
        gdn.backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], g_out, g_Sf, chunk=w.chunk,
                     stream=stream)

    sampler = ClockSampler(dev)
    sampler.start()
    for _ in range(args.warmup):
        step()
    gdn.timing_start()
    ms = time_region(step, args.steps, stream, world)
    ktimes = gdn.timing_stop()
    clocks = sampler.stop()
    ms_step = max_over_ranks(ms / args.steps, world)
    flop = 2 * w.B * w.T * w.H * fwd_flop_per_token_head(w.dk, w.dv, w.chunk)
    tflops = flop / (ms_step / 1e3) / 1e12
    kernels = {kind: {"launches_per_step": n / args.steps, "ms_per_launch": kms / n, "share": kms / ms}
               for kind, (kms, n) in ktimes.items()}
    # the library's choice: bf16, d = 128, chunk 64 on the tensor cores unless the environment asks for
    # the CUDA-core reverse mode (whose bf16 form also launches two casts: three backward launches)
    tensor_cores = ("backward" in ktimes and ktimes["backward"][1] == 2 * args.steps and w.dtype == "bf16"
                    and os.environ.get("GDN_BWD_PATH") != "simt" and os.environ.get("GDN_BWD_RECOMPUTE") != "simt")
    if tensor_cores:
        peaks, peak_kind = load_peaks()
        roof = {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": tflops / peaks["bf16_tflops"], "traffic": None, "peak_kind": peak_kind + " bf16 burst",
                "flop_per_step": flop}
    else:
        roof = {"bound": "alu", "achieved": tflops, "peak": FP32_ALU_TFLOPS, "unit": "TFLOP/s",
                "frac": tflops / FP32_ALU_TFLOPS, "traffic": None,
                "peak_kind": "derived: 148 SMs x 128 FP32 lanes x 2 x 1.965 GHz", "flop_per_step": flop}
    if rank == 0:
        line = {"metric": "gated-delta backward tokens/s", "value": world * w.B * w.T / (ms_step / 1e3),
                "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16" if tensor_cores else "f32", "data": "synthetic",
                "path": "tensor cores (tcgen05)" if tensor_cores else "CUDA cores",
                "config": {"workload": w.name + "_backward", "B": w.B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv,
                           "chunk": w.chunk, "input_dtype": w.dtype,
                           "parallelism": "replicas" if world > 1 else "single"},
                "tflops": tflops,
                "roofline": roof,
                "kernels": kernels, "clocks": clocks,
                "gpu_launches": sum(int(n) for _, n in ktimes.values())}
        print(json.dumps(line), flush=True)
    return 0


def run_conv(args, world, rank):
    """gdn_causal_conv over one q/k/v-shaped tensor of the forward workload (B, T, H x d channels,
    bf16), width 4, state carried in place; HBM-bound: x read once, y written once."""
    import gated_delta_rule_142_b200 as gdn
    gdn.load()
    peaks, peak_kind = load_peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    w = WORKLOADS[args.workload]
    C, W = w.H * w.dk, 4
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed + 1000 * rank + 5)
    x = torch.randn((w.B, w.T, C), generator=g).to(torch.bfloat16).to(dev)
    wt = torch.randn((C, W), generator=g).to(dev)
    st = torch.zeros((w.B, W - 1, C), device=dev)
    y = torch.empty_like(x)

    def step():
        gdn.causal_conv(x, wt, st, out=y, state_out=st, stream=stream)

    sampler = ClockSampler(dev)
    sampler.start()
    for _ in range(args.warmup):
        step()
    gdn.timing_start()
    ms = time_region(step, args.steps, stream, world)
    ktimes = gdn.timing_stop()
    clocks = sampler.stop()
    ms_step = max_over_ranks(ms / args.steps, world)
    nbytes = 2 * w.B * w.T * C * 2 + C * W * 4 + 2 * w.B * (W - 1) * C * 4
    gbs = nbytes / (ms_step / 1e3) / 1e9
    if rank == 0:
        line = {"metric": "short causal convolution GB/s vs HBM", "value": world * w.B * w.T / (ms_step / 1e3),
                "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": {"workload": "conv_w4_" + w.name, "B": w.B, "T": w.T, "channels": C, "width": W,
                           "l2": "inputs larger than L2"},
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": gbs / peaks["hbm_gbs"], "traffic": None, "peak_kind": peak_kind,
                             "bytes_per_launch": nbytes},
                "kernels": {k: {"ms_per_launch": v[0] / v[1], "launches_per_step": v[1] / args.steps}
                            for k, v in ktimes.items()},
                "clocks": clocks, "gpu_launches": sum(int(n) for _, n in ktimes.values())}
        print(json.dumps(line), flush=True)
    return 0


def run_forward_conv(args, world, rank):
    """gdn_forward_conv on the forward workload: raw q, k, v and gate logits, the short convolution
    (width 4, carried state) of all three in one launch, then the raw forward, one call per step
    (bf16, inputs in HBM).  The same step composed of the public calls (three gdn_causal_conv
    passes, then gdn_forward_raw) is timed beside it."""
    import gated_delta_rule_142_b200 as gdn
    gdn.load()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    w = WORKLOADS[args.workload]
    if args.tokens:
        w = dataclasses.replace(w, T=args.tokens, name="%s_first%d" % (w.name, args.tokens))
    W = 4
    r = raw_inputs((w.B, w.T, w.H), w.dk, w.dv, w.dtype, seed=w.seed + 1000 * rank, s0_shape=(w.B, w.H, w.dv, w.dk),
                   s0_std=w.s0_std, alpha_mu=w.alpha_mu)
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed + 1000 * rank + 9)
    C = w.H * w.dk
    d = {n: (None if r[n] is None else r[n].to(dev)) for n in ("q", "k", "v", "x_alpha", "x_beta", "S0")}
    cw = (torch.randn((3, C, W), generator=g) * 0.5).to(dev)
    cs = torch.randn((3, w.B, W - 1, C), generator=g).to(dev)
    out = torch.empty((w.B, w.T, w.H, w.dv), dtype=d["q"].dtype, device=dev)
    Sf = torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device=dev)
    cso = torch.empty_like(cs)
    ys = [torch.empty_like(d[n]) for n in ("q", "k", "v")]

    def call():
        gdn.forward_conv(d["q"], d["k"], d["v"], d["x_alpha"], d["x_beta"], cw, cs, d["S0"], chunk=w.chunk, out=out,
                         S_final=Sf, conv_state_out=cso, stream=stream)

    def composed():
        for i, n in enumerate(("q", "k", "v")):
            gdn.causal_conv(d[n], cw[i], cs[i], out=ys[i], state_out=cso[i], stream=stream)
        gdn.forward_raw(ys[0], ys[1], ys[2], d["x_alpha"], d["x_beta"], d["S0"], chunk=w.chunk, out=out, S_final=Sf,
                        stream=stream)

    sampler = ClockSampler(dev)
    sampler.start()
    for _ in range(args.warmup):
        call()
        composed()
    gdn.timing_start()
    ms = time_region(call, args.steps, stream, world)
    ktimes = gdn.timing_stop()
    ms_c = time_region(composed, args.steps, stream, world)
    clocks = sampler.stop()
    ms_step = max_over_ranks(ms / args.steps, world)
    ms_comp = max_over_ranks(ms_c / args.steps, world)
    nbytes = fwd_bytes(w.B, w.T, w.H, w.dk, w.dv, 2 if w.dtype == "bf16" else 4, w.s0_std is not None, True)
    if rank == 0:
        line = {"metric": "gated-delta forward with the short convolution, tokens/s",
                "value": world * w.B * w.T / (ms_step / 1e3), "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
                "config": {"workload": "conv4_raw_" + w.name, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv,
                           "chunk": w.chunk, "conv_width": W, "l2": "inputs larger than L2"},
                "compulsory_gb_per_s": nbytes / (ms_step / 1e3) / 1e9,
                "composed_ms_per_step": ms_comp,
                "composed": "gdn_causal_conv on q, k, v (three passes), then gdn_forward_raw",
                "kernels": {k: {"ms_per_launch": v[0] / v[1], "launches_per_step": v[1] / args.steps}
                            for k, v in ktimes.items()},
                "clocks": clocks, "gpu_launches": sum(int(n) for _, n in ktimes.values())}
        print(json.dumps(line), flush=True)
    return 0


def run_grouped(args, world, rank):
    """gdn_forward_grouped on the ATMA head shape: 8 query heads reading 2 key-value memories,
    d = 128, over the forward workload's B and T (bf16, inputs in HBM)."""
    import gated_delta_rule_142_b200 as gdn
    gdn.load()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    w = WORKLOADS[args.workload]
    if args.tokens:
        w = dataclasses.replace(w, T=args.tokens, name="%s_first%d" % (w.name, args.tokens))
    Hq, Hkv = 8, 2
    a = forward_inputs(w.B, w.T, Hq, w.dk, w.dv, w.dtype, seed=w.seed + 1000 * rank, alpha_mu=w.alpha_mu)
    b = forward_inputs(w.B, w.T, Hkv, w.dk, w.dv, w.dtype, seed=w.seed + 1000 * rank + 1, s0_std=w.s0_std,
                       alpha_mu=w.alpha_mu)
    d = {"q": a["q"].to(dev), "k": b["k"].to(dev), "v": b["v"].to(dev), "la": b["log_alpha"].to(dev),
         "be": b["beta"].to(dev), "S0": None if b["S0"] is None else b["S0"].to(dev)}
    out = torch.empty((w.B, w.T, Hq, w.dv), dtype=d["q"].dtype, device=dev)
    Sf = torch.empty((w.B, Hkv, w.dv, w.dk), dtype=torch.float32, device=dev)

    def step():
        gdn.forward_grouped(d["q"], d["k"], d["v"], d["la"], d["be"], d["S0"], chunk=w.chunk, out=out, S_final=Sf,
                            stream=stream)

    sampler = ClockSampler(dev)
    sampler.start()
    for _ in range(args.warmup):
        step()
    gdn.timing_start()
    ms = time_region(step, args.steps, stream, world)
    ktimes = gdn.timing_stop()
    clocks = sampler.stop()
    ms_step = max_over_ranks(ms / args.steps, world)
    if rank == 0:
        line = {"metric": "gated-delta grouped-heads forward tokens/s", "value": world * w.B * w.T / (ms_step / 1e3),
                "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": w.dtype, "data": "synthetic",
                "config": {"workload": "grouped_q8_kv2_" + w.name, "B": w.B, "T": w.T, "Hq": Hq, "Hkv": Hkv,
                           "dk": w.dk, "dv": w.dv, "chunk": w.chunk,
                           "note": "each query head recomputes its group's memory"},
                "kernels": {k: {"ms_per_launch": v[0] / v[1], "launches_per_step": v[1] / args.steps}
                            for k, v in ktimes.items()},
                "clocks": clocks, "gpu_launches": sum(int(n) for _, n in ktimes.values())}
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["gdn", "reference"], default="gdn")
    ap.add_argument("--workload", default=None,
                    choices=[n for n, w in WORKLOADS.items() if w.kind == "forward"],
                    help="forward workload timed as the step (default: the 64K-token one)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="time only the first T tokens of the workload (profiler captures); not a bench line")
    ap.add_argument("--raw", action="store_true",
                    help="time gdn_forward_raw (input stage fused: raw q, k and gate logits) instead")
    ap.add_argument("--backward", action="store_true",
                    help="time gdn_backward on the workload (default workload then: the 2K training shape)")
    ap.add_argument("--conv", action="store_true", help="time gdn_causal_conv on a q-shaped tensor instead")
    ap.add_argument("--forward-conv", action="store_true",
                    help="time gdn_forward_conv (the short convolution of q, k, v, then the raw forward) instead")
    ap.add_argument("--grouped", action="store_true",
                    help="time gdn_forward_grouped with 8 query / 2 key-value heads instead")
    ap.add_argument("--varlen-long", type=int, default=0,
                    help="with --varlen: the first sequence has this many tokens")
    ap.add_argument("--varlen", type=int, default=0,
                    help="time packed prefill of this many sequences of mixed length instead of the forward step")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-only", default=None, choices=[n for n, w in WORKLOADS.items() if w.kind == "decode"],
                    help="time only this decode workload (profiler captures of the decode kernel); not a bench line")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-step-seconds", type=float, default=8.0)
    args = ap.parse_args()
    if args.workload is None:
        args.workload = "fwd_bf16_b8h16_t2k_d128" if args.backward else FWD_WORKLOAD
    if args.impl == "reference":
        # CPU oracle arm: rank 0 alone runs and prints; other ranks exit without work.
        return run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
    world, rank, local = dist_setup()
    try:
        if args.varlen:
            return run_varlen(args, world, rank)
        if args.backward:
            return run_backward(args, world, rank)
        if args.conv:
            return run_conv(args, world, rank)
        if args.grouped:
            return run_grouped(args, world, rank)
        if args.forward_conv:
            return run_forward_conv(args, world, rank)
        if args.decode_only:
            return run_decode_only(args, world, rank)
        return run_gdn(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
