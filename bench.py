"""Benchmark: bidirectional linear attention forward + backward on B200, one JSON line.

A step is one forward (la_bidir_fwd, which also stores the fp32 state) plus one
backward (la_bidir_bwd, consuming that state) over one batch of the workload,
inputs resident in HBM.  The default workload is B=8 H=16 T=4096 D=64, fp16
storage with fp32 accumulation, phi = elu+1, eps = 1e-6, Q,K,V ~ 0.5 N(0,1),
dO ~ N(0,1) (seed 0 + rank).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--T T] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own batch of the
same shape (independent heads, no collective on the data path: weak scaling);
the timed region is bracketed by barriers and the reported time is the max
over ranks.  ``--impl reference`` times the fp64 CPU oracle on the host cores
instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import glob
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "linear-attn fwd+bwd tokens/s and % of HBM roofline, B8 H16 D64 T=4K-16K"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0

# The pages' own A800 Triton timings for B8-H16-D64 (ms): T -> (fwd, bwd).  Context only.
PAGE_TIMINGS_MS = {128: (0.049152, 0.651264), 256: (0.056320, 0.625664), 512: (0.058368, 0.630784),
                   1024: (0.090112, 0.719872), 2048: (0.151552, 0.702464), 4096: (0.276480, 1.324032),
                   8192: (0.521216, 2.556928), 16384: (0.980992, 5.022208)}

# Algorithmic HBM bytes of each kernel per launch, in units of one [B,H,T,D] tensor of the
# storage dtype: the tensors it must read or write (state and partials are not counted).
KERNEL_TENSORS = {
    "simt_state_partial": 2, "simt_output": 2, "simt_bwd_q": 3, "simt_bwd_k": 4,
    "tc_state_reduce": 2, "tc_output": 2, "tc_bwd_q": 3, "tc_bwd_kv": 4,
    "tc_state_reduce_simple": 2, "tc_output_simple": 2, "tc_bwd_q_simple": 3, "tc_bwd_kv_simple": 4,
    "simt_ret_fwd": 4, "simt_ret_bwd_dq": 4, "simt_ret_bwd_dkdv": 6,
    # retention backward: the op's minimum (q, k, v, dO in; dq, dk, dv out), not the 12 tensors the
    # three-pass kernel actually moves, so its fraction shows the cost of that design
    "tc_retention_fwd": 4, "tc_retention_bwd": 7,
    # causal linear attention with the norm term on the tensor cores (fp16, D = 64): f(q), f(k)
    # formed (q, k in, both out); the forward (f(q), f(k), v in, o out); the backward's first
    # pass (those and dout in, du out); the dn terms (f(q), f(k), dq and dk in fp32 = two
    # 16-bit tensors each, in; dq, dk out)
    "tc_causal_norm_phi": 4, "tc_causal_norm_fwd": 4, "tc_causal_norm_prep": 5,
    "tc_causal_norm_dn_parts": 2, "tc_causal_norm_dn_apply": 8,
}

# CUDA-core work of the recurrent kernels per token-head, in flops (2 per multiply-add, 1 per
# other product), counting the state once (the arithmetic the recurrence needs, not a layout's):
# causal-norm forward: the D + 1 columns of [S | z] updated and read out, D FMAs each; dq sweep:
# those plus the D row sums of S.dO; reverse sweep: R and r updated, the row sums (dk) and the
# column sums (dv).  Gated: a state entry's update a_i S_ij + k_i v_j is 3 flops, a read-out 2.
CAUSAL_FLOPS = {
    "simt_causal_norm_fwd": lambda D: 4 * D * (D + 1),
    "simt_causal_norm_bwd_q": lambda D: 4 * D * (D + 1) + 2 * D * D,
    "simt_causal_norm_bwd_kv": lambda D: 6 * D * D + 2 * D,
    "simt_gated_fwd": lambda D: 5 * D * D,
    "simt_gated_bwd_q": lambda D: 5 * D * D,
    "simt_gated_bwd_kv": lambda D: 7 * D * D + 4 * D,
}


def fp32_fma_peak_tflops(sm_mhz):
    """FP32 FMA peak of the CUDA cores: 148 SMs x 128 lanes x 2 flops per clock."""
    return 148 * 128 * 2 * (sm_mhz or 1965.0) * 1e6 / 1e12


# ------------------------------------------------------------------ ranks --

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def init_dist(world, local_rank, backend="nccl", timeout_s=120):
    import datetime
    import torch.distributed as dist
    if world <= 1:
        return None
    if backend == "nccl":
        torch.cuda.set_device(local_rank)
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def max_over_ranks(value: float, dist, device=None) -> float:
    """Largest value over all ranks (the device timing rule for multi-GPU numbers)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def auto_steps(step, stream, dev, dist, target_s: float = 1.5, least: int = 200, most: int = 200000) -> int:
    """Number of timed steps for a timed region of about target_s seconds (at least `least`), so
    that the clock sampler sees the GPU under load; every rank takes the same count."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 10
    e0.record(stream)
    for i in range(n):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    per = max_over_ranks(e0.elapsed_time(e1) / n / 1e3, dist, dev)
    return int(min(most, max(least, math.ceil(target_s / max(per, 1e-7)))))


def aggregate_throughput(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job throughput: units processed by all ranks / the slowest rank's time."""
    return units_per_rank * world / seconds


# ---------------------------------------------------------------- helpers --

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# The files the tensor-core kernels are compiled from (their launch code included): a change
# anywhere else in the library leaves those kernels, and their DRAM traffic, as they were.
# The files each family of tensor-core kernels is compiled from (with include/la.h): a
# committed ncu capture stands for a kernel only while its family's files are unchanged.
TC_SOURCES = {
    "state": ("la_tc.cuh", "la_tc_state.cu", "la_tc_common.cuh", "la_tc_ptx.cuh", "la_internal.cuh"),
    "retention": ("la_tc.cuh", "la_tc_retention.cu", "la_tc_common.cuh", "la_tc_ptx.cuh", "la_internal.cuh"),
    "causal": ("la_tc.cuh", "la_tc_retention.cu", "la_tc_causal.cu", "la_tc_common.cuh", "la_tc_ptx.cuh",
               "la_internal.cuh"),
}


def kernel_sources(kernel: str):
    """The source files of the tensor-core kernel launched under `kernel`."""
    if kernel.startswith("tc_retention"):
        return TC_SOURCES["retention"]
    return TC_SOURCES["causal" if kernel.startswith("tc_causal_norm") else "state"]


def strip_comments(src: str) -> str:
    """C/C++ source without its comments (// to the end of the line, /* ... */), string and
    character literals kept, so that a change to comments alone leaves the hash alone."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return "".join(out)


def source_hash(names=None) -> str:
    """sha256 prefix of the library's kernel sources (every csrc file, or those in `names`) and
    of include/la.h, comments left out."""
    csrc = os.path.join(ROOT, "linear_attention_attn_b200", "csrc")
    paths = sorted(glob.glob(os.path.join(csrc, "*"))) if names is None else \
        sorted(os.path.join(csrc, n) for n in names)
    h = hashlib.sha256()
    for p in paths + [os.path.join(ROOT, "include", "la.h")]:
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode())
            h.update(strip_comments(f.read().decode("utf-8")).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, T: int, B: int, H: int, D: int, dtype: str):
    """DRAM bytes per launch of `kernel` at [B, H, T, D] in `dtype` from the committed ncu
    summaries: of the captures taken on the current kernel sources at the same B, H, D and dtype,
    the one whose T is nearest, scaled by T (None when no capture matches)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    entries = rec.get(kernel) or []
    if isinstance(entries, dict):
        entries = [entries]
    sha = source_hash(kernel_sources(kernel))
    ok = [e for e in entries if e.get("source_sha") == sha and
          (e.get("B"), e.get("H"), e.get("D"), e.get("dtype")) == (B, H, D, dtype)]
    if not ok:
        return None
    e = min(ok, key=lambda e: abs(math.log(float(e["T"]) / T)))
    return float(e["dram_bytes_per_launch"]) * (T / float(e["T"]))


def gpu_selector(dev) -> str:
    """nvidia-smi -i argument naming this CUDA device (its UUID; the CUDA ordinal may differ from
    nvidia-smi's index when CUDA_VISIBLE_DEVICES is set)."""
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev.index or 0)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: str):
        self.gpu = gpu
        self.proc = None
        self.path = os.path.join("/tmp", "la_clocks_%d.csv" % os.getpid())

    def start(self):
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu, "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        # the timed region starts only once nvidia-smi is writing samples (bounded wait)
        t0 = time.time()
        while time.time() - t0 < 5.0 and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.01)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, flag in zip(names, parts[5:9]):
                if flag.lower() == "active":
                    reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# --------------------------------------------------------------- oracle arm --

def _oracle_step(w, q, k, v, g, gamma, nthreads):
    """One fp64 oracle fwd+bwd of the workload's op on [1, n, Ts, D] heads."""
    import oracle
    if w.op == "bidir":
        oracle.bidir_fwd(q, k, v, eps=w.eps, nthreads=nthreads)
        oracle.bidir_bwd(q, k, v, g, eps=w.eps, nthreads=nthreads)
    elif w.op == "simple":
        oracle.simple_fwd(q, k, v, nthreads=nthreads)
        oracle.simple_bwd(q, k, v, g, nthreads=nthreads)
    elif w.op == "causal_norm":
        oracle.causal_norm_fwd(q, k, v, None, "elu1", w.eps, nthreads=nthreads)
        oracle.causal_norm_bwd(q, k, v, g, None, "elu1", w.eps, nthreads=nthreads)
    elif w.op == "gated":
        oracle.gated_fwd(q, k, v, gamma, nthreads=nthreads)       # gamma carries the log gates here
        oracle.gated_bwd(q, k, v, gamma, g, nthreads=nthreads)
    else:
        oracle.retention_fwd(q, k, v, gamma, nthreads=nthreads)
        oracle.retention_bwd(q, k, v, g, gamma, nthreads=nthreads)


def oracle_step_sample(w, inp, budget_s: float, threads: int):
    """Time the fp64 oracle on a bounded sample of the workload: n (b,h) heads at a prefix of
    T tokens, sized to take about budget_s.  Returns (tokens/s, seconds, sample text, threads used)."""
    BH = w.B * w.H
    q = inp["q"].reshape(BH, w.T, w.D)
    k = inp["k"].reshape(BH, w.T, w.D)
    v = inp["v"].reshape(BH, w.T, w.D)
    g = inp["do"].reshape(BH, w.T, w.D)
    gam = inp.get("gamma")
    lgate = inp["g"].reshape(BH, w.T, w.D) if "g" in inp else None

    def heads(n, Ts):
        x = [t[:n, :Ts].reshape(1, n, Ts, w.D) for t in (q, k, v, g)]
        if lgate is not None:          # gated: the log gates of the same heads and tokens
            return x + [lgate[:n, :Ts].reshape(1, n, Ts, w.D)]
        gm = None if gam is None else gam.reshape(-1)[[i % w.H for i in range(n)]]
        return x + [gm]

    # calibrate the per-token cost on one head, single thread (untimed)
    tc = min(w.T, 512)
    t0 = time.perf_counter()
    _oracle_step(w, *heads(1, tc), nthreads=1)
    per_token = (time.perf_counter() - t0) / tc
    budget_tokens = max(1.0, budget_s / per_token) * threads
    n = int(max(1, min(BH, budget_tokens // w.T)))
    Ts = w.T if n > 1 or budget_tokens >= w.T else int(max(64, min(w.T, budget_tokens)))
    used = min(threads, n)
    args = heads(n, Ts)
    t0 = time.perf_counter()
    _oracle_step(w, *args, nthreads=used)
    dt = time.perf_counter() - t0
    tokens = n * Ts / float(w.H)          # token = one position of one batch row, all H heads
    sample = "%d of %d (b,h) heads x %d of %d tokens, fp64 fwd+bwd, %d threads" % (n, BH, Ts, w.T, used)
    return tokens / dt, dt, sample, used


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def metric_of(w) -> str:
    """The line's metric: the specification's for the bidirectional workload, else the op's own
    fwd+bwd tokens/s (the same on both arms)."""
    return METRIC if w.op == "bidir" else "%s fwd+bwd tokens/s" % ("causal" if w.name == "causal_bf16" else w.op)


def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    inp = synth.make_inputs(w, seed=0)
    cores = host_cores()
    budget = max(0.02, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_step_sample(w, inp, budget, cores)
    rates, secs, sample, used = [], 0.0, "", cores
    for _ in range(args.steps):
        r, dt, sample, used = oracle_step_sample(w, inp, budget, cores)
        rates.append(r)
        secs += dt
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": metric_of(w), "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------- ours --

WORKLOAD_TEXT = {
    "bidir": "bidirectional linear attention fwd+bwd, fp16 storage / fp32 accumulate, B=%d H=%d T=%d D=%d, "
             "phi=elu+1, eps=1e-06, Q,K,V ~ 0.5 N(0,1), dO ~ N(0,1)",
    "simple": "simple_la fwd+bwd, bf16 storage / fp32 accumulate, B=%d H=%d T=%d D=%d, "
              "q,k ~ N(0,1) D^-1/2, v, dO ~ N(0,1)",
    "retention": "chunked causal decay (retention) fwd+bwd, bf16 storage / fp32 accumulate, B=%d H=%d T=%d D=%d, "
                 "gamma_h = 1 - 2^(-5-7h/(H-1)), q ~ N(0,1) D^-1/2, k, v, dO ~ N(0,1)",
    "bidir_d128": "bidirectional linear attention fwd+bwd on the CUDA-core kernels (no tensor-core kernel at D=128), "
                  "fp16 storage / fp32 accumulate, B=%d H=%d T=%d D=%d, phi=elu+1, eps=1e-06, Q,K,V ~ 0.5 N(0,1), "
                  "dO ~ N(0,1)",
    "simple_d128": "simple_la fwd+bwd on the CUDA-core kernels (no tensor-core kernel at D=128), bf16 storage / fp32 "
                   "accumulate, B=%d H=%d T=%d D=%d, q,k ~ N(0,1) D^-1/2, v, dO ~ N(0,1)",
    "causal": "plain causal linear attention fwd+bwd (the decay op with gamma = 1 on every head: no feature map, "
              "no norm term), bf16 storage / fp32 accumulate, B=%d H=%d T=%d D=%d, q ~ N(0,1) D^-1/2, k, v, dO ~ N(0,1)",
    "gated": "gated linear attention fwd+bwd (recurrent form in 256-token chunks on CUDA cores), bf16 storage / "
             "fp32 accumulate, "
             "B=%d H=%d T=%d D=%d, log gates log(sigmoid(N(0,1)))/16 per token and key dimension, "
             "q ~ N(0,1) D^-1/2, k, v, dO ~ N(0,1)",
    "vision": "long-sequence vision-style bidirectional linear attention fwd only, fp16 storage / fp32 accumulate, "
              "B=%d H=%d T=%d D=%d (256x256 token grid), phi=elu+1, eps=1e-06, Q,K,V ~ 0.5 N(0,1) plus a smooth 2-D "
              "sinusoidal offset of amplitude 0.1",
    "causal_norm": "causal linear attention with the norm term fwd+bwd (fp16 at D=64: the chunked decay kernel "
                   "on tensor cores with a column of ones carrying the normaliser), fp16 storage / "
                   "fp32 accumulate, B=%d H=%d T=%d D=%d, phi=elu+1, no decay, eps=1e-06, Q,K,V ~ 0.5 N(0,1), "
                   "dO ~ N(0,1)",
}


def config_of(w, args):
    step_bytes = 11 * w.B * w.H * w.T * w.D * 2
    kind = "causal" if w.name == "causal_bf16" else w.op
    return {"workload": WORKLOAD_TEXT[kind] % (w.B, w.H, w.T, w.D),
            "B": w.B, "H": w.H, "T": w.T, "D": w.D, "global_batch": w.B * max(1, args.gpus), "seq_len": w.T,
            "parallelism": "dp%d (independent batches, no collective)" % max(1, args.gpus),
            "l2": "inputs larger than L2: %.0f MB of algorithmic traffic per step vs 126 MB L2, no flush"
                  % (step_bytes / 1e6)}


def time_step_at(la, w, dev, stream, steps, warmup):
    """Device time (ms) of one fwd+bwd step of workload w, averaged over `steps`."""
    host = synth.make_inputs(w, seed=0)
    q, k, v, g = (host[n].to(dev) for n in ("q", "k", "v", "do"))
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    state = torch.empty((w.B, w.H, w.D, w.D + 1), dtype=torch.float32, device=dev)
    nws = max(la.la_workspace_size("bidir_fwd", w.B, w.H, w.T, w.D, q.dtype),
              la.la_workspace_size("bidir_bwd", w.B, w.H, w.T, w.D, q.dtype))
    ws = torch.empty(max(256, nws), dtype=torch.uint8, device=dev)

    def step():
        la.la_bidir_fwd(q, k, v, o, state, eps=w.eps, workspace=ws)
        la.la_bidir_bwd(q, k, v, g, dq, dk, dv, state, eps=w.eps, workspace=ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1) / steps


class L2Flush:
    """Writes a buffer twice the size of L2 (between timed steps whose data fits in L2)."""

    def __init__(self, dev):
        self.buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def __call__(self):
        self.buf.fill_(1.0)


def time_each(fn, steps, warmup, stream, flush=None):
    """Mean device time (ms) of fn() over `steps` calls, each bracketed by its own events on
    `stream`; with `flush`, L2 is overwritten before every call, outside the events."""
    for _ in range(warmup):
        fn()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        if flush is not None:
            flush()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / steps


# Sub-records of the default line: every workload of the specification besides the headline,
# at the sizes it names (simple_la and retention T sweeps, the vision forward), plus the causal
# norm and gated ops at the headline shape.  (workload, T values, forward only)
CONFIG_RECORDS = (("simple_bf16", (128, 1024, 4096, 16384), False),
                  ("retention_bf16", (2048, 8192), False),
                  ("causal_bf16", (4096,), False),
                  ("vision_f16", (65536,), True),
                  ("causal_norm_f16", (4096,), False),
                  ("gated_bf16", (4096,), False),
                  ("bidir_f16_d128", (4096,), False),
                  ("simple_bf16_d128", (4096,), False))


def config_records(la, dev, stream):
    """Device-timed fwd+bwd (or fwd) of the other workloads: ms per step, tokens/s, GB/s at the
    algorithmic bytes (4 tensors forward, 7 backward, of [B,H,T,D] in the storage dtype) and the
    fraction of the measured copy bandwidth.  Each call timed on its own, L2 flushed in between
    when a step's data fits in L2."""
    peak, peak_kind = measured_peaks()
    flush = L2Flush(dev)
    out = {}
    for base, Ts, fwd_only in CONFIG_RECORDS:
        recs = []
        for T in Ts:
            w = synth.WORKLOADS[base].with_T(T)
            host = synth.make_inputs(w, seed=0, with_grad=not fwd_only)
            q, k, v = (host[n].to(dev) for n in ("q", "k", "v"))
            g = host["do"].to(dev) if not fwd_only else None
            o = torch.empty_like(q)
            dq, dk, dv = ((torch.empty_like(q) for _ in range(3)) if not fwd_only else (None, None, None))
            B, H, D = w.B, w.H, w.D
            st = torch.empty((B, H, D, D + 1), dtype=torch.float32, device=dev)
            ops = {"bidir": ("bidir_fwd", "bidir_bwd"), "simple": ("simple_fwd", "simple_bwd"),
                   "retention": ("chunk_decay_fwd", "chunk_decay_bwd"),
                   "causal_norm": ("causal_norm_fwd", "causal_norm_bwd"), "gated": ("gated_fwd", "gated_bwd")}[w.op]
            nws = max(la.la_workspace_size(n, B, H, T, D, q.dtype) for n in ops)
            ws = torch.empty(max(256, nws), dtype=torch.uint8, device=dev)
            lg = host["g"].to(dev) if w.op == "gated" else None
            dg = torch.empty_like(q) if w.op == "gated" else None
            gam = host.get("gamma")

            def fwd():
                if w.op == "bidir":
                    la.la_bidir_fwd(q, k, v, o, st, eps=w.eps, workspace=ws)
                elif w.op == "simple":
                    la.la_simple_fwd(q, k, v, o, st, workspace=ws)
                elif w.op == "retention":
                    la.la_chunk_decay_fwd(q, k, v, o, gam, workspace=ws)
                elif w.op == "causal_norm":
                    la.la_causal_norm_fwd(q, k, v, o, None, "elu1", w.eps, workspace=ws)
                else:
                    la.la_gated_fwd(q, k, v, lg, o, workspace=ws)

            def bwd():
                if w.op == "bidir":
                    la.la_bidir_bwd(q, k, v, g, dq, dk, dv, st, eps=w.eps, workspace=ws)
                elif w.op == "simple":
                    la.la_simple_bwd(q, k, v, g, dq, dk, dv, st, workspace=ws)
                elif w.op == "retention":
                    la.la_chunk_decay_bwd(q, k, v, g, gam, dq, dk, dv, workspace=ws)
                elif w.op == "causal_norm":
                    la.la_causal_norm_bwd(q, k, v, g, dq, dk, dv, None, "elu1", w.eps, workspace=ws)
                else:
                    la.la_gated_bwd(q, k, v, lg, g, dq, dk, dv, dg, workspace=ws)

            tb = B * H * T * D * q.element_size()
            step_bytes = (4 if fwd_only else 11) * tb
            fl = flush if step_bytes < 2 * L2_BYTES else None
            n = 100 if step_bytes < 64e6 else 20
            ms_f = time_each(fwd, n, 3, stream, fl)
            rec = {"T": T, "B": B, "H": H, "D": D, "dtype": w.dtype, "fwd_ms": ms_f,
                   "fwd_frac": 4 * tb / (ms_f / 1e3) / 1e9 / peak}
            ms = ms_f
            if not fwd_only:
                ms_b = time_each(bwd, n, 3, stream, fl)
                ms_s = time_each(lambda: (fwd(), bwd()), n, 3, stream, fl)
                rec.update(bwd_ms=ms_b, bwd_frac=7 * tb / (ms_b / 1e3) / 1e9 / peak)
                ms = ms_s
            rec.update(ms_per_step=ms, tokens_per_s=B * T / (ms / 1e3),
                       achieved_gbs=step_bytes / (ms / 1e3) / 1e9, frac=step_bytes / (ms / 1e3) / 1e9 / peak,
                       l2_flushed=fl is not None)
            recs.append(rec)
            del q, k, v, g, o, dq, dk, dv, st, ws, lg, dg
            torch.cuda.empty_cache()
        kind = {"vision_f16": "vision", "causal_bf16": "causal", "bidir_f16_d128": "bidir_d128",
                "simple_bf16_d128": "simple_d128"}.get(base, synth.WORKLOADS[base].op)
        out[base] = {"workload": WORKLOAD_TEXT[kind]
                     % (synth.WORKLOADS[base].B, synth.WORKLOADS[base].H, Ts[-1], synth.WORKLOADS[base].D),
                     "step": "fwd" if fwd_only else "fwd+bwd", "peak_gbs": peak, "peak_source": peak_kind,
                     "records": recs}
    return out


def run_ours(args, w):
    import linear_attention_attn_b200 as la
    rank, world, local = dist_env()
    dist = init_dist(world, local)
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    seqpar = getattr(args, "seqpar", False)
    if seqpar:
        # the workload's T is the whole sequence; this rank holds a shard of T / world tokens
        from linear_attention_attn_b200 import seqpar as sp
        if w.op in ("retention", "causal_norm", "gated") or w.T % world:
            raise SystemExit("--seqpar needs the bidir or simple workload and T divisible by the GPU count")
        host = synth.make_inputs(w.with_T(w.T // world), seed=rank)
    else:
        host = synth.make_inputs(w, seed=rank)
    q, k, v, g = (host[n].to(dev) for n in ("q", "k", "v", "do"))
    B, H, D = w.B, w.H, w.D
    T = q.shape[2]
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    state = torch.empty((B, H, D, D + 1), dtype=torch.float32, device=dev)
    dstate = torch.empty_like(state)
    names = {"bidir": ("bidir_fwd", "bidir_bwd"), "simple": ("simple_fwd", "simple_bwd"),
             "retention": ("chunk_decay_fwd", "chunk_decay_bwd"),
             "causal_norm": ("causal_norm_fwd", "causal_norm_bwd"), "gated": ("gated_fwd", "gated_bwd")}[w.op]
    if seqpar:
        names = ("state_reduce", "state_bwd_q")
    ws_bytes = max(la.la_workspace_size(n, B, H, T, D, q.dtype) for n in names)
    ws = torch.empty(max(256, ws_bytes), dtype=torch.uint8, device=dev)
    gamma = host.get("gamma")
    gated = w.op == "gated"
    lgate = host["g"].to(dev) if gated else None     # the log gates
    dgate = torch.empty_like(q) if gated else None
    feature = "elu1" if w.op == "bidir" else "identity"

    def step():
        if seqpar:
            sp.forward(q, k, v, o, state, feature=feature, eps=w.eps, workspace=ws)
            sp.backward(q, k, v, g, state, dq, dk, dv, dstate, feature=feature, eps=w.eps, workspace=ws)
        elif w.op == "bidir":
            la.la_bidir_fwd(q, k, v, o, state, eps=w.eps, workspace=ws)
            la.la_bidir_bwd(q, k, v, g, dq, dk, dv, state, eps=w.eps, workspace=ws)
        elif w.op == "simple":
            la.la_simple_fwd(q, k, v, o, state, workspace=ws)
            la.la_simple_bwd(q, k, v, g, dq, dk, dv, state, workspace=ws)
        elif w.op == "causal_norm":
            la.la_causal_norm_fwd(q, k, v, o, None, "elu1", w.eps, workspace=ws)
            la.la_causal_norm_bwd(q, k, v, g, dq, dk, dv, None, "elu1", w.eps, workspace=ws)
        elif gated:
            la.la_gated_fwd(q, k, v, lgate, o, workspace=ws)
            la.la_gated_bwd(q, k, v, lgate, g, dq, dk, dv, dgate, workspace=ws)
        else:
            la.la_chunk_decay_fwd(q, k, v, o, gamma, workspace=ws)
            la.la_chunk_decay_bwd(q, k, v, g, gamma, dq, dk, dv, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if args.steps is None:
        args.steps = 200 if args.profile_only else auto_steps(lambda i: step(), stream, dev, dist)
    if args.profile_only:
        for _ in range(args.steps):
            step()
        torch.cuda.synchronize(dev)
        la.la_device_check()
        return 0

    # ---- timed region: K steps, device events, barriers on both sides
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(gpu_selector(dev))
    sampler.start()
    launches0 = la.la_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    launches = la.la_launch_count() - launches0
    if dist is not None:
        dist.barrier()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1)
    ms = max_over_ranks(ms, dist, dev)
    seconds = ms / 1e3
    tokens_per_rank = B * T * args.steps
    value = aggregate_throughput(tokens_per_rank, world, seconds)

    # ---- per-kernel device times: the same steps again with two events around every
    #      launch (events between kernels keep them from overlapping, so this pass is
    #      separate from the timed one)
    #      The stream is first held by a spin of ~20 ms (torch's), so that the host has enqueued
    #      every launch of the pass before the GPU starts on them: the kernels then run back to
    #      back and the first kernel of each call is not charged with the host's launch gap.
    k_prof = max(3, min(args.steps, 50))
    la.la_prof_enable(True)
    la.la_prof_collect()              # drop anything recorded before
    torch.cuda.synchronize(dev)
    torch.cuda._sleep(int(4e7))
    for _ in range(k_prof):
        step()
    torch.cuda.synchronize(dev)
    la.la_prof_enable(False)
    per_kernel = la.la_prof_collect()

    # ---- end to end through the C ABI with host buffers (pinned), copies inside the timed region:
    #      every step copies its inputs in and its outputs out; the copies of neighbouring steps
    #      overlap the compute (three streams, two device buffer sets), as a serving loop would run
    e2e = None
    in_names = ["q", "k", "v", "do"] + (["g"] if gated else [])
    hins = [host[n].pin_memory() for n in in_names]
    n_out = 5 if gated else 4                    # o, dq, dk, dv (and the log gates' gradient)
    hout = [[torch.empty_like(hins[0]).pin_memory() for _ in range(n_out)] for _ in range(2)]
    sets = []
    for si in range(2):
        if si == 0:
            ins = [q, k, v, g] + ([lgate] if gated else [])
            outs = [o, dq, dk, dv] + ([dgate] if gated else [])
        else:
            ins = [torch.empty_like(q) for _ in in_names]
            outs = [torch.empty_like(q) for _ in range(n_out)]
        sets.append((ins, outs, torch.empty_like(state)))
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        si = i % 2
        ins, outs, xst = sets[si]
        xq, xk, xv, xg = ins[:4]
        xo, xdq, xdk, xdv = outs[:4]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_cmp[si])           # step i-2 is done with this input set
            for d_, h_ in zip(ins, hins):
                d_.copy_(h_, non_blocking=True)
            ev_in[si].record(s_in)
        s_cmp.wait_event(ev_in[si])
        if i >= 2:
            s_cmp.wait_event(ev_out[si])              # step i-2's outputs have left this set
        if w.op == "bidir":
            la.la_bidir_fwd(xq, xk, xv, xo, xst, eps=w.eps, workspace=ws, stream=s_cmp)
            la.la_bidir_bwd(xq, xk, xv, xg, xdq, xdk, xdv, xst, eps=w.eps, workspace=ws, stream=s_cmp)
        elif w.op == "simple":
            la.la_simple_fwd(xq, xk, xv, xo, xst, workspace=ws, stream=s_cmp)
            la.la_simple_bwd(xq, xk, xv, xg, xdq, xdk, xdv, xst, workspace=ws, stream=s_cmp)
        elif w.op == "causal_norm":
            la.la_causal_norm_fwd(xq, xk, xv, xo, None, "elu1", w.eps, workspace=ws, stream=s_cmp)
            la.la_causal_norm_bwd(xq, xk, xv, xg, xdq, xdk, xdv, None, "elu1", w.eps, workspace=ws, stream=s_cmp)
        elif gated:
            la.la_gated_fwd(xq, xk, xv, ins[4], xo, workspace=ws, stream=s_cmp)
            la.la_gated_bwd(xq, xk, xv, ins[4], xg, xdq, xdk, xdv, outs[4], workspace=ws, stream=s_cmp)
        else:
            la.la_chunk_decay_fwd(xq, xk, xv, xo, gamma, workspace=ws, stream=s_cmp)
            la.la_chunk_decay_bwd(xq, xk, xv, xg, gamma, xdq, xdk, xdv, workspace=ws, stream=s_cmp)
        ev_cmp[si].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[si])
            for h_, d_ in zip(hout[si], outs):
                h_.copy_(d_, non_blocking=True)
            ev_out[si].record(s_out)

    e2e_ok = not seqpar
    if e2e_ok:
        k_e2e = max(3, min(args.steps, 20))
        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        x0.record(s_in)
        s_cmp.wait_event(x0)
        s_out.wait_event(x0)
        for i in range(k_e2e):
            e2e_step(i)
        s_out.wait_stream(s_in)
        s_out.wait_stream(s_cmp)
        x1.record(s_out)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(x0.elapsed_time(x1), dist, dev)
        tensor_bytes = B * H * T * D * q.element_size()
        e2e = {"value": aggregate_throughput(B * T * k_e2e, world, e2e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": len(in_names) * tensor_bytes, "d2h_bytes_per_step": n_out * tensor_bytes,
               "steps": k_e2e, "note": "pinned host q, k, v, dO copied in and o, dq, dk, dv copied out every step "
                                       "through the C ABI; copies of neighbouring steps overlap the compute "
                                       "(three streams, two device buffer sets)"}
    tensor_bytes = B * H * T * D * q.element_size()

    # ---- roofline of the dominant kernel (rank 0's per-kernel events)
    roof = None
    if per_kernel:
        name, n_launch, tot_ms = max(per_kernel, key=lambda r: r[2])
        peak, peak_kind = measured_peaks()
        if name in KERNEL_TENSORS and n_launch > 0:
            alg_bytes = KERNEL_TENSORS[name] * tensor_bytes
            avg_s = tot_ms / n_launch / 1e3
            achieved = alg_bytes / avg_s / 1e9
            traffic = ncu_traffic(name, T, B, H, D, w.dtype)
            roof = {"bound": "hbm", "kernel": name, "achieved": achieved, "peak": peak, "unit": "GB/s",
                    "frac": achieved / peak, "peak_source": peak_kind, "traffic": traffic,
                    "algorithmic_bytes_per_launch": alg_bytes, "avg_launch_ms": tot_ms / n_launch,
                    "share_of_step": tot_ms / max(1e-9, sum(r[2] for r in per_kernel))}
        elif name in CAUSAL_FLOPS and n_launch > 0:
            flops = CAUSAL_FLOPS[name](D) * B * H * T
            avg_s = tot_ms / n_launch / 1e3
            fpeak = fp32_fma_peak_tflops((clocks or {}).get("sm_mhz"))
            roof = {"bound": "alu", "kernel": name, "achieved": flops / avg_s / 1e12, "peak": fpeak,
                    "unit": "TFLOP/s", "frac": flops / avg_s / 1e12 / fpeak,
                    "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 flops x the sampled SM clock",
                    "traffic": None, "algorithmic_flops_per_launch": flops, "avg_launch_ms": tot_ms / n_launch,
                    "share_of_step": tot_ms / max(1e-9, sum(r[2] for r in per_kernel))}
    step_bytes = 11 * tensor_bytes
    peak, peak_kind = measured_peaks()
    step_roof = {"bytes_per_step": step_bytes, "achieved_gbs": step_bytes / (seconds / args.steps) / 1e9,
                 "frac": step_bytes / (seconds / args.steps) / 1e9 / peak, "peak": peak, "peak_source": peak_kind}

    # ---- the same step at the longer sequence lengths of the metric (device events only)
    sweep = []
    if world == 1 and args.sweep and w.op == "bidir" and not seqpar:
        del o, dq, dk, dv, q, k, v, g, ws
        torch.cuda.empty_cache()
        for Ts in (8192, 16384):
            if Ts == T:
                continue
            ms_s = time_step_at(la, w.with_T(Ts), dev, stream, steps=max(3, min(args.steps, 50)), warmup=3)
            b_s = 11 * w.B * w.H * Ts * w.D * 2
            sweep.append({"T": Ts, "value": w.B * Ts / (ms_s / 1e3), "ms_per_step": ms_s,
                          "achieved_gbs": b_s / (ms_s / 1e3) / 1e9,
                          "frac": b_s / (ms_s / 1e3) / 1e9 / measured_peaks()[0]})

    # ---- the other workloads of the specification, device-timed (rank 0's GPU, N = 1 only)
    configs = None
    if world == 1 and args.sweep and w.op == "bidir" and not seqpar:   # the headline's tensors went with the sweep
        torch.cuda.empty_cache()
        configs = config_records(la, dev, stream)

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return 0

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cores = host_cores()
        r, dt, sample, used = oracle_step_sample(w, host, 15.0, cores)
        cpu = {"value": r, "unit": UNIT, "cores": used, "kind": "oracle", "sample": sample, "seconds": dt}

    vs = None
    if w.op == "bidir" and not seqpar and T in PAGE_TIMINGS_MS and (B, H, D) == (8, 16, 64):
        page_rate = B * T / (sum(PAGE_TIMINGS_MS[T]) / 1e3)
        vs = value / page_rate

    line = {
        "metric": metric_of(w),
        "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "strong" if seqpar else "weak",
        "vs_baseline": vs, "dtype": w.dtype, "data": "synthetic", "config": config_of(w, args),
        "roofline": roof, "step_roofline": step_roof, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches, "clocks": clocks, "t_sweep": sweep, "configs": configs,
        "kernels": [{"name": n, "launches": c, "total_ms": t} for n, c, t in per_kernel],
        "kernel_timing": "per-kernel CUDA events on the launch stream over %d further steps after the timed region, "
                         "all enqueued behind a spin that holds the stream, so kernels run back to back" % k_prof,
    }
    if seqpar:
        line["config"]["parallelism"] = ("sp%d (the sequence split along T: %d tokens per GPU, one all-reduce of the "
                                         "[B,H,D,D+1] state per pass)" % (world, T))
        line["config"]["shard_T"] = T
        line["config"]["global_batch"] = B
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------- decode --

DECODE_SHAPE = (64, 32, 128)   # B, H, D: a serving batch whose fp32 state (134 MB) exceeds the 126 MB L2


def run_decode_reference(args):
    """The oracle's decode step on the host cores, on a bounded sample of the decode workload."""
    import oracle
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    B, H, D = DECODE_SHAPE
    nh = 64
    gam = synth.retention_gammas(H)
    qs, ks, vs = (synth.normal((B, H, D), 0, i).reshape(B * H, D)[:nh].double().numpy()[None] for i in range(3))
    st = synth.normal((B, H, D, D), 0, 3).reshape(B * H, D, D)[:nh].double().numpy()[None] * D ** -0.5
    gs = gam.double().numpy()[:1].repeat(nh)
    for _ in range(args.warmup):
        _, st = oracle.retention_step(qs, ks, vs, gs, st)
    rates, secs = [], 0.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        _, st = oracle.retention_step(qs, ks, vs, gs, st)
        dt_s = time.perf_counter() - t0
        secs += dt_s
        rates.append(nh / H / dt_s)
    value = statistics.median(rates)
    sample = "%d of %d (b,h) heads per step, fp64, one thread" % (nh, B * H)
    print(json.dumps({
        "impl": "reference", "metric": "retention decode tokens/s", "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "recurrent decode step of the decay op, B=%d H=%d D=%d" % (B, H, D)},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)
    return 0


def run_decode(args):
    """Recurrent decode steps of the decay op: every step reads and writes the fp32 state of all
    B*H heads once (S <- gamma S + k^T v, o = q S), B new tokens per step."""
    import linear_attention_attn_b200 as la
    rank, world, local = dist_env()
    dist = init_dist(world, local)
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    B, H, D = DECODE_SHAPE
    dt = torch.bfloat16
    pool = 8                                   # distinct token inputs cycled through the steps
    gam = synth.retention_gammas(H)
    hq = [synth.normal((B, H, D), rank * 100 + i, 0).mul(D ** -0.5).to(dt) for i in range(pool)]
    hk = [synth.normal((B, H, D), rank * 100 + i, 1).to(dt) for i in range(pool)]
    hv = [synth.normal((B, H, D), rank * 100 + i, 2).to(dt) for i in range(pool)]
    q, k, v = ([t.to(dev) for t in x] for x in (hq, hk, hv))
    o = torch.empty((B, H, D), dtype=dt, device=dev)
    state = (synth.normal((B, H, D, D), rank, 3) * (D ** -0.5)).to(dev)

    def step(i):
        la.la_chunk_decay_step(q[i % pool], k[i % pool], v[i % pool], o, state, gam)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    if args.steps is None:
        args.steps = auto_steps(step, stream, dev, dist)
    if dist is not None:
        dist.barrier()
    sampler = ClockSampler(gpu_selector(dev))
    sampler.start()
    launches0 = la.la_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    launches = la.la_launch_count() - launches0
    if dist is not None:
        dist.barrier()
    clocks = sampler.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    value = aggregate_throughput(B * args.steps, world, ms / 1e3)

    # end to end: this step's q, k, v from pinned host memory, o back to the host; the state stays on the GPU
    pq, pk, pv = (x[0].pin_memory() for x in (hq, hk, hv))
    po = torch.empty((B, H, D), dtype=dt).pin_memory()
    k_e2e = max(3, min(args.steps, 50))
    for it in range(2 + k_e2e):
        if it == 2:
            torch.cuda.synchronize(dev)
            x0 = torch.cuda.Event(enable_timing=True)
            x0.record(stream)
        q[0].copy_(pq, non_blocking=True)
        k[0].copy_(pk, non_blocking=True)
        v[0].copy_(pv, non_blocking=True)
        step(0)
        po.copy_(o, non_blocking=True)
    x1 = torch.cuda.Event(enable_timing=True)
    x1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(x0.elapsed_time(x1), dist, dev)
    tok_bytes = B * H * D * 2
    e2e = {"value": aggregate_throughput(B * k_e2e, world, e2e_ms / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": 3 * tok_bytes, "d2h_bytes_per_step": tok_bytes, "steps": k_e2e,
           "note": "pinned host q, k, v copied in and o copied out every step; the fp32 state stays on the GPU"}

    step_bytes = B * H * (2 * D * D * 4 + 4 * D * 2)
    peak, peak_kind = measured_peaks()
    achieved = step_bytes / (ms / args.steps / 1e3) / 1e9
    roof = {"bound": "hbm", "kernel": "decay_step", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_source": peak_kind, "traffic": None,
            "algorithmic_bytes_per_launch": step_bytes, "avg_launch_ms": ms / args.steps}
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return 0
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        nh = 64                                  # a bounded sample: 64 of the B*H heads, 20 steps
        qs, ks, vs = (x[0].reshape(B * H, D)[:nh].double().numpy()[None] for x in (hq, hk, hv))
        st = state.reshape(B * H, D, D)[:nh].double().cpu().numpy()[None]
        gs = gam.double().numpy()[:1].repeat(nh)
        t0 = time.perf_counter()
        for _ in range(20):
            _, st = oracle.retention_step(qs, ks, vs, gs, st)
        dt_s = time.perf_counter() - t0
        cpu = {"value": 20 * nh / H / dt_s, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": "%d of %d (b,h) heads x 20 steps, fp64, one thread" % (nh, B * H), "seconds": dt_s}
    line = {
        "metric": "retention decode tokens/s", "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "recurrent decode step of the decay op (S <- gamma S + k^T v, o = q S), bf16 q/k/v/o, "
                               "fp32 state, B=%d H=%d D=%d, gamma_h = 1 - 2^(-5-7h/(H-1))" % (B, H, D),
                   "B": B, "H": H, "D": D, "global_batch": B * max(1, world),
                   "parallelism": "dp%d (independent batches, no collective)" % max(1, world),
                   "l2": "state of %.0f MB per step vs 126 MB L2, no flush" % (B * H * D * D * 4 / 1e6)},
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: enough for a timed region of about 1.5 s, at least 200; "
                         "the oracle arm: 200)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--T", type=int, default=None, help="sequence length (default: the workload's)")
    ap.add_argument("--workload", choices=["bidir", "simple", "retention", "causal", "decode", "causal_norm", "gated"],
                    default="bidir",
                    help="bidir (the benchmark metric, B8 H16 D64 fp16), simple (B8 H16 D64 bf16), "
                         "retention (B8 H32 D128 bf16), decode (recurrent decay step, B64 H32 D128) or "
                         "causal_norm (causal linear attention with the norm term, B8 H16 D64 fp16) or "
                         "gated (gated linear attention, B8 H16 D64 bf16)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seqpar", action="store_true",
                    help="bidir/simple: split the workload's sequence along T across the GPUs (one all-reduce of "
                         "the state per pass; strong scaling) instead of independent batches per GPU")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", dest="sweep", action="store_false",
                    help="skip the extra T=8192/16384 device timings added to the JSON line")
    ap.add_argument("--profile-only", action="store_true",
                    help="run the warm-up and timed steps only (no e2e, CPU baseline or clock sampling): "
                         "the command profiled under ncu")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload == "decode":
        if args.impl == "reference":
            if args.steps is None:
                args.steps = 200
            return run_decode_reference(args)
        return run_decode(args)
    base = {"bidir": "bidir_f16", "simple": "simple_bf16", "retention": "retention_bf16", "causal": "causal_bf16",
            "causal_norm": "causal_norm_f16", "gated": "gated_bf16"}[args.workload]
    w = synth.WORKLOADS[base]
    w = w.with_T(args.T if args.T is not None else (4096 if args.workload != "retention" else 8192))
    if args.impl == "reference":
        if args.steps is None:
            args.steps = 200
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
