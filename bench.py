#!/usr/bin/env python
"""Benchmark of the delta-rule sequence-mixing library on B200.

Headline: the chunked DeltaNet forward on the prefill workload (B4 H16 T4096,
Dk = Dv = 128, bf16 q/k/v, fp32 beta and state, C = 64, S0 = 0), tokens/s over
all GPUs, a token being one position of one sequence with all of its heads
(tokens/s = B * T / time; the head-token rate B * H * T / time is 16x that).  One step = one deltanet_chunk_fwd call over one batch (two
launches: the chunk-parallel WY pre-pass and the chunk kernel).  Inputs are resident in HBM when the timed region starts;
two input sets alternate so consecutive steps touch disjoint 274 MB working
sets (larger than the 126 MB L2).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

For N > 1 launch with torchrun; every rank runs its own independent batch
(weak scaling, no collective on the data path) and rank 0 prints the line.
The same JSON line carries the roofline of the chunk kernel, an end-to-end
figure through the public API with host buffers, the float64 CPU oracle timed
on this host (cpu_baseline), the SM clocks seen during the timed region and
secondary measurements (linear attention, gated variant, long context,
batched decode) under "extras".
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "chunked DeltaNet fwd tokens/s + % bf16 TC peak; decode steps/s + HBM GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- helpers ----

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def algo_counts(B, H, T, Dk, Dv, C, es=2, gated=False, linear=False):
    """Algorithmic FLOPs and HBM bytes of one chunked forward.

    FLOP per head-token: delta rule 6 Dk Dv + 2 C (2 Dk + 2 Dv) (the WY chunk
    form: QK^T, KK^T, T.X, P.U, Q.S, W.S, K^T.U); linear attention
    4 Dk Dv + 2 C (Dk + Dv).  Bytes: q, k, v, beta (and alpha) read once,
    o written once, final state written once (S0 = 0 is not read).
    """
    ht = B * H * T
    if linear:
        flop = ht * (4 * Dk * Dv + 2 * C * (Dk + Dv))
        byts = ht * (2 * Dk + Dv) * es + ht * Dv * es + B * H * (Dk * Dv + Dk) * 4
    else:
        flop = ht * (6 * Dk * Dv + 2 * C * (2 * Dk + 2 * Dv))
        byts = (ht * (2 * Dk + Dv) * es + ht * 4 * (2 if gated else 1) + ht * Dv * es
                + B * H * Dk * Dv * 4)
    return flop, byts


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled every 10 ms during a
    timed region, read through NVML (read-only queries; nothing is changed)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap"}

    def __init__(self, device):
        import threading

        self.samples, self.reasons, self.smax, self.power = [], set(), None, []
        self._stop = threading.Event()
        self._thread = None
        self._handle = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nvml = pynvml
            props = torch.cuda.get_device_properties(device)
            uuid = str(getattr(props, "uuid", ""))
            h = None
            if uuid:
                for cand in (uuid, "GPU-" + uuid):
                    try:
                        h = pynvml.nvmlDeviceGetHandleByUUID(cand)
                        break
                    except Exception:
                        pass
            if h is None and pynvml.nvmlDeviceGetCount() == 1:
                h = pynvml.nvmlDeviceGetHandleByIndex(0)
            self._handle = h
            if h is not None:
                self.smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._handle = None

    def sample_now(self):
        """Take one sample (read-only NVML queries)."""
        if self._handle is None:
            return
        nv, h = self._nvml, self._handle
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
            mask = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            for bit, name in self.REASONS.items():
                if mask & bit:
                    self.reasons.add(name)
            self.power.append(nv.nvmlDeviceGetPowerUsage(h) / 1000.0)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self.sample_now()
            self._stop.wait(0.01)

    def __enter__(self):
        import threading

        if self._handle is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.smax, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.smax,
                "samples": len(self.samples), "sm_mhz_min": min(self.samples),
                "power_w_max": max(self.power) if self.power else None,
                "reasons": sorted(self.reasons)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def input_seeds(rank: int, nsets: int = 2):
    """Seeds of the input sets a rank draws: every rank owns an independent
    batch (weak scaling), so no two ranks share a seed."""
    return [rank * nsets + i for i in range(nsets)]


def whole_job_rate(world: int, units_per_rank: int, steps: int, ms_max: float) -> float:
    """Units per second over all ranks: every rank processes ``units_per_rank``
    per step, and the job takes the slowest rank's time (``ms_max``)."""
    return world * units_per_rank * steps / (ms_max * 1e-3)


def time_region(step, K, W, world, stream, sampler=None):
    """W warm-up steps, then exactly K timed steps bracketed by barrier + sync.
    Returns milliseconds (max over ranks) and the clock summary."""
    for i in range(W):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        torch.cuda.synchronize()
        start.record(stream)
        for i in range(K):
            step(i)
        end.record(stream)
        if sampler is not None:  # the queued steps are running now: one more sample
            sampler.sample_now()
        end.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    ms = start.elapsed_time(end)
    return max_over_ranks(ms, world)


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


PROFILE_SUMMARY = "chunk_main_kernel_prefill_B4H16T4096D128.md"
CHUNK_SOURCES = ("tsolve.cu", "chunk_main.cu", "common.cuh")
LAUNCHES_PER_CALL = 2  # tsolve_kernel (WY pre-pass) + chunk_main_kernel


def kernel_hash():
    """Hash of the sources of the two kernels one deltanet_chunk_fwd call runs."""
    h = hashlib.sha256()
    for fn in CHUNK_SOURCES:
        p = os.path.join(ROOT, "deltanet_sequence_mixing_b200", "csrc", fn)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def traffic_from_profile():
    """DRAM bytes of one deltanet_chunk_fwd call (pre-pass + chunk kernel) from
    the committed ncu summary, or None if it was taken on other kernel sources."""
    p = os.path.join(ROOT, "profiles", PROFILE_SUMMARY)
    if not os.path.exists(p):
        return None
    vals = {}
    for line in open(p):
        if line.startswith("traffic_bytes_per_call:") or line.startswith("kernel_source_hash:"):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("kernel_source_hash") != kernel_hash():
        return None
    try:
        return float(vals["traffic_bytes_per_call"])
    except (KeyError, ValueError):
        return None


# ------------------------------------------------------------ CPU oracle -----

def cpu_oracle_rate(target_s=10.0, max_reps=4):
    """Time the float64 oracle (as it stands) on the prefill workload on this
    host's cores; returns (tokens/s, cores, sample description)."""
    import oracle
    from deltanet_sequence_mixing_b200 import inputs as gen

    oracle.build()
    w = gen.PREFILL
    x = gen.make_workload(w, seed=0)
    cores = os.cpu_count() or 1
    tokens, secs, reps = 0, 0.0, 0
    while reps < max_reps and secs < target_s:
        t0 = time.perf_counter()
        oracle.deltanet(x["q"], x["k"], x["v"], x["beta"], nthreads=cores)
        secs += time.perf_counter() - t0
        tokens += w.B * w.T  # tokens of all heads: B * T per pass
        reps += 1
    sample = (f"{reps} pass(es) over the full prefill workload (B4 H16 T4096 D128 bf16 inputs), "
              f"float64 per-token recurrence, {cores} threads over (b,h)")
    return tokens / secs, cores, sample


def run_reference(args):
    """The reference arm: the float64 CPU oracle, timed on the host cores."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from deltanet_sequence_mixing_b200 import inputs as gen

    oracle.build()
    w = gen.PREFILL
    cores = os.cpu_count() or 1
    nseq = min(w.B * w.H, cores)
    x = gen.make_inputs(1, nseq, w.T, w.Dk, w.Dv, w.dtype, seed=0)
    # calibrate: tokens per sequence per step so that all steps take ~2 minutes
    t0 = time.perf_counter()
    oracle.deltanet(x["q"][:, :, :256], x["k"][:, :, :256], x["v"][:, :, :256],
                    x["beta"][:, :, :256], nthreads=cores)
    per_tok = (time.perf_counter() - t0) / 256
    budget = 120.0 / max(1, args.steps + args.warmup)
    L = int(max(64, min(w.T, (budget / max(per_tok, 1e-9)) // 64 * 64)))
    sl = {k: (None if v is None else v[:, :, :L].contiguous()) for k, v in x.items()}

    def step():
        oracle.deltanet(sl["q"], sl["k"], sl["v"], sl["beta"], nthreads=cores)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    secs = time.perf_counter() - t0
    # a token of the workload carries H heads: nseq (b, h) sequences of L
    # positions are nseq * L / H tokens
    tok = nseq * L * args.steps / w.H
    value = tok / secs
    sample = (f"per step: {nseq} (b,h) sequences x {L} positions of the prefill workload "
              f"(D128, bf16 inputs; {nseq * L / w.H:g} tokens of {w.H} heads), float64 per-token "
              f"recurrence, {cores} threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": gen.PREFILL.name, "B": w.B, "H": w.H, "T": w.T, "Dk": w.Dk,
                   "Dv": w.Dv, "C": w.C, "sampled": True},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------- GPU arm -------

def extras_measure(dn, gen, dev, stream, peaks):
    """Secondary workloads, each timed on its own (a few steps)."""
    out = {}
    hbm = peaks["hbm_gbs"]
    tc = peaks["bf16_tflops"]

    def timed(fn, n, w=3):
        for _ in range(w):
            fn()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(n):
            fn()
        e.record(stream)
        e.synchronize()
        return s.elapsed_time(e) / n

    # linear attention on the prefill shapes
    w = gen.PREFILL_LINEAR
    x = gen.make_workload(w, seed=1, device=dev)
    o = torch.empty_like(x["v"])
    S = torch.empty(w.B, w.H, w.Dk, w.Dv, device=dev)
    z = torch.empty(w.B, w.H, w.Dk, device=dev)
    ms = timed(lambda: dn.linear_attn_fwd(x["q"], x["k"], x["v"], C=w.C, o=o, S_out=S, z_out=z), 20)
    fl, by = algo_counts(w.B, w.H, w.T, w.Dk, w.Dv, w.C, linear=True)
    out["linear_attn_prefill"] = {"tokens_per_s": w.B * w.T / (ms * 1e-3), "ms": ms,
                                  "GBps": by / (ms * 1e-3) / 1e9,
                                  "hbm_frac": by / (ms * 1e-3) / 1e9 / hbm,
                                  "TFLOPs": fl / (ms * 1e-3) / 1e12,
                                  "tc_frac": fl / (ms * 1e-3) / 1e12 / tc}
    del x, o, S, z

    # gated (forgetting) variant
    w = gen.FORGET
    x = gen.make_workload(w, seed=2, device=dev)
    o = torch.empty_like(x["v"])
    S = torch.empty(w.B, w.H, w.Dk, w.Dv, device=dev)
    ms = timed(lambda: dn.deltanet_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], x["alpha"], C=w.C,
                                             o=o, S_out=S), 5)
    fl, by = algo_counts(w.B, w.H, w.T, w.Dk, w.Dv, w.C, gated=True)
    out["gated_forget"] = {"tokens_per_s": w.B * w.T / (ms * 1e-3), "ms": ms,
                           "GBps": by / (ms * 1e-3) / 1e9, "hbm_frac": by / (ms * 1e-3) / 1e9 / hbm,
                           "TFLOPs": fl / (ms * 1e-3) / 1e12, "tc_frac": fl / (ms * 1e-3) / 1e12 / tc}
    del x, o, S

    # long context, C = 64 and C = 128
    for w in (gen.LONG64, gen.LONG128):
        x = gen.make_workload(w, seed=3, device=dev)
        o = torch.empty_like(x["v"])
        S = torch.empty(w.B, w.H, w.Dk, w.Dv, device=dev)
        try:
            ms = timed(lambda: dn.deltanet_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], C=w.C, o=o,
                                                     S_out=S), 3, 1)
        except dn.DeltaNetError as e:
            out[f"long_C{w.C}"] = {"unavailable": str(e)}
            continue
        fl, by = algo_counts(w.B, w.H, w.T, w.Dk, w.Dv, w.C)
        out[f"long_C{w.C}"] = {"tokens_per_s": w.B * w.T / (ms * 1e-3), "ms": ms,
                               "GBps": by / (ms * 1e-3) / 1e9,
                               "hbm_frac": by / (ms * 1e-3) / 1e9 / hbm,
                               "TFLOPs": fl / (ms * 1e-3) / 1e12,
                               "tc_frac": fl / (ms * 1e-3) / 1e12 / tc}
        del x, o, S

    # long context over few heads (B1 H8 T65536 D128 bf16 C64): unsplit, and with
    # the sequence split (segments side by side, joined afterwards)
    w = dataclasses.replace(gen.LONG64, H=8, name=gen.LONG64.name.replace("H32", "H8"))
    x = gen.make_workload(w, seed=4, device=dev)
    o = torch.empty_like(x["v"])
    S = torch.empty(w.B, w.H, w.Dk, w.Dv, device=dev)
    fl, by = algo_counts(w.B, w.H, w.T, w.Dk, w.Dv, w.C)
    for split in (False, True):
        ms = timed(lambda: dn.deltanet_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], C=w.C, o=o, S_out=S,
                                                 seq_split=split), 5, 2)
        key = "long_8heads_split" if split else "long_8heads"
        out[key] = {"segments": dn.seq_segments(w.B, w.H, w.T, w.Dk, w.Dv) if split else 1,
                    "tokens_per_s": w.B * w.T / (ms * 1e-3), "ms": ms, "GBps": by / (ms * 1e-3) / 1e9,
                    "hbm_frac": by / (ms * 1e-3) / 1e9 / hbm}
    del x, o, S

    # the options and the backward on the prefill shape (B4 H16 T4096 D128 bf16)
    w = gen.PREFILL
    fl, by = algo_counts(w.B, w.H, w.T, w.Dk, w.Dv, w.C)
    x = gen.make_inputs(w.B, w.H, w.T, w.Dk, w.Dv, w.dtype, gated=False, seed=6, device=dev, raw=True)
    o = torch.empty_like(x["v"])
    S = torch.empty(w.B, w.H, w.Dk, w.Dv, device=dev)
    ms = timed(lambda: dn.deltanet_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], C=w.C, o=o, S_out=S,
                                             prestep=True), 20)
    out["prestep_prefill"] = {"path": "tcgen05 (layer pre-step inside the call)", "ms": ms,
                              "tokens_per_s": w.B * w.T / (ms * 1e-3), "GBps": by / (ms * 1e-3) / 1e9,
                              "hbm_frac": by / (ms * 1e-3) / 1e9 / hbm}
    del x
    x = gen.make_inputs(w.B, w.H, w.T, w.Dk, w.Dv, w.dtype, gated=True, seed=7, device=dev,
                        gate_per_dim=True)
    ms = timed(lambda: dn.deltanet_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], x["alpha"], C=w.C,
                                             o=o, S_out=S), 3, 1)
    by_kda = by + w.B * w.H * w.T * w.Dk * 4  # plus the per-dimension decays
    out["kda_prefill"] = {"path": "CUDA cores, float32 (per-dimension decay)", "ms": ms,
                          "tokens_per_s": w.B * w.T / (ms * 1e-3), "GBps": by_kda / (ms * 1e-3) / 1e9,
                          "hbm_frac": by_kda / (ms * 1e-3) / 1e9 / hbm,
                          "TFLOPs_fp32": fl / (ms * 1e-3) / 1e12}
    del x
    x = gen.make_workload(w, seed=8, device=dev)
    dO = torch.randn(w.B, w.H, w.T, w.Dv, device=dev).to(w.dtype)
    nb = dn.lib().deltanet_chunk_bwd_workspace_bytes(w.B, w.H, w.T, w.Dk, w.Dv, 1)
    bws = torch.empty(nb, dtype=torch.uint8, device=dev)
    ms = timed(lambda: dn.deltanet_chunk_bwd(x["q"], x["k"], x["v"], x["beta"], dO, workspace=bws), 2, 1)
    ht = w.B * w.H * w.T
    # inputs q, k, v, dO, beta read; dq, dk, dv (float32), dbeta written; state checkpoints
    # written and read once
    by_bwd = ht * (3 * w.Dk + w.Dv) * 2 + ht * 4 + ht * (2 * w.Dk + w.Dv) * 4 + ht * 4 + 2 * (nb - 256)
    out["backward_prefill"] = {"path": "CUDA cores, float32", "ms": ms,
                               "tokens_per_s": w.B * w.T / (ms * 1e-3),
                               "GBps": by_bwd / (ms * 1e-3) / 1e9, "hbm_frac": by_bwd / (ms * 1e-3) / 1e9 / hbm,
                               "bytes": by_bwd}
    del x, dO, bws, o, S

    # batched decode: 256 x 32 states from a 512-token prefill, then 1024 steps
    B, H, D = gen.DECODE_SEQS, gen.DECODE_HEADS, 128
    pre = gen.make_inputs(B, H, gen.DECODE_PREFILL, D, D, torch.bfloat16, seed=4, device=dev)
    _, S = dn.deltanet_chunk_fwd(pre["q"], pre["k"], pre["v"], pre["beta"])
    del pre
    steps = gen.make_inputs(B, H, gen.DECODE_STEPS, D, D, torch.bfloat16, seed=5, device=dev)
    # per-step slices, contiguous, generated before timing
    qs = steps["q"].permute(2, 0, 1, 3).contiguous()
    ks = steps["k"].permute(2, 0, 1, 3).contiguous()
    vs = steps["v"].permute(2, 0, 1, 3).contiguous()
    bs = steps["beta"].permute(2, 0, 1).contiguous()
    del steps
    o = torch.empty(B, H, D, dtype=torch.bfloat16, device=dev)
    n = gen.DECODE_STEPS
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for t in range(n):
        dn.deltanet_decode_step(qs[t], ks[t], vs[t], bs[t], S, o=o)
    e.record(stream)
    e.synchronize()
    ms = s.elapsed_time(e) / n
    by = B * H * (2 * D * D * 4 + 3 * D * 2 + 4 + D * 2)
    out["decode"] = {"steps_per_s": 1e3 / ms, "us_per_step": ms * 1e3,
                     "GBps": by / (ms * 1e-3) / 1e9, "hbm_frac": by / (ms * 1e-3) / 1e9 / hbm,
                     "bytes_per_step": by, "states": B * H, "steps": n}
    # the same steps with the pre-step and a per-dimension decay (alpha (B,H,Dk) read as well)
    a = torch.rand(B, H, D, device=dev) * 0.1 + 0.9
    s.record(stream)
    for t in range(n):
        dn.deltanet_decode_step(qs[t], ks[t], vs[t], bs[t], S, alpha=a, o=o, prestep=True)
    e.record(stream)
    e.synchronize()
    ms = s.elapsed_time(e) / n
    by2 = by + B * H * D * 4
    out["decode_prestep_kda"] = {"steps_per_s": 1e3 / ms, "us_per_step": ms * 1e3,
                                 "GBps": by2 / (ms * 1e-3) / 1e9, "hbm_frac": by2 / (ms * 1e-3) / 1e9 / hbm}
    return out


def profile_run(args):
    """Launch one kernel on its workload (warm-up launches + 1), for ncu."""
    import deltanet_sequence_mixing_b200 as dn
    from deltanet_sequence_mixing_b200 import inputs as gen

    dev = torch.device("cuda", 0)
    n = args.warmup + 1
    if args.profile in ("chunk", "gated", "linear", "long64", "long128", "long64q", "long128q", "split8",
                        "split2"):
        # long64q / long128q: the long workloads on a quarter of the sequence
        # (T = 16384, still far larger than L2), small enough for a full ncu capture;
        # split8 / split2: the long workload over 8 / 2 heads (B1 T65536) with the sequence split
        quarter = lambda w: dataclasses.replace(w, T=w.T // 4, name=w.name.replace("T65536", "T16384"))
        w = {"chunk": gen.PREFILL, "gated": gen.FORGET, "linear": gen.PREFILL_LINEAR,
             "long64": gen.LONG64, "long128": gen.LONG128,
             "long64q": quarter(gen.LONG64), "long128q": quarter(gen.LONG128),
             "split8": dataclasses.replace(gen.LONG64, H=8, name=gen.LONG64.name.replace("H32", "H8")),
             "split2": dataclasses.replace(gen.LONG64, H=2, name=gen.LONG64.name.replace("H32", "H2")),
             }[args.profile]
        x = gen.make_workload(w, seed=0, device=dev)
        for _ in range(n):
            if args.profile == "linear":
                dn.linear_attn_fwd(x["q"], x["k"], x["v"], C=w.C)
            else:
                dn.deltanet_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], x["alpha"], C=w.C,
                                      seq_split=args.profile.startswith("split"))
    else:
        B, H, D = gen.DECODE_SEQS, gen.DECODE_HEADS, 128
        S = torch.randn(B, H, D, D, device=dev) * 0.01
        st = gen.make_decode_step_inputs(B, H, D, D, torch.bfloat16, seed=0, device=dev)
        for _ in range(n):
            dn.deltanet_decode_step(st["q"], st["k"], st["v"], st["beta"], S)
    torch.cuda.synchronize()
    status = dn.deltanet_get_device_status(dev)
    print(json.dumps({"profile": args.profile, "launches": n, "status": status}))
    return 0 if status == 0 else 1


def graph_replay(step, reps, stream, tokens):
    """The same prefill step replayed from a CUDA graph (two calls per graph,
    one per input set, so every replay still streams 2 x 274 MB through L2):
    CUDA events around each of `reps` replays, median and minimum per call.
    A supplement to the eagerly launched timed region, which the JSON line's
    value comes from; a capture the runtime refuses is reported, not raised."""
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step(0)
            step(1)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            step(0)
            step(1)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        times = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b) / 2)
        del g
        med, mn = statistics.median(times), min(times)
        return {"ms_per_call_median": med, "ms_per_call_min": mn, "replays": reps, "calls_per_replay": 2,
                "tokens_per_s_median": tokens / (med * 1e-3), "tokens_per_s_max": tokens / (mn * 1e-3)}
    except Exception as exc:  # noqa: BLE001 - reported in the JSON line
        torch.cuda.synchronize()
        return {"error": f"{type(exc).__name__}: {exc}"[:300]}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--profile", choices=["chunk", "linear", "gated", "long64", "long128", "long64q", "long128q",
                                          "split8", "split2", "decode"],
                    default=None,
                    help="untimed run for a profiler: --warmup launches of one kernel on its "
                         "workload, then one more (the one to capture)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.profile:
        return profile_run(args)

    world, rank, local = dist_setup(args)
    import deltanet_sequence_mixing_b200 as dn
    from deltanet_sequence_mixing_b200 import inputs as gen

    dn.lib()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = load_peaks()
    w = gen.PREFILL
    sets = [gen.make_workload(w, seed=sd, device=dev) for sd in input_seeds(rank)]
    o = [torch.empty_like(s["v"]) for s in sets]
    S = [torch.empty(w.B, w.H, w.Dk, w.Dv, device=dev) for _ in sets]
    ws = dn.workspace_for(dev, dn.lib().deltanet_workspace_bytes(w.B, w.H, w.T, w.Dk, w.Dv, w.C, 1))

    def step(i):
        j = i & 1
        x = sets[j]
        dn.deltanet_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], None, None, C=w.C, o=o[j],
                              S_out=S[j], workspace=ws)

    sampler = ClockSampler(dev)
    ms = time_region(step, args.steps, args.warmup, world, stream, sampler)
    status = dn.deltanet_get_device_status(dev)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    ms_step = ms / args.steps
    tokens = w.B * w.T  # B * T tokens per step, each with all H heads
    graph = graph_replay(step, 30, stream, tokens) if rank == 0 else None
    value = whole_job_rate(world, tokens, args.steps, ms)

    flop, byts = algo_counts(w.B, w.H, w.T, w.Dk, w.Dv, w.C)
    achieved = byts / (ms_step * 1e-3) / 1e9
    tflops = flop / (ms_step * 1e-3) / 1e12
    traffic = traffic_from_profile()
    roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
            "traffic_source": (f"ncu profile summary profiles/{PROFILE_SUMMARY} (DRAM read + write "
                               "of one call), matched to the current kernel sources by hash")
            if traffic is not None else "no profile of the current kernel sources",
            "peak_source": peak_src, "algorithmic_bytes_per_launch": byts,
            "tensor": {"achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                       "frac": tflops / peaks["bf16_tflops"], "algorithmic_flop_per_launch": flop}}

    # end to end through the public API with pinned host buffers
    hx = {k: (None if v is None else v.cpu().pin_memory()) for k, v in sets[0].items()}
    ho = torch.empty(o[0].shape, dtype=o[0].dtype).pin_memory()
    hS = torch.empty(S[0].shape, dtype=torch.float32).pin_memory()

    hws = dn.host_workspace_for(dev, w.B, w.H, w.T, w.Dk, w.Dv, w.C, w.dtype)

    def e2e_step(i):
        # the C-ABI host-buffer call: it copies the inputs in, computes and copies
        # o and S back, streaming groups of heads so the copies overlap the compute
        dn.deltanet_chunk_fwd_host(hx["q"], hx["k"], hx["v"], hx["beta"], None, None, C=w.C,
                                   o=ho, S_out=hS, workspace=hws, device=dev)

    e2e_ms = time_region(e2e_step, args.e2e_steps, 3, world, stream)
    h2d = sum(hx[k_].numel() * hx[k_].element_size() for k_ in ("q", "k", "v", "beta"))
    d2h = ho.numel() * ho.element_size() + hS.numel() * 4
    status = dn.deltanet_get_device_status(dev, workspace=hws)
    if status != 0:
        raise RuntimeError(f"device status {status} after the end-to-end region")
    e2e = {"value": whole_job_rate(world, tokens, args.e2e_steps, e2e_ms), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "ms_per_step": e2e_ms / args.e2e_steps,
           "path": "deltanet_chunk_fwd_host: pinned host buffers in and out, heads in 4 groups"}
    del hx, ho, hS, hws

    extras = None
    if not args.no_extras and rank == 0:
        del sets, o, S
        torch.cuda.empty_cache()
        extras = extras_measure(dn, gen, dev, stream, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, sample = cpu_oracle_rate()
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": sample}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "Dk": w.Dk, "Dv": w.Dv,
                       "C": w.C, "state": "fp32", "per_gpu": "independent batch per GPU",
                       "tokens_per_step": tokens, "head_tokens_per_step": tokens * w.H,
                       "parallelism": f"dp{world}",
                       "l2": "inputs larger than L2: two alternating input sets of 274 MB each"},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": LAUNCHES_PER_CALL * args.steps,
            "clocks": sampler.summary(), "graph": graph, "extras": extras,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
