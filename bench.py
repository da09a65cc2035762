#!/usr/bin/env python
"""Throughput of the LoLA chunkwise hybrid-attention layer on B200: one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lola|reference]
                    [--workload 3] [--extra 2,5] [--no-decode] [--no-next]
    python bench.py --sweep [--steps K]     # single-layer latency over (eta, lambda)

A step is one pass of the whole layer over one batch of synthetic input:
reset the memories, then chunkwise prefill of B x T tokens (window advance,
SRE scoring, top-lambda retention, fold and the hybrid output of every
chunk).  The headline workload is the largest single-GPU one: the
Llama-3.1-8B-shaped 16K prefill (B = 4, 32 q / 8 kv heads, d = 128, phi dim
128, eta = 512, lambda = 1024, chunk 128, bf16 inputs, 16 needles per
sequence).  The line also carries the 8B-shaped 4K and the 1B-shaped 32K
prefills under "workloads", the per-token decode throughput of the 8B-shaped
decode workload (B = 64 after a 4096-token prefill, all 1024 steps) under
"decode", and the analysis / ablation legs on the 4K workload under "next".

Multi-GPU: one process per GPU; every rank runs its own copy of the workload
(the path shards into independent (sequence, kv head) streams and needs no
collective), timing is the max over ranks, value = all ranks' tokens / time.
"""
from __future__ import annotations

import argparse
from dataclasses import replace
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "prefill tokens/s and decode tokens/s at 1 B200; % of roofline; oracle match"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# Algorithmic work (counts only what the method must compute or move)
# ---------------------------------------------------------------------------
def prefill_work(w: synth.Workload) -> dict:
    """FLOPs and bytes per prefill launch of each kernel class."""
    B, T, Hq, Hkv, d, Dh, D, C = w.B, w.T, w.Hq, w.Hkv, w.d, w.Dh, w.D, w.chunk
    e = 2 if w.dtype == "bf16" else 4
    att = lin = 0
    scan_fl = 0
    n_fold = 0
    for c in range(T // C):
        t0 = c * C
        n_g = min(w.lam, max(0, t0 - w.eta))
        n_w = min(w.eta, t0)
        # causal chunk: query i sees i + 1 block keys
        keys = C * (n_g + n_w) + C * (C + 1) // 2
        att += 4 * d * keys
        lin += C * (2 * D * d + 2 * D + 2 * d * Dh)
        n_l = max(0, t0 + C - w.eta) - max(0, t0 - w.eta)
        if n_l and n_g + n_l > w.lam:
            n = n_g + n_l
            f = n - w.lam
            scan_fl += 2 * n * D * d + 2 * n * D + 3 * n * d + 2 * f * D * d + f * D
            n_fold += f
    out_fl = B * Hq * (att + lin)
    return {
        "phi": dict(flops=2 * B * T * Hkv * d * Dh,
                    bytes=B * T * Hkv * d * e + Hkv * d * Dh * e + B * T * Hkv * D * 4),
        "scan": dict(flops=B * Hkv * scan_fl, bytes=B * Hkv * 2 * D * d * 4),
        "output": dict(flops=out_fl, bytes=B * T * Hq * d * (e + 4) + 2 * B * T * Hkv * d * e),
        "total_flops": B * Hkv * scan_fl + out_fl + 2 * B * T * Hkv * d * Dh,
    }


def sre_map_work(w: synth.Workload) -> tuple[int, int]:
    """(pairs, FLOPs) of one SRE-map launch after a prefill of w.T tokens from position 0:
    every folded pair at every state time costs H^T phi (2 D d), phi . s (2 D) and the
    residual's divide, subtract and square-add (3 d)."""
    pairs = 0
    for c in range(w.T // w.chunk + 1):
        left = max(0, c * w.chunk - w.eta)
        pairs += left - min(w.lam, left)
    pairs *= w.B * w.Hkv
    return pairs, pairs * (2 * w.D * w.d + 2 * w.D + 3 * w.d)


def scorer_work(w: synth.Workload) -> int:
    """FLOPs of one window-score launch (alternative rules) over a prefill of w.T tokens
    from position 0: every (key, query, head) credit costs q.k (2 d), phi(q).phi(k) (2 D)
    and the rule's term (3); every query row's feature map costs 2 d Dh once."""
    credits = 0
    for i in range(w.T):
        credits += min(w.T, ((i + w.eta) // w.chunk + 1) * w.chunk) - i
    S = w.B * w.Hkv
    return S * (credits * w.Gq * (2 * w.d + 2 * w.D + 3) + w.T * w.Gq * 2 * w.d * w.Dh)


def decode_step_bytes(w: synth.Workload) -> int:
    """HBM bytes one decode step must move (all streams, steady state)."""
    e = 2 if w.dtype == "bf16" else 4
    d, D = w.d, w.D
    rd = D * d * 4 + D * 4 + w.lam * 2 * d * e + w.eta * 2 * d * e + (w.Gq + 2) * d * e
    wr = D * d * 4 + D * 4 + w.Gq * d * 4 + 2 * 2 * d * e + 2 * 4
    return w.B * w.Hkv * (rd + wr)


def decode_step_flops(w: synth.Workload) -> int:
    d, D, n = w.d, w.D, w.lam + 1
    keys = w.lam + w.eta + 1
    per = (w.Gq * (4 * d * keys + 2 * D * d + 2 * d * w.Dh) + 2 * n * D * d + 2 * D * d + 2 * d * w.Dh)
    return w.B * w.Hkv * per


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
SM_MAX_MHZ_DEFAULT = 1965.0     # clocks.max.sm of a B200 when no measured value is available


def max_over_ranks(x: float, world: int, device) -> float:
    """The maximum of x over all ranks (the collective runs on `device`: the rank's
    GPU under nccl, the CPU under gloo)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return units_per_rank * world / (ms_max / 1e3)


def fp32_alu_peak_tflops(num_sms: int, sm_mhz: float) -> float:
    """FP32 FMA peak of the CUDA cores: SMs x 128 lanes x 2 FLOP x max SM clock."""
    return num_sms * 128 * 2 * sm_mhz * 1e6 / 1e12


# Nominal dense tensor-core rates of a B200 (PFLOP/s), used only as ratios to carry
# the measured bf16 peak over to another operand type.
NOMINAL_DENSE_PFLOPS = {"bf16": 2.25, "tf32": 1.1}


def layer_bytes(w: synth.Workload) -> int:
    """Algorithmic HBM bytes of one prefill step: q, k, v in, y out (f32), W, and the
    final state of every stream (H, s, cache and window K/V and positions)."""
    e = 2 if w.dtype == "bf16" else 4
    S = w.B * w.Hkv
    io = w.B * w.T * (w.Hq + 2 * w.Hkv) * w.d * e + w.B * w.T * w.Hq * w.d * 4
    state = S * (w.D * w.d * 4 + w.D * 4 + (w.lam + w.eta) * (2 * w.d * e + 4))
    return io + w.Hkv * w.d * w.Dh * e + state


def layer_roofline(w: synth.Workload, ms_step: float, peaks) -> dict:
    """The layer against max(FLOP time at the bf16 tensor peak, byte time at HBM peak)."""
    fl = prefill_work(w)["total_flops"]
    by = layer_bytes(w)
    t_fl = fl / (peaks["bf16_tflops"] * 1e12) * 1e3
    t_by = by / (peaks["hbm_gbs"] * 1e9) * 1e3
    roof = max(t_fl, t_by)
    return {"flops": fl, "bytes": by, "ms_flops_at_peak": t_fl, "ms_bytes_at_peak": t_by,
            "ms_at_roofline": roof, "bound": "tensor" if t_fl >= t_by else "hbm", "frac": roof / ms_step}


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


# What each part of the path computes in (bf16 inputs).
PRECISIONS = {"inputs": "bf16 q, k, v, W", "phi": "f32",
              "sre": "3xTF32 tensor-core products (f32-accurate), f32 accumulation",
              "fold": "bf16 tensor-core products of 3-part bf16 splits (products to 2^-24 relative), f32 state",
              "select": "exact radix select over f32 score bits",
              "attention": "bf16 QK^T, f16 PV (P in tensor memory), tf32 phi(q)^T H on the tensor cores, f32 softmax and accumulation",
              "output": "f32 y", "decode": "f32 on the CUDA cores"}
DTYPE = "bf16+f16+tf32+f32"


# Sources a kernel class's counters depend on: its own files plus the shared headers.
KERNEL_SOURCES = {"phi": ["phi.cu"], "scan": ["scan.cu", "scan_tc.cu", "chain_common.cuh"],
                  "output": ["output_tc.cu", "output_ws.cu", "output.cu"],
                  "finalize": ["finalize.cu"], "decode": ["decode.cu"], "sre_map": ["sre_map.cu"],
                  "scores": ["scores.cu"]}
SHARED_SOURCES = ["device_common.cuh", "lola_internal.h", "umma.cuh"]


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_kv_caching_b200", "csrc")
    for f in sorted(KERNEL_SOURCES[kernel] + SHARED_SOURCES):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes (per step for prefill kernel classes, per launch for decode) from the
    committed ncu summary, if it was taken on the current kernels."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        ent = t.get(f"{kernel}@{workload}")
        if ent and ent.get("source_hash") == kernel_source_hash(kernel):
            return ent.get("dram_bytes_per_step", ent.get("dram_bytes_per_launch"))
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clocks/throttle sampling while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines: list[str] = []

    def start(self):
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
            if self.gpu_id:
                cmd += ["-i", self.gpu_id]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict | None:
        if not self.proc:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# the oracle on the host cores (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------
def _oracle_stream_job(job):
    """One (sequence, kv head) stream through the CPU oracle (runs in a spawned worker).

    job = (workload, b, g, expected sets by chunk start or None, library y [Gq,T,d] or None).
    Returns (seconds, match stats) where the oracle follows the library's retained sets
    up to ties when `expected` is given."""
    w, b, g, exp, yg = job
    from oracle import LolaStream, valid_alternative
    a = synth.stream_arrays(w, b, g)
    Wg = synth.weights(w)[g]
    stats = dict(hard=0, ties=0)

    def choose(rec):
        gset = exp.get(rec["t0"]) if exp else None
        if gset is None or gset == rec["keep"]:
            return None
        if valid_alternative(rec["E"], rec["score"], w.lam, gset):
            stats["ties"] += 1
            return gset
        stats["hard"] += 1
        return None

    t0 = time.perf_counter()
    st = LolaStream(Wg, w.eta, w.lam)
    y = st.prefill(a["q"][:, :w.T], a["k"][:w.T], a["v"][:w.T], w.chunk, choose=choose if exp else None)
    secs = time.perf_counter() - t0
    err = None
    if yg is not None:
        err = float(np.abs(yg - y).max() / np.abs(y).max())
    return secs, stats, err, y.shape[0] * y.shape[1]


def _limit_blas_threads():
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


def oracle_sample(w: synth.Workload, streams, workers: int, gpu=None):
    """Run the CPU oracle over whole streams, one stream per worker process (spawned,
    one BLAS thread each), all workers at once.

    Returns (layer tokens, wall seconds, streams done, match) where a stream of T tokens
    counts as T / Hkv layer tokens (a token spans Hkv streams).  With `gpu` = (y
    [B,T,Hq,d] host tensor, trace [S, chunks+1, lambda]) the oracle follows the
    library's retained sets up to ties and reports the match."""
    import multiprocessing as mp
    jobs = []
    for (b, g) in streams:
        exp, yg = None, None
        if gpu is not None:
            y_host, trace = gpu
            if trace is not None:
                tr = trace[b * w.Hkv + g]
                exp = {ci * w.chunk: sorted(int(p) for p in tr[ci + 1] if p >= 0) for ci in range(w.T // w.chunk)}
            yg = y_host[b, :, g * w.Gq:(g + 1) * w.Gq, :].permute(1, 0, 2).double().numpy()
        jobs.append((w, b, g, exp, yg))
    t0 = time.perf_counter()
    if workers <= 1:
        res = [_oracle_stream_job(j) for j in jobs]
    else:
        with mp.get_context("spawn").Pool(workers, initializer=_limit_blas_threads) as pool:
            res = pool.map(_oracle_stream_job, jobs, chunksize=1)
    wall = time.perf_counter() - t0
    match = dict(streams=0, hard_mismatch=0, tie_swaps=0, max_rel_err_y=0.0, rows_checked=0)
    for secs, stats, err, rows in res:
        if err is not None:
            match["streams"] += 1
            match["hard_mismatch"] += stats["hard"]
            match["tie_swaps"] += stats["ties"]
            match["max_rel_err_y"] = max(match["max_rel_err_y"], err)
            match["rows_checked"] += rows
    return len(jobs) * w.T / w.Hkv, wall, len(jobs), match


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


# ---------------------------------------------------------------------------
def run_reference(args, w, rank):
    if rank != 0:
        return 0
    cores = host_cores()
    streams = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    per_step = min(len(streams), cores)
    times = []
    toks = []
    for i in range(args.warmup + args.steps):
        sel = [streams[(i * per_step + j) % len(streams)] for j in range(per_step)]
        n, secs, _, _ = oracle_sample(w, sel, per_step)
        if i >= args.warmup:
            times.append(secs)
            toks.append(n)
    value = sum(toks) / sum(times)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": workload_config(w, 1),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": per_step, "kind": "oracle",
                             "cpu": cpu_model(), "host_cores": cores,
                             "sample": f"{per_step} whole (sequence, kv head) streams of {w.T} tokens per step, "
                                       f"one per core in parallel (= {per_step * w.T / w.Hkv:.0f} layer tokens)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w: synth.Workload, world: int) -> dict:
    return {"workload": w.name, "B": w.B, "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "phi_dim": w.D,
            "eta": w.eta, "lambda": w.lam, "chunk": w.chunk, "input_dtype": w.dtype,
            "l2": "flushed between timed steps (256 MB write)",
            "parallelism": f"replicas x{world} (independent streams)"}


# The pages' single-layer forward latencies (App. B, Tables 7-8; RTX 4090, batch 2,
# 4096 tokens, 32 heads, emb 4096, precision not stated): context only.
PAGES_LAYER_MS_RTX4090 = {"eta512": {"lambda0": 4.2, "lambda512": 9.7},
                          "eta64": {"lambda0": 18.3, "lambda512": 35.5}}


def run_sweep(args):
    """Per-layer prefill latency over the (eta, lambda) grid: one JSON line."""
    import torch
    import sparse_kv_caching_b200 as lola

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w0 = synth.sweep_workload(synth.SWEEP_ETAS[0], synth.SWEEP_LAMBDAS[0])
    full = synth.full_arrays(w0)          # the same inputs at every grid point

    def to_dev(x):
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(x).to(dev)

    q, k, v, W = (to_dev(full[x]) for x in ("q", "k", "v", "W"))
    y = torch.empty((w0.B, w0.T, w0.Hq, w0.d), dtype=torch.float32, device=dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    points = []
    for eta in synth.SWEEP_ETAS:
        for lam in synth.SWEEP_LAMBDAS:
            w = synth.sweep_workload(eta, lam)
            cfg = lola.make_config(w.B, w.Hq, w.Hkv, w.d, w.Dh, w.eta, w.lam, w.chunk, w.dtype, w.T)
            layer = lola.LolaLayer(cfg, W, device=dev)
            for _ in range(args.warmup):
                layer.reset()
                layer.prefill(q, k, v, y)
            torch.cuda.synchronize()
            layer.profile(True)
            total = 0.0
            for _ in range(args.steps):
                flush.zero_()
                ev0 = torch.cuda.Event(enable_timing=True)
                ev1 = torch.cuda.Event(enable_timing=True)
                ev0.record(stream)
                layer.reset()
                layer.prefill(q, k, v, y)
                ev1.record(stream)
                ev1.synchronize()
                total += ev0.elapsed_time(ev1)
            prof = layer.profile_read()
            layer.profile(False)
            ms = total / args.steps
            kern = {kk: round(prof[kk][0] / args.steps, 4) for kk in ("phi", "scan", "output", "finalize")}
            points.append({"eta": eta, "lambda": lam, "ms": round(ms, 4),
                           "tokens_per_s": w.B * w.T / (ms / 1e3), "kernel_ms_per_step": kern})
            layer.close()
            del layer
    line = {"metric": "single-layer prefill latency over the (eta, lambda) grid", "unit": "ms",
            "higher_is_better": False, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "dtype": DTYPE, "data": "synthetic",
            "config": {"workload": "layer-sweep", "B": w0.B, "T": w0.T, "Hq": w0.Hq, "Hkv": w0.Hkv, "d": w0.d,
                       "phi_dim": w0.D, "chunk": w0.chunk, "input_dtype": w0.dtype,
                       "l2": "flushed between timed steps (256 MB write)"},
            "sweep": points,
            "context": {"pages_single_layer_ms_rtx4090": PAGES_LAYER_MS_RTX4090}}
    print(json.dumps(line))
    return 0


def _to_dev(x, dev):
    import torch
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    return torch.from_numpy(x).to(dev)


def _timed_prefills(layer, q, k, v, y, flush, steps, stream) -> float:
    """Mean device time (ms) of `steps` reset + prefill passes, L2 flushed before each."""
    import torch
    total = 0.0
    for _ in range(steps):
        flush.zero_()
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        layer.reset()
        layer.prefill(q, k, v, y)
        ev1.record(stream)
        ev1.synchronize()
        total += ev0.elapsed_time(ev1)
    return total / steps


def kernel_roofline(w, prof, steps, peaks, peaks_kind, alu, alu_kind) -> dict:
    """The dominant kernel class of a prefill step (by measured time, summed over the
    step's launches) against the measured bf16 tensor peak; secondary fractions
    against the peak of the type it actually computes in."""
    work = prefill_work(w)
    dom = max(("phi", "scan", "output"), key=lambda kk: prof[kk][0])
    dom_ms = prof[dom][0] / steps
    fl = work[dom]["flops"]
    achieved = fl / (dom_ms / 1e3) / 1e12
    peak = peaks["bf16_tflops"]
    tf32 = peak * NOMINAL_DENSE_PFLOPS["tf32"] / NOMINAL_DENSE_PFLOPS["bf16"]
    return {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "peak_kind": f"{peaks_kind} bf16 dense (burst)",
            "traffic": traffic_for(dom, w.name), "flops_per_step": fl, "kernel_ms_per_step": dom_ms,
            "launches_per_step": prof[dom][1] / steps,
            "secondary": {"tf32_peak": tf32, "tf32_frac": achieved / tf32,
                          "tf32_peak_kind": f"{peaks_kind} bf16 x nominal tf32/bf16 ratio "
                                            f"({NOMINAL_DENSE_PFLOPS['tf32']}/{NOMINAL_DENSE_PFLOPS['bf16']})",
                          "fp32_alu_peak": alu, "fp32_alu_frac": achieved / alu, "fp32_alu_peak_kind": alu_kind}}


def prefill_leg(w, dev, steps, warmup, flush, stream, peaks, barrier, ranks_max, keep=False):
    """Time the reset + prefill step of workload w; returns (summary, profile, layer state)."""
    import sparse_kv_caching_b200 as lola
    full = synth.full_arrays(w)
    q, k, v, W = (_to_dev(full[x], dev) for x in ("q", "k", "v", "W"))
    cfg = lola.make_config(w.B, w.Hq, w.Hkv, w.d, w.Dh, w.eta, w.lam, w.chunk, w.dtype, w.T)
    layer = lola.LolaLayer(cfg, W, device=dev)
    import torch
    y = torch.empty((w.B, w.T, w.Hq, w.d), dtype=torch.float32, device=dev)
    for _ in range(warmup):
        layer.reset()
        layer.prefill(q, k, v, y)
    barrier()
    layer.profile(True)
    l0 = lola.launch_count()
    ms = ranks_max(_timed_prefills(layer, q, k, v, y, flush, steps, stream))
    launches = lola.launch_count() - l0
    barrier()
    prof = layer.profile_read()
    layer.profile(False)
    layer.check()
    summary = {"workload": w.name, "ms_per_step": ms, "tokens_per_s": w.B * w.T / (ms / 1e3),
               "layer_roofline": layer_roofline(w, ms, peaks),
               "kernel_ms_per_step": {kk: round(prof[kk][0] / steps, 4) for kk in ("phi", "scan", "output",
                                                                                   "finalize")},
               "gpu_launches_per_step": launches / steps}
    state = dict(layer=layer, q=q, k=k, v=v, y=y, full=full) if keep else None
    if not keep:
        layer.close()
        del layer, q, k, v, W, y
    return summary, prof, launches, state


def next_legs(st, w, flush, stream, alu, alu_kind):
    """Analysis and ablation legs (stored-pair SRE map, alternative scoring rules,
    read-branch masks) on workload w, reusing its layer."""
    import torch
    import sparse_kv_caching_b200 as lola
    layer, q, k, v, y = st["layer"], st["q"], st["k"], st["v"], st["y"]
    out = {}
    layer.reset()
    layer.prefill(q, k, v, y)
    sre_buf, rel_buf = layer.sre_map(k, v)
    for _ in range(2):
        layer.sre_map(k, v, sre_buf, rel_buf)
    layer.profile(True)
    for _ in range(5):
        flush.zero_()
        layer.sre_map(k, v, sre_buf, rel_buf)
    pm = layer.profile_read()["sre_map"]
    layer.profile(False)
    map_ms = pm[0] / max(1, pm[1])
    map_pairs, map_fl = sre_map_work(w)
    out["sre_map"] = {"workload": w.name, "ms_per_launch": map_ms, "pairs_per_launch": map_pairs,
                      "roofline": {"bound": "alu", "kernel": "sre_map",
                                   "achieved": map_fl / (map_ms / 1e3) / 1e12, "peak": alu, "unit": "TFLOP/s",
                                   "frac": map_fl / (map_ms / 1e3) / 1e12 / alu, "peak_kind": alu_kind,
                                   "flops_per_launch": map_fl, "traffic": traffic_for("sre_map", w.name)}}
    del sre_buf, rel_buf
    scorer_lines = {}
    for rule in lola.SCORERS[1:]:
        layer.reset()
        layer.set_scorer(rule)
        for _ in range(2):
            layer.reset()
            layer.prefill(q, k, v, y)
        layer.profile(True)
        sc_ms = _timed_prefills(layer, q, k, v, y, flush, 3, stream)
        ps = layer.profile_read()
        layer.profile(False)
        ks_ms = ps["scores"][0] / max(1, ps["scores"][1])
        ks_fl = scorer_work(w)
        scorer_lines[rule] = {"ms_per_step": sc_ms, "tokens_per_s": w.B * w.T / (sc_ms / 1e3),
                              "window_score_ms": ks_ms, "chain_ms": ps["scan"][0] / max(1, ps["scan"][1]),
                              "window_score_roofline": {"bound": "alu", "achieved": ks_fl / (ks_ms / 1e3) / 1e12,
                                                        "peak": alu, "unit": "TFLOP/s",
                                                        "frac": ks_fl / (ks_ms / 1e3) / 1e12 / alu,
                                                        "flops_per_launch": ks_fl,
                                                        "traffic": traffic_for("scores", w.name)}}
    layer.reset()
    layer.set_scorer("sre")
    out["scorers"] = scorer_lines
    mask_lines = {}
    for mask, label in ((1, "hide_state"), (2, "hide_sparse"), (3, "window_only")):
        layer.set_read_options(mask)
        for _ in range(2):
            layer.reset()
            layer.prefill(q, k, v, y)
        m_ms = _timed_prefills(layer, q, k, v, y, flush, 3, stream)
        mask_lines[label] = {"ms_per_step": m_ms, "tokens_per_s": w.B * w.T / (m_ms / 1e3)}
    layer.set_read_options(0)
    out["read_masks"] = mask_lines
    layer.check()
    torch.cuda.synchronize()
    return out


def decode_leg(args, dev, peaks, peaks_kind, world, barrier, ranks_max, stream):
    """All 1024 decode steps of the decode workload after its 4096-token prefill,
    once untimed (warm-up) and once timed from a fresh prefill."""
    import torch
    import sparse_kv_caching_b200 as lola
    wd = synth.workload(4) if args.decode_batch is None else synth.workload(4, B=args.decode_batch)
    fd = synth.full_arrays(wd)
    qd, kd, vd, Wd = (_to_dev(fd[x], dev) for x in ("q", "k", "v", "W"))
    del fd
    cfgd = lola.make_config(wd.B, wd.Hq, wd.Hkv, wd.d, wd.Dh, wd.eta, wd.lam, wd.chunk, wd.dtype, wd.T)
    ld = lola.LolaLayer(cfgd, Wd, device=dev)
    pre = (qd[:, :wd.T].contiguous(), kd[:, :wd.T].contiguous(), vd[:, :wd.T].contiguous())
    n = wd.decode_steps
    steps = [(qd[:, t].contiguous(), kd[:, t].contiguous(), vd[:, t].contiguous())
             for t in range(wd.T, wd.T + n)]
    yd = torch.empty((wd.B, wd.Hq, wd.d), dtype=torch.float32, device=dev)
    ld.prefill(*pre)
    for i in range(n):                            # warm-up: the whole decode run once
        ld.decode(*steps[i], yd)
    ld.reset()
    ld.prefill(*pre)
    barrier()
    ld.profile(True)
    l0 = lola.launch_count()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(n):
        ld.decode(*steps[i], yd)
    ev1.record(stream)
    ev1.synchronize()
    launches = lola.launch_count() - l0
    dms = ranks_max(ev0.elapsed_time(ev1) / n)
    pd = ld.profile_read()
    ld.profile(False)
    ld.check()
    kms = pd["decode"][0] / max(1, pd["decode"][1])
    by = decode_step_bytes(wd)
    line = {"workload": wd.name, "value": wd.B * world / (dms / 1e3), "unit": "tokens/s", "ms_per_step": dms,
            "steps": n, "B": wd.B, "context": f"{wd.T} prefilled, then all {n} decode steps timed",
            "l2": "per-step working set above L2 (126 MB)",
            "gpu_launches": launches,
            "roofline": {"bound": "hbm", "kernel": "decode", "achieved": by / (kms / 1e3) / 1e9,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": by / (kms / 1e3) / 1e9 / peaks["hbm_gbs"],
                         "bytes_per_launch": by, "ms_per_launch": kms,
                         "peak_kind": f"{peaks_kind} HBM copy", "traffic": traffic_for("decode", wd.name)},
            "flops_per_step": decode_step_flops(wd)}
    # the same sequences again, the first 50 steps with update-first decode
    ld.reset()
    ld.prefill(*pre)
    ld.set_read_options(0, True)
    n_uf = min(50, n)
    ev0.record(stream)
    for i in range(n_uf):
        ld.decode(*steps[i], yd)
    ev1.record(stream)
    ev1.synchronize()
    uf_ms = ranks_max(ev0.elapsed_time(ev1) / n_uf)
    line["update_first"] = {"ms_per_step": uf_ms, "value": wd.B * world / (uf_ms / 1e3), "steps": n_uf}
    ld.check()
    ld.close()
    del ld, qd, kd, vd, steps, pre
    torch.cuda.empty_cache()
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="lola", choices=["lola", "reference"])
    ap.add_argument("--workload", type=int, default=3)
    ap.add_argument("--extra", default="2,5", help="further prefill workloads reported under 'workloads'")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the headline workload's batch (reduced cases for profiler captures)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the headline workload's prefill length (a multiple of its chunk)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-next", action="store_true", help="skip the SRE-map, scoring-rule and read-mask legs")
    ap.add_argument("--cpu-streams", type=int, default=None,
                    help="streams of the cpu_baseline oracle sample (default: one per host core)")
    ap.add_argument("--sweep", action="store_true", help="single-layer latency over the (eta, lambda) grid")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="sequences of the decode leg (default: the workload's 64; smaller for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.sweep:
        return run_sweep(args)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    over = {k: v for k, v in (("B", args.batch), ("T", args.tokens)) if v is not None}
    w = synth.workload(args.workload, **over)
    if over:
        w = replace(w, name=w.name + "-reduced-" + "-".join(f"{k}{v}" for k, v in over.items()))
    if args.impl == "reference":
        return run_reference(args, w, rank)

    import torch
    import torch.distributed as dist
    import sparse_kv_caching_b200 as lola
    from datetime import timedelta

    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def ranks_max(x: float) -> float:
        return max_over_ranks(x, world, dev)

    peaks, peaks_kind = load_peaks()
    sm_mhz = float(peaks.get("sm_max_mhz", SM_MAX_MHZ_DEFAULT))
    props = torch.cuda.get_device_properties(dev)
    gpu_uuid = None
    try:
        gpu_uuid = "GPU-" + str(props.uuid)
    except Exception:
        pass
    alu = fp32_alu_peak_tflops(props.multi_processor_count, sm_mhz)
    alu_kind = (f"derived fp32 FMA: {props.multi_processor_count} SMs x 128 lanes x 2 FLOP x {sm_mhz:.0f} MHz "
                f"({'measured' if 'sm_max_mhz' in peaks else 'default'} max SM clock)")
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)   # > L2 (126 MB)

    # ---- headline prefill workload (timed with the clocks sampled) -------------
    clocks = ClockSampler(gpu_uuid)
    clocks.start()
    head, prof, launches, st = prefill_leg(w, dev, args.steps, args.warmup, flush, stream, peaks, barrier,
                                           ranks_max, keep=True)
    clk = clocks.stop()
    ms_step = head["ms_per_step"]
    value = job_throughput(w.B * w.T, world, ms_step)
    roofline = kernel_roofline(w, prof, args.steps, peaks, peaks_kind, alu, alu_kind)
    shares = {kk: round(prof[kk][0] / max(1e-9, sum(p[0] for p in prof.values())), 4)
              for kk in ("phi", "scan", "output", "finalize", "decode")}
    layer, full = st["layer"], st["full"]
    # ---- e2e through the host-buffer entry point ------------------------------
    hq, hk, hv = (torch.from_numpy(full[x].view(np.int16) if full[x].dtype == np.uint16 else full[x])
                  .pin_memory() for x in ("q", "k", "v"))
    if w.dtype == "bf16":
        hq, hk, hv = (x.view(torch.bfloat16) for x in (hq, hk, hv))
    hy = torch.empty((w.B, w.T, w.Hq, w.d), dtype=torch.float32).pin_memory()
    e2e_steps = max(3, min(args.steps, 5))
    for _ in range(2):
        layer.reset()
        layer.prefill_host(hq, hk, hv, hy)
    barrier()
    e2e_ms = 0.0
    for _ in range(e2e_steps):
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        layer.reset()
        layer.prefill_host(hq, hk, hv, hy)
        ev1.record(stream)
        ev1.synchronize()
        e2e_ms += ev0.elapsed_time(ev1)
    e2e_ms = ranks_max(e2e_ms / e2e_steps)
    h2d = hq.numel() * hq.element_size() + hk.numel() * hk.element_size() + hv.numel() * hv.element_size()
    d2h = hy.numel() * 4
    # y and trace of a device-path step, for the oracle match
    layer.reset()
    layer.prefill(st["q"], st["k"], st["v"], st["y"])
    layer.check()
    ex = layer.export()
    trace = ex["trace_pos"].cpu().numpy() if w.lam > 0 else None
    y_host = st["y"].cpu()
    layer.close()
    del layer, st, full, hq, hk, hv, hy, ex
    torch.cuda.empty_cache()

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": DTYPE, "precisions": PRECISIONS, "data": "synthetic",
            "config": workload_config(w, world),
            "roofline": roofline,
            "layer_roofline": head["layer_roofline"],
            "kernel_time_share": shares,
            "kernel_ms_per_step": head["kernel_ms_per_step"],
            "gpu_launches": launches,
            "clocks": clk,
            "e2e": {"value": job_throughput(w.B * w.T, world, e2e_ms), "unit": "tokens/s", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            }

    # ---- further prefill workloads, then the analysis / ablation legs on the 4K one ----
    extra = [int(x) for x in args.extra.split(",") if x.strip()] if args.extra else []
    line["workloads"] = {}
    for wid in extra:
        if wid == args.workload:
            continue
        we = synth.workload(wid)
        keep = wid == 2 and not args.no_next
        summ, prof_e, _, st_e = prefill_leg(we, dev, max(3, args.steps // 2), args.warmup, flush, stream, peaks,
                                            barrier, ranks_max, keep=keep)
        summ["roofline"] = kernel_roofline(we, prof_e, max(3, args.steps // 2), peaks, peaks_kind, alu, alu_kind)
        summ["value"] = job_throughput(we.B * we.T, world, summ["ms_per_step"])
        line["workloads"][we.name] = summ
        if keep:
            line["next"] = next_legs(st_e, we, flush, stream, alu, alu_kind)
            st_e["layer"].close()
            del st_e
            torch.cuda.empty_cache()

    # ---- decode workload ----------------------------------------------------
    if not args.no_decode:
        line["decode"] = decode_leg(args, dev, peaks, peaks_kind, world, barrier, ranks_max, stream)

    # ---- cpu_baseline: the oracle on a bounded sample, plus the oracle match ----
    if rank == 0:
        cores = host_cores()
        nstreams = min(w.B * w.Hkv, args.cpu_streams or cores)
        streams = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
        # spread the sample over the batch and the kv heads, first and last stream included
        idx = sorted({round(i * (len(streams) - 1) / max(1, nstreams - 1)) for i in range(nstreams)})
        sample = [streams[i] for i in idx]
        n, secs, done, match = oracle_sample(w, sample, min(len(sample), cores), gpu=(y_host, trace))
        line["cpu_baseline"] = {"value": n / secs, "unit": "tokens/s", "cores": min(len(sample), cores),
                                "kind": "oracle", "cpu": cpu_model(), "host_cores": cores,
                                "sample": f"{done} whole (sequence, kv head) streams of {w.T} tokens "
                                          f"(= {n:.0f} layer tokens), one per core in parallel, {secs:.1f} s wall",
                                "oracle_match": match}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
