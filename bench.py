#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  1. fa_fwd on the long sliding-window shape (B=1, H=16, Nq=Nk=16384,
     d=128, bf16, causal, window_left=4096): the N >= 8K, d = 128 forward
     the throughput target is stated for;
  2. fa_fwd_kvcache on the paged decode batch (B=64, H=32, d=128, bf16,
     pages of 256 tokens, lengths U[1024, 32768], automatic split count):
     split kernel + merge kernel.
The headline value is the forward's TFLOP/s (4*d*H*B*(unmasked query/key
pairs) per launch over its CUDA-event time); the decode's KV GB/s
(2*2*H*d bytes per cached token over the call's time) is reported beside it.
Both inputs exceed the 126 MB L2 (forward Q+K+V 201 MB, decode K/V 34 GB),
so no explicit flush is needed between iterations. After the timed steps
every forward workload of the suite (causal 2K, window 16K, window and causal
Nq 4K / Nk 16K, ALiBi + softcap) is timed on its own with L2 flushed between
launches and reported under "forward_configs", and the backward pass (causal
2K in both dQ modes, window 16K, ALiBi + softcap) under "backward_configs".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
  python bench.py --sweep          # every forward workload and decode split
                                   # count, one JSON line each (L2 flushed)

With N > 1 (launched by torch.distributed.run) every rank runs its own
replica of the step (the path has no exchange step); value counts all ranks'
work over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import math
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

from exact_io_aware_79_b200 import workloads as W  # noqa: E402

METRIC = "attn fwd TFLOP/s (% of BF16 peak); paged-decode KV GB/s (% of HBM BW)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# ncu captures of the kernels as they stand.
# Decode: a capture of the split kernel on the 4-sequence case (B=4, H=32,
# d=128, pages of 256) read 1.003 x its K/V bytes and wrote 2.8 MB of
# partials; reads scale with the K/V bytes, each byte being read once.
DECODE_READ_PER_KV_BYTE = 967959936.0 / 965165056.0  # (968,019,712 + 967,900,160) / 2 / K/V bytes
# Forward: per-launch DRAM bytes of ncu captures of the forward kernel as it
# stands, on the named workload; a workload without such a capture reports
# None.
FWD_TRAFFIC = {W.WINDOW_16K.name: 201669888.0 + 48675840.0}
# Backward workloads timed after the step (atomic dQ, and the deterministic
# mode on the first); credited 2.5 x the forward's flops (five products of
# the forward's size against two).
BWD_CONFIGS = [W.CAUSAL_2K, W.WINDOW_16K, W.ALIBI_SOFTCAP]
# Forward workloads timed one by one after the step (L2 flushed between launches).
FWD_CONFIGS = [W.CAUSAL_2K, W.WINDOW_16K, W.WINDOW_Q4K_K16K, W.CAUSAL_Q4K_K16K, W.ALIBI_SOFTCAP]
HEADLINE_FWD = W.WINDOW_16K
# The 8-bit forward, timed the same way on these workloads' shapes (E4M3
# inputs with per-tensor descales); its roofline is the fp8 tensor peak,
# taken as twice the measured bf16 burst (the nominal dense fp8 / bf16 ratio).
FP8_CONFIGS = [W.WINDOW_16K]
FP8_OVER_BF16 = 2.0


# ---------------------------------------------------------------- algorithmic work

def unmasked_pairs(w: W.FwdWorkload) -> int:
    """Query/key pairs that survive the mask, per (batch, head): sum over
    rows of the visible interval length (interval arithmetic, no oracle)."""
    return int(visible_keys_per_row(w).sum())


def visible_keys_per_row(w: W.FwdWorkload) -> np.ndarray:
    """Number of keys each query row sees (interval arithmetic)."""
    i = np.arange(w.Nq, dtype=np.int64)
    pos = i + w.Nk - w.Nq
    lo = np.zeros_like(i) if w.window_left < 0 else np.maximum(0, pos - w.window_left)
    hi = np.full_like(i, w.Nk - 1)
    if w.causal:
        hi = np.minimum(hi, pos)
    if w.window_right >= 0:
        hi = np.minimum(hi, pos + w.window_right)
    return np.maximum(0, hi - lo + 1)


def fwd_flops(w: W.FwdWorkload) -> float:
    return 4.0 * w.d * w.B * w.H * unmasked_pairs(w)


def varlen_flops(w: W.VarlenWorkload, lens) -> float:
    """4*d*H*(visible query/key pairs) summed over the packed sequences
    (query and key lengths equal; causal: n(n+1)/2 pairs)."""
    n = np.asarray(lens, dtype=np.int64)
    pairs = n * (n + 1) // 2 if w.causal else n * n
    return 4.0 * w.d * w.H * float(pairs.sum())


def decode_kv_bytes(w: W.DecodeWorkload, seqlens: torch.Tensor) -> float:
    L = seqlens.to(torch.int64)
    if w.window_left >= 0:
        L = torch.clamp(L, max=w.window_left + 1)
    return 2.0 * 2.0 * w.kv_heads * w.d * float(L.sum())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks

CLOCK_FIELDS = ["timestamp", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
                "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
                "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
REASON_NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


class ClockSampler:
    """nvidia-smi sampled every 50 ms in the background; samples are tagged
    with host time so the timed region's samples can be picked out."""

    def __init__(self, gpu_index: str):
        self.samples = []
        self.proc = None
        self.gpu = gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, "--query-gpu=" + ",".join(CLOCK_FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True, bufsize=1)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == len(CLOCK_FIELDS):
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        inside = [p for (t, p) in self.samples if t0 <= t <= t1]
        if not inside:
            inside = [p for (t, p) in self.samples]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(p[1]) for p in inside if p[1].replace(".", "").isdigit()]
        smax = [float(p[2]) for p in inside if p[2].replace(".", "").isdigit()]
        reasons = set()
        for p in inside:
            for name, val in zip(REASON_NAMES, p[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        power = [float(p[3]) for p in inside if p[3].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(inside),
                "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------- distributed plumbing

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(world: int, backend: str = "nccl"):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, max_seconds: float, world: int) -> float:
    """Whole-job throughput of N independent replicas: every rank processes
    units_per_rank, and the job takes the slowest rank's time."""
    return world * units_per_rank / max_seconds


def physical_gpu(local: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local < len(ids):
            return ids[local]
    return str(local)


# ---------------------------------------------------------------- CPU oracle baseline

def oracle_fwd_sample(w: W.FwdWorkload, x, budget_s: float):
    """Times the oracle on a growing sample of query rows (all batches and
    heads) until about budget_s of CPU work; returns (TFLOP/s, rows, seconds)."""
    import oracle
    vis = visible_keys_per_row(w)
    n = 2
    rng = np.random.default_rng(0)
    while True:
        rows = np.sort(rng.choice(w.Nq, size=min(n, w.Nq), replace=False))
        t0 = time.perf_counter()
        oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.window_left, w.window_right, x["slopes"],
                        w.softcap, rows=rows.tolist())
        dt = time.perf_counter() - t0
        flops = 4.0 * w.d * w.B * w.H * float(vis[rows].sum())
        if dt >= budget_s * 0.4 or len(rows) >= w.Nq:
            return flops / dt / 1e12, len(rows), dt
        n = int(min(w.Nq, max(n * 2, n * budget_s / max(dt, 1e-3) * 0.8)))


def oracle_decode_sample(w: W.DecodeWorkload, xd, budget_s: float, max_seqs: int = 6):
    """Times the oracle's paged decode on a sample of at most max_seqs
    sequences (all heads; their pages are copied to host memory first),
    repeating the sample until about budget_s of CPU work; returns
    (GB/s of K/V, sequences, seconds)."""
    import oracle
    lens = xd["cache_seqlens"].cpu()
    table = xd["block_table"].cpu()
    picks = torch.randperm(w.B, generator=torch.Generator().manual_seed(1))[:max_seqs].tolist()
    used = sorted({int(p) for b in picks for p in table[b, :(int(lens[b]) + w.page_size - 1) // w.page_size]})
    remap = {p: i for i, p in enumerate(used)}
    idx = torch.tensor(used, device=xd["k_cache"].device)
    kc = xd["k_cache"].index_select(0, idx).cpu()
    vc = xd["v_cache"].index_select(0, idx).cpu()
    sub = torch.zeros(len(picks), w.max_blocks, dtype=torch.int32)
    for r, b in enumerate(picks):
        nb = (int(lens[b]) + w.page_size - 1) // w.page_size
        sub[r, :nb] = torch.tensor([remap[int(p)] for p in table[b, :nb]], dtype=torch.int32)
    q = xd["q"][picks].cpu()
    nbytes = decode_kv_bytes(w, lens[picks])
    total_t, total_b, reps = 0.0, 0.0, 0
    while total_t < budget_s * 0.5 or reps == 0:
        t0 = time.perf_counter()
        oracle.attn_decode_paged(q, kc, vc, sub, lens[picks], w.scale, w.window_left, None, w.softcap)
        total_t += time.perf_counter() - t0
        total_b += nbytes
        reps += 1
    return total_b / total_t / 1e9, "%d x %d" % (reps, len(picks)), total_t


# ---------------------------------------------------------------- GPU arm

def gpu_arm(args):
    import exact_io_aware_79_b200 as fa
    fa.library()  # fail loudly if the CUDA library is missing
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dist_init(world)
    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()

    fw = HEADLINE_FWD
    dw = W.DECODE
    x = W.make_fwd_inputs(fw, device=dev)
    xd = W.make_decode_inputs(dw, device=dev)
    out = torch.empty_like(x["q"])
    lse = torch.empty((fw.B, fw.H, fw.Nq), dtype=torch.float32, device=dev)
    d_out = torch.empty_like(xd["q"])
    d_lse = torch.empty((dw.B, dw.H, 1), dtype=torch.float32, device=dev)
    splits = fa.fa_kvcache_num_splits(dw.B, dw.H, dw.d, dw.max_blocks, dw.page_size, 0)
    ws_bytes = fa.fa_kvcache_workspace_size(dw.B, dw.H, dw.d, dw.max_blocks, dw.page_size, 0)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    F = fwd_flops(fw)
    KVB = decode_kv_bytes(dw, xd["cache_seqlens"].cpu())
    launches_per_step = 1 + (2 if splits > 1 else 1)

    def run_fwd(q, k, v, o, l):
        fa.fa_fwd(q, k, v, o, l, fw.scale, fw.causal, fw.window_left, fw.window_right, None, fw.softcap)

    def run_dec(q, bt, sl, o, l):
        fa.fa_fwd_kvcache(q, xd["k_cache"], xd["v_cache"], bt, sl, o, l, dw.scale, dw.window_left, None,
                          dw.softcap, 0, ws)

    ev = lambda: torch.cuda.Event(enable_timing=True)
    K, Wu = args.steps, args.warmup
    for _ in range(Wu):
        run_fwd(x["q"], x["k"], x["v"], out, lse)
        run_dec(xd["q"], xd["block_table"], xd["cache_seqlens"], d_out, d_lse)
    torch.cuda.synchronize()

    sampler = ClockSampler(physical_gpu(local))
    sampler.start()
    time.sleep(0.3)
    fe = [(ev(), ev()) for _ in range(K)]
    de = [(ev(), ev()) for _ in range(K)]
    r0, r1 = ev(), ev()
    barrier(world)
    torch.cuda.synchronize()
    t_host0 = time.time()
    r0.record()
    for s in range(K):
        fe[s][0].record()
        run_fwd(x["q"], x["k"], x["v"], out, lse)
        fe[s][1].record()
        de[s][0].record()
        run_dec(xd["q"], xd["block_table"], xd["cache_seqlens"], d_out, d_lse)
        de[s][1].record()
    r1.record()
    torch.cuda.synchronize()
    barrier(world)
    t_host1 = time.time()
    time.sleep(0.2)
    sampler.stop()
    clocks = sampler.summary(t_host0, t_host1)

    region_ms = max_over_ranks(r0.elapsed_time(r1), world, dev)
    fwd_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in fe) / K, world, dev)
    dec_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in de) / K, world, dev)
    fwd_tflops = weak_scaling_value(F, fwd_ms * 1e-3, world) / 1e12
    dec_gbs = weak_scaling_value(KVB, dec_ms * 1e-3, world) / 1e9

    # ---- every forward workload on its own (L2 flushed between launches)
    fwd_configs = time_fwd_configs(fa, dev, world, peaks, args, physical_gpu(local))
    # ---- the backward pass on its workloads (L2 flushed between calls)
    bwd_configs = time_bwd_configs(fa, dev, world, peaks, args, physical_gpu(local))

    # ---- end to end through the public API with pinned host buffers
    hq, hk, hv = (x[n].cpu().pin_memory() for n in ("q", "k", "v"))
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h_lse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    hdq = xd["q"].cpu().pin_memory()
    hbt = xd["block_table"].cpu().pin_memory()
    hsl = xd["cache_seqlens"].cpu().pin_memory()
    h_dout = torch.empty(d_out.shape, dtype=d_out.dtype).pin_memory()
    h_dlse = torch.empty(d_lse.shape, dtype=d_lse.dtype).pin_memory()
    # forward leg: a copy stream uploads step s + 1's q, k, v into the other of
    # two device buffer sets while the compute stream runs step s and reads
    # its O and LSE back (copies in both directions overlap the kernels, as a
    # serving pipeline would); every step's copies are inside the timed region
    gin = [tuple(torch.empty_like(x[n]) for n in ("q", "k", "v")) for _ in range(2)]
    gdq, gbt, gsl = torch.empty_like(xd["q"]), torch.empty_like(xd["block_table"]), torch.empty_like(
        xd["cache_seqlens"])
    Ke = max(3, min(K, args.e2e_steps))
    comp = torch.cuda.current_stream()
    copy = torch.cuda.Stream()

    def e2e_fwd(steps, t0, t1):
        up = [torch.cuda.Event() for _ in range(steps)]
        used = [torch.cuda.Event() for _ in range(steps)]
        t0.record(comp)
        copy.wait_stream(comp)
        for s in range(steps):
            with torch.cuda.stream(copy):
                if s >= 2:
                    copy.wait_event(used[s - 2])  # the kernel of step s - 2 is done with this buffer set
                for dst, src in zip(gin[s % 2], (hq, hk, hv)):
                    dst.copy_(src, non_blocking=True)
                up[s].record(copy)
            comp.wait_event(up[s])
            run_fwd(*gin[s % 2], out, lse)
            used[s].record(comp)
            h_out.copy_(out, non_blocking=True)
            h_lse.copy_(lse, non_blocking=True)
        t1.record(comp)

    def e2e_dec(ed):
        ed[0].record()
        gdq.copy_(hdq, non_blocking=True)
        gbt.copy_(hbt, non_blocking=True)
        gsl.copy_(hsl, non_blocking=True)
        run_dec(gdq, gbt, gsl, d_out, d_lse)
        h_dout.copy_(d_out, non_blocking=True)
        h_dlse.copy_(d_lse, non_blocking=True)
        ed[1].record()

    e2e_fwd(2, ev(), ev())
    for _ in range(2):
        e2e_dec((ev(), ev()))
    torch.cuda.synchronize()
    ef0, ef1 = ev(), ev()
    ede = [(ev(), ev()) for _ in range(Ke)]
    barrier(world)
    torch.cuda.synchronize()
    e2e_fwd(Ke, ef0, ef1)
    for s in range(Ke):
        e2e_dec(ede[s])
    torch.cuda.synchronize()
    barrier(world)
    e_fwd_ms = max_over_ranks(ef0.elapsed_time(ef1) / Ke, world, dev)
    e_dec_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ede) / Ke, world, dev)
    fwd_h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    fwd_d2h = sum(t.numel() * t.element_size() for t in (h_out, h_lse))
    dec_h2d = sum(t.numel() * t.element_size() for t in (hdq, hbt, hsl))
    dec_d2h = sum(t.numel() * t.element_size() for t in (h_dout, h_dlse))

    # ---- CPU oracle baseline (rank 0, single GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        xf_cpu = {k2: (None if t is None else t.cpu()) for k2, t in x.items()}
        v_f, rows, t_f = oracle_fwd_sample(fw, xf_cpu, args.cpu_budget)
        v_d, seqs, t_d = oracle_decode_sample(dw, xd, args.cpu_budget)
        cpu = {"value": v_f, "unit": "TFLOP/s", "cores": oracle.max_threads(), "kind": "oracle",
               "sample": "forward: %d of %d query rows, all %d (batch, head) pairs, %.1f s; credited "
                         "flops = 4*d*visible keys of the sampled rows" % (rows, fw.Nq, fw.B * fw.H, t_f),
               "decode": {"value": v_d, "unit": "GB/s",
                          "sample": "%s (repeats x sequences) of %d sequences, all heads, %.1f s; credited "
                                    "bytes = K+V of the sampled sequences" % (seqs, dw.B, t_d)}}

    # the forward is one sub-millisecond launch inside the step, so its
    # roofline is the burst tensor peak
    peak_t = peaks["bf16_tflops"]
    peak_h = peaks["hbm_gbs"]
    result = {
        "metric": METRIC,
        "value": round(fwd_tflops, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": Wu,
        "ms_per_step": round(region_ms / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": "%s + %s" % (fw.name, dw.name),
            "forward": {"B": fw.B, "H": fw.H, "Nq": fw.Nq, "Nk": fw.Nk, "d": fw.d, "causal": fw.causal,
                        "flops_per_launch": F},
            "decode": {"B": dw.B, "H": dw.H, "d": dw.d, "page_size": dw.page_size,
                       "seqlens": [dw.len_lo, dw.len_hi], "num_splits": splits, "kv_bytes_per_launch": KVB},
            "l2": "step: inputs larger than L2 (forward Q+K+V 201 MB, decode K/V 34 GB), no flush; "
                  "forward_configs, backward_configs: L2 flushed (256 MB write) before every call",
            "parallelism": "replicas" if world > 1 else "single GPU",
        },
        "roofline": {"kernel": "decode (split + merge)", "bound": "hbm", "achieved": round(dec_gbs / world, 1),
                     "peak": peak_h, "unit": "GB/s", "frac": round(dec_gbs / world / peak_h, 4),
                     "traffic": round(DECODE_READ_PER_KV_BYTE * KVB),
                     "traffic_source": "ncu capture of the 4-sequence case, scaled by K/V bytes",
                     "peak_source": peak_src},
        "roofline_fwd": {"kernel": "fwd_kernel", "workload": fw.name, "bound": "tensor",
                         "achieved": round(fwd_tflops / world, 2), "peak": peak_t, "unit": "TFLOP/s",
                         "frac": round(fwd_tflops / world / peak_t, 4),
                         "frac_of_sustained": round(fwd_tflops / world / peaks["bf16_tflops_sustained"], 4),
                         "traffic": round(FWD_TRAFFIC[fw.name]) if FWD_TRAFFIC.get(fw.name) else None,
                         "traffic_source": "ncu capture of this workload",
                         "peak_source": peak_src + " burst"},
        "forward_configs": fwd_configs,
        "backward_configs": bwd_configs,
        "decode": {"value": round(dec_gbs, 1), "unit": "GB/s", "ms_per_launch": round(dec_ms, 4)},
        "fwd_ms_per_launch": round(fwd_ms, 4),
        "e2e": {"value": round(world * F / (e_fwd_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": fwd_h2d + dec_h2d, "d2h_bytes_per_step": fwd_d2h + dec_d2h,
                "note": "forward: q, k, v uploaded from pinned host memory every step on a copy stream, step "
                        "s + 1's upload overlapping step s's kernel and O / LSE read-back (two device input "
                        "sets); time of the whole run of steps on the device / steps",
                "decode": {"value": round(world * KVB / (e_dec_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                           "note": "K/V cache resident in HBM (serving state); per step q, block table "
                                   "and lengths go in, O and LSE come out"}},
        "gpu_launches": K * launches_per_step,
        "clocks": clocks,
    }
    if cpu is not None:
        result["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def time_fwd_configs(fa, dev, world, peaks, args, gpu_index):
    """Times fa_fwd on every workload of FWD_CONFIGS: W warm-up launches, then
    the median of K CUDA-event-timed launches, each after a 256 MB write that
    flushes L2; returns {workload: {ms, TFLOP/s, frac of the burst peak}}
    with the SM clocks seen while they ran."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    res = {}
    sampler = ClockSampler(gpu_index)
    sampler.start()
    t0 = time.time()
    for w in FWD_CONFIGS:
        x = W.make_fwd_inputs(w, device=dev)
        out = torch.empty_like(x["q"])
        lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
        run = lambda: fa.fa_fwd(x["q"], x["k"], x["v"], out, lse, w.scale, w.causal, w.window_left,
                                w.window_right, x["slopes"], w.softcap)
        for _ in range(max(3, args.warmup)):
            run()
        times = []
        n = max(5, min(args.steps, args.config_steps))
        barrier(world)
        for _ in range(n):
            flush.zero_()
            a, b = ev(), ev()
            a.record()
            run()
            b.record()
            times.append((a, b))
        torch.cuda.synchronize()
        ms = max_over_ranks(statistics.median([a.elapsed_time(b) for a, b in times]), world, dev)
        tf = weak_scaling_value(fwd_flops(w), ms * 1e-3, world) / 1e12
        res[w.name] = {"ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                       "frac": round(tf / world / peaks["bf16_tflops"], 4), "flops_per_launch": fwd_flops(w),
                       "launches": n}
        del x, out, lse
    for w in FP8_CONFIGS:
        x = W.make_fwd_inputs_fp8(w, device=dev)
        out = torch.empty(x["q"].shape, dtype=torch.bfloat16, device=dev)
        lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
        ws = torch.empty(max(fa.fa_fwd_fp8_workspace_size(w.B, w.H, w.Nk, w.d), 16), dtype=torch.uint8, device=dev)
        run = lambda: fa.fa_fwd_fp8(x["q"], x["k"], x["v"], out, lse, w.scale, x["descale_q"], x["descale_k"],
                                    x["descale_v"], w.causal, w.window_left, w.window_right, x["slopes"], w.softcap,
                                    ws)
        for _ in range(max(3, args.warmup)):
            run()
        times = []
        n = max(5, min(args.steps, args.config_steps))
        barrier(world)
        for _ in range(n):
            flush.zero_()
            a, b = ev(), ev()
            a.record()
            run()
            b.record()
            times.append((a, b))
        torch.cuda.synchronize()
        ms = max_over_ranks(statistics.median([a.elapsed_time(b) for a, b in times]), world, dev)
        tf = weak_scaling_value(fwd_flops(w), ms * 1e-3, world) / 1e12
        res["fp8_e4m3_" + w.name] = {"ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                                     "frac": round(tf / world / (FP8_OVER_BF16 * peaks["bf16_tflops"]), 4),
                                     "frac_of_bf16_burst": round(tf / world / peaks["bf16_tflops"], 4),
                                     "flops_per_launch": fwd_flops(w), "launches": n,
                                     "note": "includes the V transpose pre-pass"}
        del x, out, lse, ws
    t1 = time.time()
    sampler.stop()
    res["peak"] = "measured burst bf16 %.1f TFLOP/s (fp8: %.0f x that)" % (peaks["bf16_tflops"], FP8_OVER_BF16)
    res["clocks"] = sampler.summary(t0, t1)
    del flush
    return res


def time_bwd_configs(fa, dev, world, peaks, args, gpu_index):
    """Times fa_bwd (row-dot kernel, the key-block kernel, and the dQ cast or
    the deterministic dQ pass) on BWD_CONFIGS like time_fwd_configs: L2
    flushed before each timed call, median of the CUDA-event times."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    res = {}
    sampler = ClockSampler(gpu_index)
    sampler.start()
    t0 = time.time()
    for i, w in enumerate(BWD_CONFIGS):
        x = W.make_fwd_inputs(w, device=dev)
        gen = torch.Generator().manual_seed(w.seed + 100)
        dout = torch.randn(x["q"].shape, generator=gen).to(w.dtype).to(dev)
        out = torch.empty_like(x["q"])
        lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
        fa.fa_fwd(x["q"], x["k"], x["v"], out, lse, w.scale, w.causal, w.window_left, w.window_right,
                  x["slopes"], w.softcap)
        dq, dk, dv = torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"])
        ws = torch.empty(max(fa.fa_bwd_workspace_size(w.B, w.H, w.Nq, w.d), 16), dtype=torch.uint8, device=dev)
        for det in ((False, True) if i == 0 else (False,)):
            run = lambda: fa.fa_bwd(x["q"], x["k"], x["v"], out, lse, dout, dq, dk, dv, w.scale, w.causal,
                                    w.window_left, w.window_right, x["slopes"], w.softcap, deterministic=det,
                                    workspace=ws)
            for _ in range(max(3, args.warmup)):
                run()
            times = []
            n = max(5, min(args.steps, args.config_steps))
            barrier(world)
            for _ in range(n):
                flush.zero_()
                a, b = ev(), ev()
                a.record()
                run()
                b.record()
                times.append((a, b))
            torch.cuda.synchronize()
            ms = max_over_ranks(statistics.median([a.elapsed_time(b) for a, b in times]), world, dev)
            fl = 2.5 * fwd_flops(w)
            tf = weak_scaling_value(fl, ms * 1e-3, world) / 1e12
            res[("deterministic_" if det else "") + w.name] = {
                "ms": round(ms, 4), "TFLOP/s": round(tf, 1), "frac": round(tf / world / peaks["bf16_tflops"], 4),
                "flops_per_call": fl, "launches": n}
        del x, dout, out, lse, dq, dk, dv, ws
    t1 = time.time()
    sampler.stop()
    res["peak"] = "measured burst bf16 %.1f TFLOP/s" % peaks["bf16_tflops"]
    res["clocks"] = sampler.summary(t0, t1)
    del flush
    return res


# ---------------------------------------------------------------- reference arm (the oracle)

def reference_arm(args):
    rank, world, local = dist_env()
    if rank != 0:
        return
    import oracle
    fw = HEADLINE_FWD
    x = W.make_fwd_inputs(fw)
    budget = max(0.3, min(3.0, 150.0 / max(1, args.steps + args.warmup)))
    # size one step's row sample once, then time K steps of it
    _, rows, _ = oracle_fwd_sample(fw, x, budget)
    rng = np.random.default_rng(1)
    vis = visible_keys_per_row(fw)
    times, flops = [], 0.0
    for s in range(args.warmup + args.steps):
        sel = np.sort(rng.choice(fw.Nq, size=rows, replace=False))
        t0 = time.perf_counter()
        oracle.attn_fwd(x["q"], x["k"], x["v"], fw.scale, fw.causal, fw.window_left, fw.window_right, None,
                        fw.softcap, rows=sel.tolist())
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
            flops += 4.0 * fw.d * fw.B * fw.H * float(vis[sel].sum())
    total = sum(times)
    value = flops / total / 1e12
    result = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": 1e3 * total / max(1, len(times)),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": fw.name + " (oracle: sampled query rows)", "rows_per_step": rows,
                   "forward": {"B": fw.B, "H": fw.H, "Nq": fw.Nq, "Nk": fw.Nk, "d": fw.d, "causal": fw.causal}},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": "%d of %d query rows per step, all (batch, head) pairs" % (rows, fw.Nq)},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(result), flush=True)


# ---------------------------------------------------------------- sweep (extra lines)

def sweep(args):
    import exact_io_aware_79_b200 as fa
    fa.library()
    dev = torch.device("cuda", 0)
    peaks, peak_src = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    names = args.workloads.split(",") if args.workloads else [w.name for w in W.FWD_WORKLOADS]
    for w in W.FWD_WORKLOADS:
        if w.name not in names:
            continue
        x = W.make_fwd_inputs(w, device=dev)
        out = torch.empty_like(x["q"])
        lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
        run = lambda: fa.fa_fwd(x["q"], x["k"], x["v"], out, lse, w.scale, w.causal, w.window_left,
                                w.window_right, x["slopes"], w.softcap)
        for _ in range(args.warmup):
            run()
        times = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = ev(), ev()
            a.record()
            run()
            b.record()
            times.append((a, b))
        torch.cuda.synchronize()
        ms = statistics.median([a.elapsed_time(b) for a, b in times])
        tf = fwd_flops(w) / (ms * 1e-3) / 1e12
        print(json.dumps({"workload": w.name, "ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                          "frac_burst": round(tf / peaks["bf16_tflops"], 4),
                          "frac_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
                          "flops": fwd_flops(w), "peak_source": peak_src, "l2": "flushed"}), flush=True)
        del x, out, lse
    # 8-bit forward of a forward workload: "fp8_" + its name (E4M3)
    for w in W.FWD_WORKLOADS:
        if "fp8_" + w.name not in names or w.d != 128:
            continue
        x = W.make_fwd_inputs_fp8(w, device=dev)
        out = torch.empty(x["q"].shape, dtype=torch.bfloat16, device=dev)
        lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
        ws = torch.empty(max(fa.fa_fwd_fp8_workspace_size(w.B, w.H, w.Nk, w.d), 16), dtype=torch.uint8, device=dev)
        run = lambda: fa.fa_fwd_fp8(x["q"], x["k"], x["v"], out, lse, w.scale, x["descale_q"], x["descale_k"],
                                    x["descale_v"], w.causal, w.window_left, w.window_right, x["slopes"], w.softcap,
                                    ws)
        for _ in range(args.warmup):
            run()
        times = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = ev(), ev()
            a.record()
            run()
            b.record()
            times.append((a, b))
        torch.cuda.synchronize()
        ms = statistics.median([a.elapsed_time(b) for a, b in times])
        tf = fwd_flops(w) / (ms * 1e-3) / 1e12
        print(json.dumps({"workload": "fp8_" + w.name, "ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                          "frac_fp8_peak": round(tf / (FP8_OVER_BF16 * peaks["bf16_tflops"]), 4),
                          "frac_bf16_burst": round(tf / peaks["bf16_tflops"], 4),
                          "flops": fwd_flops(w), "peak_source": peak_src, "l2": "flushed"}), flush=True)
        del x, out, lse, ws
    # backward of a forward workload: "bwd_" + its name ("bwd_det_" + its name
    # for the deterministic mode); credited 2.5x the forward's flops (five
    # products of the forward's size against two) in either mode
    for w, det in [(w, det) for w in W.FWD_WORKLOADS for det in (False, True)]:
        label = ("bwd_det_" if det else "bwd_") + w.name
        if label not in names:
            continue
        x = W.make_fwd_inputs(w, device=dev)
        gen = torch.Generator().manual_seed(w.seed + 100)
        dout = torch.randn(x["q"].shape, generator=gen).to(w.dtype).to(dev)
        out = torch.empty_like(x["q"])
        lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
        fa.fa_fwd(x["q"], x["k"], x["v"], out, lse, w.scale, w.causal, w.window_left, w.window_right,
                  x["slopes"], w.softcap)
        dq, dk, dv = torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"])
        ws = torch.empty(max(fa.fa_bwd_workspace_size(w.B, w.H, w.Nq, w.d), 16), dtype=torch.uint8, device=dev)
        run = lambda: fa.fa_bwd(x["q"], x["k"], x["v"], out, lse, dout, dq, dk, dv, w.scale, w.causal,
                                w.window_left, w.window_right, x["slopes"], w.softcap, deterministic=det,
                                workspace=ws)
        for _ in range(args.warmup):
            run()
        times = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = ev(), ev()
            a.record()
            run()
            b.record()
            times.append((a, b))
        torch.cuda.synchronize()
        ms = statistics.median([a.elapsed_time(b) for a, b in times])
        fl = 2.5 * fwd_flops(w)
        tf = fl / (ms * 1e-3) / 1e12
        print(json.dumps({"workload": label, "ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                          "frac_burst": round(tf / peaks["bf16_tflops"], 4),
                          "frac_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
                          "flops": fl, "peak_source": peak_src, "l2": "flushed"}), flush=True)
        del x, out, lse, dout, dq, dk, dv, ws
    vw = W.VARLEN
    if not args.workloads or vw.name in names:
        x = W.make_varlen_inputs(vw, device=dev)
        out = torch.empty_like(x["q"])
        lse = torch.empty((vw.H, x["q"].shape[0]), dtype=torch.float32, device=dev)
        run = lambda: fa.fa_fwd_varlen(x["q"], x["k"], x["v"], out, lse, x["cu_q"], x["cu_k"], x["max_q"],
                                       x["max_k"], vw.scale, vw.causal)
        for _ in range(args.warmup):
            run()
        times = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = ev(), ev()
            a.record()
            run()
            b.record()
            times.append((a, b))
        torch.cuda.synchronize()
        ms = statistics.median([a.elapsed_time(b) for a, b in times])
        fl = varlen_flops(vw, x["lens"])
        tf = fl / (ms * 1e-3) / 1e12
        print(json.dumps({"workload": vw.name, "ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                          "frac_burst": round(tf / peaks["bf16_tflops"], 4),
                          "frac_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
                          "flops": fl, "tokens": int(x["lens"].sum()), "peak_source": peak_src,
                          "l2": "flushed"}), flush=True)
        del x, out, lse
    for dw in W.DECODE_WORKLOADS:
        if (args.workloads and dw.name not in names) or (not args.workloads and dw is not W.DECODE):
            continue
        xd = W.make_decode_inputs(dw, device=dev)
        KVB = decode_kv_bytes(dw, xd["cache_seqlens"].cpu())
        d_out = torch.empty_like(xd["q"])
        d_lse = torch.empty((dw.B, dw.H, 1), dtype=torch.float32, device=dev)
        for s in [int(x) for x in args.splits.split(",")]:
            nb = fa.fa_kvcache_workspace_size(dw.B, dw.H, dw.d, dw.max_blocks, dw.page_size, s)
            ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=dev)
            dec = fa.fa_fwd_kvcache_gqa if dw.kv_heads != dw.H else fa.fa_fwd_kvcache
            run = lambda: dec(xd["q"], xd["k_cache"], xd["v_cache"], xd["block_table"], xd["cache_seqlens"], d_out,
                              d_lse, dw.scale, -1, None, 0.0, s, ws)
            for _ in range(args.warmup):
                run()
            times = []
            for _ in range(args.steps):
                a, b = ev(), ev()
                a.record()
                run()
                b.record()
                times.append((a, b))
            torch.cuda.synchronize()
            ms = statistics.median([a.elapsed_time(b) for a, b in times])
            gbs = KVB / (ms * 1e-3) / 1e9
            print(json.dumps({"workload": dw.name, "num_splits": s or "auto(%d)" % fa.fa_kvcache_num_splits_gqa(
                dw.B, dw.H, dw.kv_heads, dw.d, dw.max_blocks, dw.page_size, 0), "ms": round(ms, 4),
                "GB/s": round(gbs, 1),
                "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "kv_bytes": KVB, "peak_source": peak_src}),
                flush=True)
        del xd


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--config-steps", type=int, default=20, help="timed launches per forward_configs entry")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work per baseline leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true")
    ap.add_argument("--workloads", default="", help="comma-separated workload names for --sweep")
    ap.add_argument("--splits", default="0,1,2,4,8,16,32", help="decode split counts for --sweep (0 = auto)")
    args = ap.parse_args()
    if args.warmup < 3 and not args.sweep:
        args.warmup = 3
    if args.impl == "reference":
        reference_arm(args)
    elif args.sweep:
        sweep(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
