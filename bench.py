#!/usr/bin/env python
"""Benchmark: exact attention forward + backward TFLOP/s on B200.

One step = one pass of the whole path over one batch: the forward kernel
(O, lse) and the three backward phases (prepare, main, finish).  Default
workload: B=2 H=32 N=8192 d=128 bf16, K scaled by 2, causal (the prefill-shaped
configuration the >=60%-of-peak target names).  FLOPs follow the pages'
convention: forward 4*B*H*N^2*d (halved for causal), backward 2.5x forward.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...     # the fp64 CPU oracle on the same workload

Under torchrun each rank runs the same per-GPU workload on its own seeded
batch (weak scaling, no data-path collective); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from exact_io_aware_100_b200 import inputs  # noqa: E402

METRIC = "attention fwd/bwd TFLOP/s (bf16, causal & non-causal); % of B200 BF16 peak"
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 2**20
EX2_PER_CLK_PER_SM = 16      # MUFU ex2 rate measured on this GPU by a probe (16 lanes / clock / SM)
MUFU_SHARE_OF_EXP = 5 / 8    # both kernels evaluate three of every eight exp2 pairs by polynomial
KERNEL_SOURCES = ["exact_io_aware_100_b200/csrc/ptx.cuh", "exact_io_aware_100_b200/csrc/layout.cuh",
                  "exact_io_aware_100_b200/csrc/fwd_kernel.cuh", "exact_io_aware_100_b200/csrc/bwd_kernel.cuh",
                  "exact_io_aware_100_b200/csrc/fwd256_kernel.cuh", "exact_io_aware_100_b200/csrc/bwd256_kernel.cuh",
                  "exact_io_aware_100_b200/csrc/fwd64_kernel.cuh",
                  "exact_io_aware_100_b200/csrc/fa_api.cu"]


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=30)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="prefill", choices=sorted(inputs.WORKLOADS))
    p.add_argument("--fwd-only", action="store_true", help="time the forward kernel alone")
    p.add_argument("--e2e-steps", type=int, default=5)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-heads", type=int, default=6, help="heads in the CPU baseline sample")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the table of the other configurations (prefill workload only)")
    p.add_argument("--sustained-s", type=float, default=3.0,
                   help="seconds of back-to-back launches in the sustained leg (0 skips it)")
    p.add_argument("--shape", default=None,
                   help="B,H,N override of the workload's sizes (smaller cases for profiler captures)")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def committed_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it still matches the source."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get("kernels", {}).get(f"{kernel}@{workload}")
    if not e or e.get("csrc_sha256") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# --------------------------------------------------------------------- ranks
def rank_seed(w, rank: int) -> int:
    """Each rank generates its own batch (weak scaling: disjoint data, no collective on the data path)."""
    return w.seed + 100003 * rank


def max_over_ranks(x: float, dist, world: int, device) -> float:
    """The job's time is the slowest rank's (device-timed on each rank, then a MAX all-reduce)."""
    if world <= 1:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank_step: float, world: int, steps: int, ms: float) -> float:
    """Whole-job throughput: the work of every rank over the slowest rank's time."""
    return world * flops_per_rank_step * steps / (ms * 1e-3) / 1e12


# --------------------------------------------------------------------- end to end
def pipelined_e2e(torch, dev, pinned_in: dict, buf0: dict, out_names, run, steps: int):
    """Device-timed milliseconds per step of the end-to-end loop a user would run:
    every step copies its inputs from pinned host memory, runs the attention calls
    and copies its outputs back to pinned host memory.  Two device buffer sets let
    the host->device copy of step s+1, the compute of step s and the device->host
    copy of step s-1 run at once on three streams (PCIe is full duplex and the
    copy engines are not the SMs); events keep each buffer set's uses in order.
    run(buffers, stream) enqueues one step's calls on `stream`."""
    bufs = [buf0, {n: torch.empty_like(t) for n, t in buf0.items()}]
    host_out = [{n: torch.empty(buf0[n].shape, dtype=buf0[n].dtype, pin_memory=True) for n in out_names}
                for _ in range(2)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    in_ready = [torch.cuda.Event() for _ in range(2)]
    cmp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def one(s):
        b = s & 1
        if s >= 2:
            s_in.wait_event(cmp_done[b])           # step s-2's compute is done with these inputs
        with torch.cuda.stream(s_in):
            for n, t in pinned_in.items():
                bufs[b][n].copy_(t, non_blocking=True)
        in_ready[b].record(s_in)
        s_cmp.wait_event(in_ready[b])
        if s >= 2:
            s_cmp.wait_event(out_done[b])          # step s-2's outputs have been copied out
        run(bufs[b], s_cmp)
        cmp_done[b].record(s_cmp)
        s_out.wait_event(cmp_done[b])
        with torch.cuda.stream(s_out):
            for n in out_names:
                host_out[b][n].copy_(bufs[b][n], non_blocking=True)
        out_done[b].record(s_out)

    for s in range(2):                             # untimed: first use of every buffer and stream
        one(s)
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for s in range(2, 2 + steps):
        one(s)
    s_in.wait_event(out_done[0])
    s_in.wait_event(out_done[1])
    end.record(s_in)
    torch.cuda.synchronize(dev)
    return start.elapsed_time(end) / steps


PIPELINE_NOTE = ("two device buffer sets; each step's host->device input copy, compute and device->host output "
                 "copy on three streams, overlapping the neighbouring steps")


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML during the timed region."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:   # NVML unavailable: report nothing rather than guess
            self.nv = None

    def _handle(self, idx):
        """NVML handle of CUDA device `idx`: match UUIDs, else CUDA_VISIBLE_DEVICES, else idx."""
        import torch
        pynvml = self.nv
        try:
            want = "GPU-" + str(torch.cuda.get_device_properties(idx).uuid)
            for j in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(j)
                got = pynvml.nvmlDeviceGetUUID(h)
                got = got.decode() if isinstance(got, bytes) else str(got)
                if got == want:
                    return h
        except Exception:
            pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        parts = [p.strip() for p in vis.split(",") if p.strip()]
        if idx < len(parts) and parts[idx].isdigit():
            return pynvml.nvmlDeviceGetHandleByIndex(int(parts[idx]))
        return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def _reasons(self):
        f = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return f(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                bits = self._reasons()
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr is not None:
            self._thr.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# --------------------------------------------------------------------- CPU oracle
def oracle_sample(w, heads: int, seed_offset: int = 0, fwd_only: bool = False):
    """fwd (+ bwd) of `heads` whole heads of the workload with the fp64 oracle.
    Returns (seconds, algorithmic FLOPs of the sample, description)."""
    from oracle import attention_bwd, attention_bwd_varlen, attention_fwd, attention_fwd_decode, attention_fwd_varlen
    shape1 = (1, 1, w.N, w.d)
    t_total, flops = 0.0, 0.0
    if w.varlen:   # one head of one sequence of the batch per sample, lengths taken in turn
        lens = w.seq_lengths()
        used = []
        for i in range(heads):
            n = lens[(i + seed_offset) % len(lens)]
            used.append(n)
            seed = w.seed + 7919 * (i + 1 + seed_offset)
            f = {x: inputs.to_f64(inputs.make_tensor(seed, x, (n, 1, w.d)), "bf16") for x in ("q", "k", "v", "do")}
            cu = np.array([0, n])
            t0 = time.perf_counter()
            attention_fwd_varlen(f["q"], f["k"], f["v"], cu, cu, w.scale, w.causal)
            if not fwd_only:
                attention_bwd_varlen(f["q"], f["k"], f["v"], f["do"], cu, cu, w.scale, w.causal)
            t_total += time.perf_counter() - t0
            flops += (1.0 if fwd_only else 3.5) * 4.0 * n * n * w.d / (2 if w.causal else 1)
        return t_total, flops, (f"{'fwd' if fwd_only else 'fwd+bwd'} of {heads} head(s) of packed sequences "
                                f"of lengths {used} (d={w.d}), numpy float64 oracle")
    if w.lq:       # decode: one query head's lq positions against its cache
        for i in range(heads):
            seed = w.seed + 7919 * (i + 1 + seed_offset)
            f = {n: inputs.to_f64(inputs.make_tensor(seed, n, (1, 1, w.lq if n == "q" else w.N, w.d)), "bf16")
                 for n in ("q", "k", "v")}
            t0 = time.perf_counter()
            attention_fwd_decode(f["q"], f["k"], f["v"], w.scale, w.causal)
            t_total += time.perf_counter() - t0
            flops += w.fwd_flops() / (w.B * w.H)
        return t_total, flops, (f"decode of {heads} query head(s) ({w.lq} x {w.d} against {w.N} keys), "
                                f"numpy float64 oracle")
    for i in range(heads):
        seed = w.seed + 7919 * (i + 1 + seed_offset)
        f = {n: inputs.to_f64(inputs.make_tensor(seed, n, shape1, w.k_scale if n == "k" else 1.0), "bf16")
             for n in ("q", "k", "v", "do")}
        t0 = time.perf_counter()
        attention_fwd(f["q"], f["k"], f["v"], w.scale, w.causal)
        if not fwd_only:
            attention_bwd(f["q"], f["k"], f["v"], f["do"], w.scale, w.causal)
        t_total += time.perf_counter() - t0
        flops += (1.0 if fwd_only else 3.5) * 4.0 * w.N * w.N * w.d / (2 if w.causal else 1)
    desc = (f"{'fwd' if fwd_only else 'fwd+bwd'} of {heads} whole head(s) (1 x 1 x {w.N} x {w.d}) "
            f"of the workload, numpy float64 oracle")
    return t_total, flops, desc


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    fwd_only = is_fwd_only(args, w)
    for _ in range(args.warmup):
        oracle_sample(w, 1, seed_offset=1000, fwd_only=fwd_only)
    secs, flops = 0.0, 0.0
    for s in range(args.steps):
        t, f, desc = oracle_sample(w, 1, seed_offset=s, fwd_only=fwd_only)
        secs += t
        flops += f
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, "fwd" if fwd_only else "fwd+bwd",
                                  "oracle on host cores; each step one whole head"),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"per step: {desc}"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def is_fwd_only(args, w) -> bool:
    """The backward covers bf16 inputs (d = 64, 128, 256); fp32-input and decode workloads time the forward."""
    return args.fwd_only or w.dtype != "bf16" or bool(w.lq)


def workload_config(w, step: str, note: str):
    c = {"workload": f"{w.name}: B={w.B} H={w.H}" + (f" H_kv={w.kv_heads}" if w.kv_heads != w.H else "")
                     + (f" Lq={w.lq}" if w.lq else "")
                     + (f" packed, lengths N/8..N, total {sum(w.seq_lengths())}" if w.varlen else "")
                     + f" N={w.N} d={w.d} {'causal' if w.causal else 'non-causal'}"
                     + (f" K*{w.k_scale:g}" if w.k_scale != 1.0 else ""),
         "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "step": step, "l2": note}
    if w.kv_heads != w.H:
        c["H_kv"] = w.kv_heads
    if w.lq:
        c["Lq"] = w.lq
    return c


# --------------------------------------------------------------------- GPU arm
def run_decode(args, w, fa, torch, dist, world, rank, local_rank, dev):
    """Decode workloads: fa_decode (split partials + merge) over a cache larger than L2; HBM bound."""
    B, H, Hkv, Lq, N, d = w.B, w.H, w.kv_heads, w.lq, w.N, w.d
    seed = rank_seed(w, rank)
    shapes = {"q": (B, H, Lq, d), "k": (B, Hkv, N, d), "v": (B, Hkv, N, d)}
    host = {n: inputs.make_tensor(seed, n, shp) for n, shp in shapes.items()}
    pinned = {n: torch.from_numpy(host[n].view(np.int16)).view(torch.bfloat16).pin_memory() for n in host}
    dv_ = {n: pinned[n].to(dev) for n in host}
    o = torch.empty(shapes["q"], dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, Lq), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.fa_decode_workspace_size(B, H, Hkv, Lq, N, d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    io_bytes = sum(x.nbytes for x in host.values()) + o.numel() * 2 + lse.numel() * 4
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if io_bytes < 2 * L2_BYTES else None

    buf0 = {"q": dv_["q"], "k": dv_["k"], "v": dv_["v"], "o": o, "lse": lse}

    def step(ev=None, bf=buf0, st=stream):
        if ev is not None:
            ev[0].record(st)
        fa.fa_decode(bf["q"], bf["k"], bf["v"], bf["o"], bf["lse"], w.causal, ws, stream=st)
        if ev is not None:
            ev[1].record(st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fa.fa_get_device_status() != fa.FA_OK:
        raise SystemExit("device status reported a timeout during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t0.record(stream)
        for s in range(args.steps):
            if flush is not None:
                flush.fill_(s & 0xff)
            step(evs[s])
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    elapsed_ms = sum(step_ms) if flush is not None else t0.elapsed_time(t1)
    if fa.fa_get_device_status() != fa.FA_OK:
        raise SystemExit("device status reported a timeout in the timed region")
    elapsed_ms = max_over_ranks(elapsed_ms, dist, world, dev)
    flops = w.fwd_flops()
    value = job_tflops(flops, world, args.steps, elapsed_ms)
    peaks, peak_src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    dec_ms = statistics.mean(step_ms)
    gbs = io_bytes / (dec_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "kernel": "fa_decode_kernel + fa_decode_merge_kernel", "achieved": gbs,
                "peak": hbm, "unit": "GB/s", "frac": gbs / hbm, "peak_source": f"{peak_src} hbm_gbs",
                "bytes_per_launch": io_bytes, "traffic": None}
    e2e = None
    if not args.no_e2e:
        if world > 1:
            dist.barrier()
        e_ms = pipelined_e2e(torch, dev, pinned, buf0, ("o", "lse"), lambda bf, st: step(bf=bf, st=st),
                             args.e2e_steps)
        e_ms = max_over_ranks(e_ms, dist, world, dev)
        e2e = {"value": job_tflops(flops, world, 1, e_ms), "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(x.nbytes for x in host.values()),
               "d2h_bytes_per_step": o.numel() * 2 + lse.numel() * 4, "ms_per_step": e_ms, "pipelined": PIPELINE_NOTE}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        secs, f, desc = oracle_sample(w, args.cpu_heads)
        cpu = {"value": f / secs / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": desc + f"; {secs:.1f} s"}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, "decode",
                                  f"cache larger than L2 ({io_bytes / 2**20:.0f} MiB per step), no flush"
                                  if flush is None else "L2 flushed before every step"),
        "kernels": {"fa_decode": {"ms": dec_ms, "median_ms": statistics.median(step_ms), "min_ms": min(step_ms),
                                  "gbs": gbs, "frac_of_measured_hbm": gbs / hbm}},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": 2 * args.steps, "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_varlen(args, w, fa, torch, dist, world, rank, local_rank, dev):
    """Packed variable-length batch: fa_fwd_general + fa_bwd_general over B sequences of mixed lengths."""
    lens = w.seq_lengths()
    total, H, Hkv, d = sum(lens), w.H, w.kv_heads, w.d
    seed = rank_seed(w, rank)
    shapes = {"q": (total, H, d), "k": (total, Hkv, d), "v": (total, Hkv, d), "do": (total, H, d)}
    host = {n: inputs.make_tensor(seed, n, shp, w.k_scale if n == "k" else 1.0) for n, shp in shapes.items()}
    pinned = {n: torch.from_numpy(host[n].view(np.int16)).view(torch.bfloat16).pin_memory() for n in host}
    pinned["cu"] = torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)).pin_memory()
    dv_ = {n: pinned[n].to(dev) for n in pinned}
    o = torch.empty(shapes["q"], dtype=torch.bfloat16, device=dev)
    lse = torch.empty((H, total), dtype=torch.float32, device=dev)
    dq = torch.empty(shapes["q"], dtype=torch.bfloat16, device=dev)
    dk, dvv = (torch.empty(shapes["k"], dtype=torch.bfloat16, device=dev) for _ in range(2))
    L0 = fa.layout_packed(dv_["q"], dv_["k"], dv_["v"], o, dv_["cu"], dv_["cu"], max(lens), max(lens),
                          dv_["do"], dq, dk, dvv)
    ws = torch.empty(fa.fa_bwd_general_workspace_size(L0), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    buf0 = dict(dv_, o=o, lse=lse, dq=dq, dk=dk, dv=dvv)

    def step(ev=None, bf=buf0, st=stream):
        L = L0 if bf is buf0 else fa.layout_packed(bf["q"], bf["k"], bf["v"], bf["o"], bf["cu"], bf["cu"], max(lens),
                                                     max(lens), bf["do"], bf["dq"], bf["dk"], bf["dv"])
        if ev is not None:
            ev[0].record(st)
        fa.fa_fwd_general(bf["q"], bf["k"], bf["v"], bf["o"], bf["lse"], L, w.causal, stream=st)
        if ev is not None:
            ev[1].record(st)
        fa.fa_bwd_general(bf["q"], bf["k"], bf["v"], bf["o"], bf["lse"], bf["do"], bf["dq"], bf["dk"], bf["dv"], L,
                          w.causal, ws, stream=st)
        if ev is not None:
            ev[2].record(st)

    in_bytes = sum(x.nbytes for x in host.values())
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fa.fa_get_device_status() != fa.FA_OK:
        raise SystemExit("device status reported an error during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t0.record(stream)
        for s in range(args.steps):
            step(evs[s])
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed_ms = t0.elapsed_time(t1)
    if fa.fa_get_device_status() != fa.FA_OK:
        raise SystemExit("device status reported an error in the timed region")
    elapsed_ms = max_over_ranks(elapsed_ms, dist, world, dev)
    fwd_all = [e[0].elapsed_time(e[1]) for e in evs]
    bwd_all = [e[1].elapsed_time(e[2]) for e in evs]
    fwd_flops = w.fwd_flops()
    bwd_flops = 2.5 * fwd_flops
    value = job_tflops(fwd_flops + bwd_flops, world, args.steps, elapsed_ms)
    peaks, peak_src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    kernels = {}
    for name, flops, ts, note in (("fa_fwd_kernel", fwd_flops, fwd_all, "fa_fwd_general: one kernel"),
                                  ("fa_bwd_kernel", bwd_flops, bwd_all,
                                   "fa_bwd_general: prepare, main and finish kernels timed together")):
        tf = flops / (statistics.mean(ts) * 1e-3) / 1e12
        kernels[name] = {"ms": statistics.mean(ts), "median_ms": statistics.median(ts), "min_ms": min(ts),
                         "tflops": tf, "frac_of_measured_burst": tf / burst, "frac_of_measured_sustained": tf / sustained,
                         "note": note}
    dom = max(kernels, key=lambda n: kernels[n]["ms"])
    achieved = kernels[dom]["tflops"]
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                "frac": achieved / burst, "peak_source": f"{peak_src} bf16_tflops (burst)",
                "frac_of_sustained": achieved / sustained,
                "flops_per_launch": fwd_flops if dom == "fa_fwd_kernel" else bwd_flops,
                "traffic": committed_traffic(dom, w.name)}
    e2e = None
    if not args.no_e2e:
        outs = ("o", "lse", "dq", "dk", "dv")
        if world > 1:
            dist.barrier()
        e_ms = pipelined_e2e(torch, dev, pinned, buf0, outs, lambda bf, st: step(bf=bf, st=st), args.e2e_steps)
        e_ms = max_over_ranks(e_ms, dist, world, dev)
        e2e = {"value": job_tflops(fwd_flops + bwd_flops, world, 1, e_ms), "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in pinned.values()),
               "d2h_bytes_per_step": sum(buf0[n].numel() * buf0[n].element_size() for n in outs),
               "ms_per_step": e_ms, "pipelined": PIPELINE_NOTE}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        secs, f, desc = oracle_sample(w, args.cpu_heads)
        cpu = {"value": f / secs / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": desc + f"; {secs:.1f} s"}
    cfg = workload_config(w, "fwd+bwd", f"inputs larger than L2 ({in_bytes / 2**20:.0f} MiB per step), no flush")
    cfg["seq_lengths"] = lens
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
        "frac_of_measured_burst_peak": value / world / burst,
        "fwd_tflops": kernels["fa_fwd_kernel"]["tflops"], "bwd_tflops": kernels["fa_bwd_kernel"]["tflops"],
        "kernels": kernels, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": 4 * args.steps, "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# --------------------------------------------------------------------- the other configurations
# The metric covers forward and backward, causal and non-causal, at every configuration the
# workload list names.  The headline line measures the prefill configuration; this table adds the
# others, measured the same way (CUDA events on the launching stream around each call, an L2 flush
# before every step whose inputs and outputs fit in twice the L2), one after the other in the same
# process.
CONFIG_TABLE = (("1", "single_head", 20), ("2", "multi_head", 20), ("2c", "multi_head_causal", 20),
                ("3nc", "prefill_noncausal", 5), ("4", "long_context", 3), ("5", "backward", 10))


def _device_inputs(torch, dev, w, names, seed):
    shape = (w.B, w.H, w.N, w.d)
    out = {}
    for n in names:
        x = inputs.make_tensor(seed, n, shape, w.k_scale if n == "k" else 1.0, "f32" if w.dtype == "f32" else "bf16")
        t = torch.from_numpy(x) if w.dtype == "f32" else torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
        out[n] = t.to(dev)
    return out


def measure_config(fa, torch, dev, local_rank, w, steps: int, warmup: int, burst: float, sustained: float):
    """Forward (and, for bf16 inputs, backward) of one configuration: TFLOP/s from the mean of the
    per-call CUDA events, fractions of the measured and datasheet peaks, the NVML clock median."""
    fwd_only = w.dtype != "bf16"
    names = ("q", "k", "v") if fwd_only else ("q", "k", "v", "do")
    t = _device_inputs(torch, dev, w, names, w.seed)
    B, H, N, d = w.B, w.H, w.N, w.d
    o = torch.empty((B, H, N, d), dtype=torch.float32 if w.dtype == "f32" else torch.bfloat16, device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    fws = None
    if w.dtype == "f32":
        fws = torch.empty(fa.fa_fwd_workspace_size(B, H, N, d, fa.FA_F32), dtype=torch.uint8, device=dev)
    if not fwd_only:
        dq, dk, dv = (torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev) for _ in range(3))
        ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        if w.dtype == "f32":
            fa.fa_fwd_ex(t["q"], t["k"], t["v"], o, lse, w.causal, fa.FA_F32, fws, stream=stream)
        else:
            fa.fa_fwd(t["q"], t["k"], t["v"], o, lse, w.causal, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        if fwd_only:
            return
        fa.fa_bwd_prepare(o, lse, t["do"], ws, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        fa.fa_bwd_main(t["q"], t["k"], t["v"], t["do"], dk, dv, w.causal, ws, stream=stream)
        if ev is not None:
            ev[3].record(stream)
        fa.fa_bwd_finish(dq, ws, stream=stream)
        if ev is not None:
            ev[4].record(stream)

    io_bytes = sum(x.numel() * x.element_size() for x in t.values()) * (1 if fwd_only else 2) + \
        o.numel() * o.element_size()
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if io_bytes < 2 * L2_BYTES else None
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    with ClockSampler(local_rank, period_s=0.005) as clk:
        for s in range(steps):
            if flush is not None:
                flush.fill_(s & 0xff)
            step(evs[s])
        torch.cuda.synchronize(dev)
    if fa.fa_get_device_status() != fa.FA_OK:
        raise SystemExit(f"device status reported an error in configuration {w.name}")
    fwd_flops = w.fwd_flops()
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    fwd_tf = fwd_flops / (fwd_ms * 1e-3) / 1e12
    r = {"workload": workload_config(w, "fwd" if fwd_only else "fwd+bwd", "")["workload"],
         "steps": steps, "warmup": warmup,
         "l2": "flushed before every step" if flush is not None else "inputs larger than L2, no flush",
         "fwd_ms": fwd_ms, "fwd_tflops": fwd_tf, "fwd_frac_of_measured_burst": fwd_tf / burst,
         "fwd_frac_of_measured_sustained": fwd_tf / sustained, "fwd_frac_of_datasheet": fwd_tf / DATASHEET_BF16_TFLOPS}
    if w.dtype == "f32":
        r["fwd_note"] = "fa_fwd_ex(FA_F32): one cast kernel (q, k, v) and the forward"
        alg = 3 * B * H * N * d * 4 + B * H * N * d * 4 + 4 * B * H * N
        r["fwd_us"] = fwd_ms * 1e3
        r["fwd_algorithmic_gbs"] = alg / (fwd_ms * 1e-3) / 1e9
    if not fwd_only:
        bwd_flops = 2.5 * fwd_flops
        bwd_ms = statistics.mean(e[1].elapsed_time(e[4]) for e in evs)
        main_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
        bwd_tf, main_tf = bwd_flops / (bwd_ms * 1e-3) / 1e12, bwd_flops / (main_ms * 1e-3) / 1e12
        r.update({"bwd_ms": bwd_ms, "bwd_tflops": bwd_tf, "bwd_frac_of_measured_burst": bwd_tf / burst,
                  "bwd_frac_of_datasheet": bwd_tf / DATASHEET_BF16_TFLOPS,
                  "bwd_main_kernel_ms": main_ms, "bwd_main_kernel_tflops": main_tf,
                  "bwd_main_kernel_frac_of_measured_burst": main_tf / burst})
        step_tf = (fwd_flops + bwd_flops) / ((fwd_ms + bwd_ms) * 1e-3) / 1e12
        r.update({"step_tflops": step_tf, "step_frac_of_measured_burst": step_tf / burst})
    r["clocks"] = clk.summary()
    return r


def sustained_leg(fa, torch, dev, local_rank, w, seconds: float, sustained: float):
    """The configuration's forward, then its whole step (forward + the three backward phases),
    launched back to back on one stream for at least `seconds` each: device time from CUDA events
    around the loop, the NVML median SM clock during it, and the fraction of the measured sustained
    bf16 peak (the one a kernel meets inside a seconds-long run)."""
    t = _device_inputs(torch, dev, w, ("q", "k", "v", "do"), w.seed)
    B, H, N, d = w.B, w.H, w.N, w.d
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev) for _ in range(3))
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def fwd():
        fa.fa_fwd(t["q"], t["k"], t["v"], o, lse, w.causal, stream=stream)

    def full():
        fwd()
        fa.fa_bwd(t["q"], t["k"], t["v"], o, lse, t["do"], dq, dk, dv, w.causal, ws, stream=stream)

    out = {}
    fwd_flops = w.fwd_flops()
    for name, fn, flops in (("fwd", fwd, fwd_flops), ("step", full, 3.5 * fwd_flops)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        iters = max(10, int(math.ceil(seconds * 1e3 / max(a.elapsed_time(b), 1e-3))))
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local_rank, period_s=0.05) as clk:
            t0.record(stream)
            for _ in range(iters):
                fn()
            t1.record(stream)
            torch.cuda.synchronize(dev)
        ms = t0.elapsed_time(t1)
        tf = flops * iters / (ms * 1e-3) / 1e12
        out[name] = {"iterations": iters, "seconds": ms * 1e-3, "tflops": tf,
                     "frac_of_measured_sustained": tf / sustained, "frac_of_datasheet": tf / DATASHEET_BF16_TFLOPS,
                     "clocks": clk.summary()}
    if fa.fa_get_device_status() != fa.FA_OK:
        raise SystemExit("device status reported an error in the sustained leg")
    out["workload"] = workload_config(w, "fwd+bwd", "")["workload"]
    out["note"] = ("back-to-back launches on one stream for at least %.0f s each; tflops from CUDA events around "
                   "the loop; clocks sampled by NVML during it" % seconds)
    return out


def main():
    args = parse_args()
    w = inputs.WORKLOADS[args.workload]
    if args.shape:
        import dataclasses
        B_, H_, N_ = (int(x) for x in args.shape.split(","))
        w = dataclasses.replace(w, name=f"{w.name}[{B_},{H_},{N_}]", B=B_, H=H_, N=N_)
    if args.impl == "reference":
        run_reference(args, w)
        return
    import torch
    import torch.distributed as dist
    import exact_io_aware_100_b200 as fa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    fa.load_library()
    if w.lq:
        run_decode(args, w, fa, torch, dist, world, rank, local_rank, dev)
        return
    if w.varlen:
        run_varlen(args, w, fa, torch, dist, world, rank, local_rank, dev)
        return

    fwd_only = is_fwd_only(args, w)
    B, H, N, d = w.B, w.H, w.N, w.d
    shape = (B, H, N, d)
    seed = rank_seed(w, rank)          # each rank its own batch
    names = ("q", "k", "v") if fwd_only else ("q", "k", "v", "do")
    f32_in = w.dtype == "f32"               # fp32 inputs go through fa_fwd_ex (cast to bf16 on the GPU)
    gqa = w.kv_heads != w.H
    kv_shape = (B, w.kv_heads, N, d)
    host = {n: inputs.make_tensor(seed, n, kv_shape if n in ("k", "v") else shape, w.k_scale if n == "k" else 1.0,
                                  "f32" if f32_in else "bf16")
            for n in names}
    if f32_in:
        pinned = {n: torch.from_numpy(host[n]).pin_memory() for n in names}
    else:
        pinned = {n: torch.from_numpy(host[n].view(np.int16)).view(torch.bfloat16).pin_memory() for n in names}
    dv_ = {n: pinned[n].to(dev) for n in names}
    o = torch.empty(shape, dtype=torch.float32 if f32_in else torch.bfloat16, device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    fws = None
    if f32_in:
        fws = torch.empty(fa.fa_fwd_workspace_size(B, H, N, d, fa.FA_F32), dtype=torch.uint8, device=dev)
    if not fwd_only:
        dq = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        dk, dvv = (torch.empty(kv_shape, dtype=torch.bfloat16, device=dev) for _ in range(2))
        ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    causal = w.causal
    buf0 = dict(dv_, o=o, lse=lse)
    if not fwd_only:
        buf0.update(dq=dq, dk=dk, dv=dvv)

    def step(ev=None, bf=buf0, st=stream):
        q_, k_, v_, o_, lse_ = bf["q"], bf["k"], bf["v"], bf["o"], bf["lse"]
        if ev is not None:
            ev[0].record(st)
        if f32_in:
            fa.fa_fwd_ex(q_, k_, v_, o_, lse_, causal, fa.FA_F32, fws, stream=st)
        elif gqa:
            fa.fa_fwd_gqa(q_, k_, v_, o_, lse_, causal, stream=st)
        else:
            fa.fa_fwd(q_, k_, v_, o_, lse_, causal, stream=st)
        if ev is not None:
            ev[1].record(st)
        if fwd_only:
            return
        if gqa:      # one call runs the three phases; its time is reported as the main kernel's
            if ev is not None:
                ev[2].record(st)
            fa.fa_bwd_gqa(q_, k_, v_, o_, lse_, bf["do"], bf["dq"], bf["dk"], bf["dv"], causal, ws, stream=st)
            if ev is not None:
                ev[3].record(st)
                ev[4].record(st)
            return
        fa.fa_bwd_prepare(o_, lse_, bf["do"], ws, stream=st)
        if ev is not None:
            ev[2].record(st)
        fa.fa_bwd_main(q_, k_, v_, bf["do"], bf["dk"], bf["dv"], causal, ws, stream=st)
        if ev is not None:
            ev[3].record(st)
        fa.fa_bwd_finish(bf["dq"], ws, stream=st)
        if ev is not None:
            ev[4].record(st)

    launches_per_step = (2 if f32_in else 1) if fwd_only else 4    # fp32: one cast kernel (q, k, v) + the forward
    # Inputs and outputs smaller than twice L2 would stay cached between steps:
    # then every timed step is preceded by a write of a buffer larger than L2,
    # outside the kernels' events, and the step time is the sum of its events.
    io_bytes = sum(host[n].nbytes for n in names) * (2 if not fwd_only else 1) + o.numel() * o.element_size()
    flush = None
    if io_bytes < 2 * L2_BYTES:
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fa.fa_get_device_status() != fa.FA_OK:
        raise SystemExit("device status reported a timeout during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t0.record(stream)
        for s in range(args.steps):
            if flush is not None:
                flush.fill_(s & 0xff)
            step(evs[s])
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    last = 1 if fwd_only else 4
    step_ms = [e[0].elapsed_time(e[last]) for e in evs]
    elapsed_ms = sum(step_ms) if flush is not None else t0.elapsed_time(t1)
    if fa.fa_get_device_status() != fa.FA_OK:
        raise SystemExit("device status reported a timeout in the timed region")
    fwd_all = [e[0].elapsed_time(e[1]) for e in evs]
    main_all = None if fwd_only else [e[2].elapsed_time(e[3]) for e in evs]
    fwd_ms = statistics.mean(fwd_all)
    main_ms = None if fwd_only else statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    prep_ms = None if fwd_only else statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    fin_ms = None if fwd_only else statistics.mean(e[3].elapsed_time(e[4]) for e in evs)
    elapsed_ms = max_over_ranks(elapsed_ms, dist, world, dev)

    fwd_flops = w.fwd_flops()
    bwd_flops = 2.5 * fwd_flops
    step_flops = fwd_flops + (0.0 if fwd_only else bwd_flops)
    value = job_tflops(step_flops, world, args.steps, elapsed_ms)
    peaks, peak_src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))

    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    fwd_tf = fwd_flops / (fwd_ms * 1e-3) / 1e12
    kernels = {"fa_fwd_kernel": {"ms": fwd_ms, "median_ms": statistics.median(fwd_all), "min_ms": min(fwd_all),
                                 "tflops": fwd_tf, "frac_of_measured_burst": fwd_tf / burst,
                                 "frac_of_measured_sustained": fwd_tf / sustained,
                                 "frac_of_datasheet": fwd_tf / DATASHEET_BF16_TFLOPS}}
    if f32_in:
        kernels["fa_fwd_kernel"]["note"] = "fa_fwd_ex(FA_F32): one cast kernel (q, k, v) + the forward"
    if not fwd_only:
        main_tf = bwd_flops / (main_ms * 1e-3) / 1e12
        kernels["fa_bwd_kernel"] = {"ms": main_ms, "median_ms": statistics.median(main_all), "min_ms": min(main_all),
                                    "tflops": main_tf, "frac_of_measured_burst": main_tf / burst,
                                    "frac_of_measured_sustained": main_tf / sustained,
                                    "frac_of_datasheet": main_tf / DATASHEET_BF16_TFLOPS}
        if gqa:
            kernels["fa_bwd_kernel"]["note"] = "fa_bwd_gqa: prepare, main and finish kernels timed together"
        else:
            kernels["fa_bwd_pre_kernel"] = {"ms": prep_ms}
            kernels["fa_bwd_dq_kernel"] = {"ms": fin_ms}
    dom = "fa_fwd_kernel" if (fwd_only or fwd_ms >= main_ms) else "fa_bwd_kernel"
    dom_flops = fwd_flops if dom == "fa_fwd_kernel" else bwd_flops
    achieved = kernels[dom]["tflops"]
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                "frac": achieved / burst, "peak_source": f"{peak_src} bf16_tflops (burst)",
                "frac_of_sustained": achieved / sustained,
                "flops_per_launch": dom_flops, "traffic": committed_traffic(dom, w.name)}
    # forward HBM: each input read once, O and lse written once (the IO-aware minimum)
    in_elem = 4 if f32_in else 2
    fwd_bytes = B * N * d * (H * in_elem + 2 * w.kv_heads * in_elem + H * o.element_size()) + 4 * B * H * N
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    fwd_hbm = {"algorithmic_bytes": fwd_bytes, "gbs": fwd_bytes / (fwd_ms * 1e-3) / 1e9,
               "frac_of_measured_hbm": fwd_bytes / (fwd_ms * 1e-3) / 1e9 / hbm}
    # exponentials: one per visible score in the forward, recomputed once in the backward
    n_exp = B * H * (N * (N + 1) // 2 if causal else N * N)

    # ---- end to end through the C ABI with host buffers (pinned), copies timed
    e2e = None
    if not args.no_e2e:
        outs = ("o", "lse") if fwd_only else ("o", "lse", "dq", "dk", "dv")
        h2d = sum(pinned[n].numel() * pinned[n].element_size() for n in names)
        d2h = sum(buf0[n].numel() * buf0[n].element_size() for n in outs)
        if world > 1:
            dist.barrier()
        e_ms = pipelined_e2e(torch, dev, pinned, buf0, outs, lambda bf, st: step(bf=bf, st=st), args.e2e_steps)
        e_ms = max_over_ranks(e_ms, dist, world, dev)
        e2e = {"value": job_tflops(step_flops, world, 1, e_ms), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
               "pipelined": PIPELINE_NOTE}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        secs, flops, desc = oracle_sample(w, args.cpu_heads, fwd_only=fwd_only)
        cpu = {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": desc + f"; {secs:.1f} s"}

    in_bytes = sum(host[n].nbytes for n in names)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, "fwd" if fwd_only else "fwd+bwd",
                                  f"inputs larger than L2 ({in_bytes / 2**20:.0f} MiB per step), no flush"
                                  if flush is None else
                                  f"L2 flushed before every step ({2 * L2_BYTES / 2**20:.0f} MiB write, outside the "
                                  f"kernel events; value from the summed step events)"),
        "frac_of_measured_burst_peak": value / world / burst,
        "frac_of_datasheet_peak": value / world / DATASHEET_BF16_TFLOPS,
        "fwd_tflops": fwd_tf, "bwd_tflops": None if fwd_only else bwd_flops / ((prep_ms + main_ms + fin_ms) * 1e-3) / 1e12,
        "kernels": kernels, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps, "clocks": clk.summary(),
        "fwd_hbm": fwd_hbm,
    }
    sm_mhz = line["clocks"].get("sm_mhz") or 1965.0
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    mufu_s = n_exp * MUFU_SHARE_OF_EXP / (EX2_PER_CLK_PER_SM * n_sm * sm_mhz * 1e6)
    line["exp"] = {"count_fwd": n_exp, "count_bwd": 0 if fwd_only else n_exp, "on_mufu": MUFU_SHARE_OF_EXP,
                   "mufu_time_share_fwd": mufu_s / (fwd_ms * 1e-3),
                   "mufu_time_share_bwd": None if fwd_only else mufu_s / (main_ms * 1e-3)}
    if w.name == "prefill" and world == 1:
        if not args.no_configs:    # the other configurations of the metric, same process, after the headline
            table = {"3": {"workload": line["config"]["workload"], "fwd_tflops": fwd_tf,
                           "fwd_frac_of_measured_burst": fwd_tf / burst,
                           "bwd_tflops": line["bwd_tflops"], "bwd_main_kernel_tflops": kernels["fa_bwd_kernel"]["tflops"],
                           "bwd_main_kernel_frac_of_measured_burst": kernels["fa_bwd_kernel"]["frac_of_measured_burst"],
                           "note": "the headline measurement of this line", "clocks": line["clocks"]}}
            del buf0, dv_
            for key, name, n_steps in CONFIG_TABLE:
                table[key] = measure_config(fa, torch, dev, local_rank, inputs.WORKLOADS[name], n_steps, 3, burst,
                                            sustained)
                torch.cuda.empty_cache()
            line["configs"] = table
        if args.sustained_s > 0:
            line["sustained"] = sustained_leg(fa, torch, dev, local_rank, w, args.sustained_s, sustained)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
