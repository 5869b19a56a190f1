#!/usr/bin/env python
"""Benchmark of the packed causal attention hot path (SAP, one GPU per rank).

One step = the whole path over one packed batch: sap_attn_fwd (partial
attention per (q-tile, kv-chunk)), sap_merge (exact LSE merge), sap_attn_bwd
(D, dK/dV/dQ, dQ conversion).  Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Metric: TFLOP/s on unmasked FLOPs, 14 * head_dim * pairs * hq per step
(forward 4, backward 10), pairs = sum over documents of L(L+1)/2.  Under
torchrun every rank runs its own independent batch (seed + rank): data
parallel replicas, weak scaling, no collective on the data path.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "packed causal attn fwd+bwd TFLOP/s (unmasked FLOPs), tokens/s; % bf16 peak"
DEFAULT_WORKLOAD = "llama31_8b_128k"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), float(d["hbm_gbs"]), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


def _flops(w, pairs):
    return 4.0 * w.d * pairs * w.hq, 10.0 * w.d * pairs * w.hq


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi samples (200 ms) during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu_index)], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                    power.append(float(parts[3]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        under_load = [s for s, p in zip(sm, power) if p > 0.3 * max(power)] or sm
        return {"sm_mhz": statistics.median(under_load), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power)}


class EnergyMeter:
    """Board energy over the timed region from NVML's cumulative energy counter (millijoules).

    On this part the 1 kW board limit (sw_power_cap) sets the clock under load, so energy per step,
    not cycles per step, decides throughput; the line reports it beside the time."""

    def __init__(self, gpu_index: int):
        self.h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
            self.e0 = None
        except Exception:
            self.h = None

    def start(self):
        if self.h is not None:
            try:
                self.e0 = self.nvml.nvmlDeviceGetTotalEnergyConsumption(self.h)
            except Exception:
                self.h = None

    def stop(self):
        """Joules spent by this GPU since start(), or None."""
        if self.h is None or self.e0 is None:
            return None
        try:
            return (self.nvml.nvmlDeviceGetTotalEnergyConsumption(self.h) - self.e0) / 1e3
        except Exception:
            return None


# ------------------------------------------------------------------ traffic


def measured_traffic(workload: str):
    """DRAM bytes per launch of the backward kernel from the committed ncu capture, or None when the
    capture is of another workload or the kernel source has changed since it was taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", f"traffic_sap_bwd_kernel_{workload}.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != rec["source_sha256"]:
        return None
    return rec["dram_bytes_read"] + rec["dram_bytes_write"]


# ------------------------------------------------------------------ ranks


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank runs its own independent packed batch (data-parallel replicas)."""
    return base_seed + rank


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The job's time is the slowest rank's device time (no collective on the data path)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_step: float, steps: int, world: int, elapsed_ms: float) -> float:
    """Whole-job TFLOP/s: the units all ranks processed over the slowest rank's time."""
    return world * flops_per_step * steps / (elapsed_ms / 1e3) / 1e12


# --------------------------------------------------------------------- cpu oracle


def _doc_sample(b, budget_flops: float):
    """The shortest documents of the batch, shortest first, while their oracle cost fits the budget.

    Returns (token index list, cu_seqlens of the sub-batch, unmasked FLOPs, number of documents)."""
    w = b.workload
    cu = b.cu_seqlens
    lens = np.diff(cu)
    order = np.argsort(lens, kind="stable")
    picked, spent = [], 0.0
    for dk in order:
        L = int(lens[dk])
        if L == 0:
            continue
        f = 14.0 * w.d * w.hq * L * (L + 1) / 2
        if picked and spent + f > budget_flops:
            break
        picked.append(int(dk))
        spent += f
        if spent >= budget_flops:
            break
    picked.sort()
    idx = np.concatenate([np.arange(cu[dk], cu[dk + 1]) for dk in picked])
    sub_cu = np.concatenate([[0], np.cumsum([lens[dk] for dk in picked])]).astype(np.int32)
    return idx, sub_cu, spent, len(picked)


def run_oracle_sample(b, budget_flops: float):
    """Times the fp64 oracle (forward + backward) on a bounded document sample. Returns (tflops, seconds, desc)."""
    import torch

    import oracle  # the CPU baseline leg is the one place the benchmark runs the oracle

    w = b.workload
    idx, sub_cu, flops, ndocs = _doc_sample(b, budget_flops)
    ti = torch.as_tensor(idx, device=b.q.device)
    q, k, v, do = (t.index_select(0, ti).cpu() for t in (b.q, b.k, b.v, b.do))
    scale = 1.0 / math.sqrt(w.d)
    t0 = time.perf_counter()
    oracle.attn_fwd(q, k, v, sub_cu, scale)
    oracle.attn_bwd(q, k, v, do, sub_cu, scale)
    dt = time.perf_counter() - t0
    desc = (f"oracle fwd+bwd (fp64, all {w.hq} heads) on the {ndocs} shortest documents of the workload "
            f"({len(idx)} tokens, {flops:.3g} unmasked FLOPs)")
    return flops / dt / 1e12, dt, desc


# ------------------------------------------------------------------------- main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=1e11, help="unmasked FLOPs of the CPU-baseline sample")
    ap.add_argument("--fused-merge", action="store_true",
                    help="one forward pass over all kv chunks of a q tile (no partials, no merge kernel)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="run the workload's recipe at a smaller token count (profiling captures only)")
    ap.add_argument("--parallelism", default="dp", choices=["dp", "sap", "hsap"],
                    help="dp: independent replicas (default); sap / hsap: one batch split across the ranks "
                         "(sequence-aware exchange, with a Ulysses head split of degree --ulysses for hsap)")
    ap.add_argument("--ulysses", type=int, default=1, help="Ulysses (head-split) degree for --parallelism hsap")
    ap.add_argument("--equal-chunks", action="store_true", help="sap / hsap / emulation: equal chunks, not balanced")
    ap.add_argument("--fwd-variant", default="1cta", choices=["1cta", "2cta"],
                    help="forward kernel: one CTA per work item (default) or two-CTA clusters (tcgen05 "
                         "cta_group::2; head_dim 128 with hq/hkv a multiple of 4)")
    ap.add_argument("--emulate-ranks", type=int, default=0,
                    help="one GPU: run the rank plans of a W-way sequence split one after another and report "
                         "per-rank kernel times (the exchange is emulated by device copies)")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = workloads.WORKLOADS[args.workload]
    if args.tokens:
        import dataclasses
        w = dataclasses.replace(w, n=args.tokens, big=min(w.big, args.tokens), name=f"{w.name}@{args.tokens}")

    if args.impl == "reference":
        return run_reference(args, w, rank, world)
    if args.emulate_ranks:
        return run_emulated_ranks(args, w)
    if args.parallelism != "dp":
        return run_split(args, w, rank, world, local_rank)

    import torch
    import torch.distributed as dist

    import packed_sequence_causal_b200 as sap

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if args.fwd_variant == "2cta":
        sap.sap_set_forward_variant(1)

    b = workloads.make_batch(w, rank_seed(args.seed, rank), device=str(dev), with_do=True)
    n, hq, hkv, d = w.n, w.hq, w.hkv, w.d
    scale = 1.0 / math.sqrt(d)
    t_plan = time.perf_counter()
    plan = sap.sap_plan(b.cu_seqlens, n, w.p)
    if args.fused_merge:
        sap.sap_plan_set_fused_merge(plan, True)
    t_plan = time.perf_counter() - t_plan
    sap.sap_plan_upload(plan)
    stats = sap.sap_plan_stats(plan)
    pairs = stats["unmasked_pairs"]
    n_items = len(sap.sap_plan_items(plan))
    _, _, merges = sap.sap_plan_fwd_schedule(plan)
    # merge kernel: algorithmic bytes per call = per (row, head) of a merged q tile, its k fp32
    # partials (O and LSE) read and bf16 O + fp32 LSE written
    merge_bytes = 0
    for qt, _, k in np.asarray(merges).reshape(-1, 3).tolist():
        rows = min(128, n - qt * 128)
        merge_bytes += rows * hq * (k * (4 * d + 4) + 2 * d + 4)
    q, k, v, do = b.q, b.k, b.v, b.do
    o = torch.empty_like(q)
    lse = torch.empty((hq, n), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_f = sap.alloc_workspace(plan, hq, hkv, d, sap.SAP_WS_FWD, dev)
    ws_b = sap.alloc_workspace(plan, hq, hkv, d, sap.SAP_WS_BWD, dev)
    stream = torch.cuda.current_stream()
    # forward, merge (when some q tile has several partials), backward pre-pass, backward, dQ
    # conversion, dK/dV conversion (when some kv tile goes through the fp32 accumulators; one launch
    # per 65535 such tiles)
    n_acc = len(sap.sap_plan_bwd_direct(plan)) - int(sap.sap_plan_bwd_direct(plan).sum())
    launches_per_step = 1 + (1 if len(merges) else 0) + 3 + (n_acc + 65534) // 65535

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        sap.sap_attn_fwd(plan, q, k, v, scale, o, lse, ws_f, stream)
        if ev:
            ev[1].record(stream)
        sap.sap_merge(plan, ws_f, hq, d, o, lse, stream)
        if ev:
            ev[2].record(stream)
        sap.sap_attn_bwd(plan, q, k, v, o, lse, do, scale, dq, dk, dv, ws_b, stream)
        if ev:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = sap.sap_device_status()
    if status != 0:
        raise RuntimeError(f"device error word {status} after warm-up")

    gpu_index = local_rank
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    if vis and "," not in vis and vis.strip().isdigit():
        gpu_index = int(vis)
    sampler = ClockSampler(gpu_index)
    sampler.start()
    meter = EnergyMeter(gpu_index)
    time.sleep(0.4)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    meter.start()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    joules = meter.stop()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    elapsed_ms = max_over_ranks(start.elapsed_time(end), dist if world > 1 else None, dev)
    status = sap.sap_device_status()
    if status != 0:
        raise RuntimeError(f"device error word {status} after the timed steps")

    f_fwd, f_bwd = _flops(w, pairs)
    f_step = f_fwd + f_bwd
    # board energy, summed over the ranks' GPUs (every rank takes the collective, measured or not)
    je = torch.tensor([joules or 0.0, 0.0 if joules is not None else 1.0], dtype=torch.float64,
                      device=dev if world > 1 else "cpu")
    if world > 1:
        dist.all_reduce(je)
    energy = None
    if je[1].item() == 0 and je[0].item() > 0:
        j_all = float(je[0].item())
        energy = {"joules_per_step": round(j_all / args.steps, 2),
                  "avg_watts_per_gpu": round(j_all / world / (start.elapsed_time(end) / 1e3), 1),
                  "tflop_per_joule": round(f_step * world / (j_all / args.steps) / 1e12, 3),
                  "source": "NVML total energy counter over the timed region"}
    ms_step = elapsed_ms / args.steps
    value = job_throughput(f_step, args.steps, world, elapsed_ms)
    tokens_s = world * n * args.steps / (elapsed_ms / 1e3)
    burst, sustained, hbm, peak_src = _peaks()
    # per-call device times from the events recorded on the launching stream
    t_fwd, t_merge, t_bwd = (sum(e[c].elapsed_time(e[c + 1]) for e in evs) / args.steps for c in range(3))

    # end to end through the public API: every step copies its inputs from pinned host memory to
    # the device and reads all of its results back to pinned host memory inside the timed region.
    # Two device sets of inputs and results let step s+1's inputs arrive and step s's results
    # leave on two copy streams while the GPU computes (the prefetch a training loop does); the
    # region opens before the first input copy and closes after the last result has landed.
    e2e = None
    if not args.no_e2e:
        h_in = [t.cpu().pin_memory() for t in (q, k, v, do)]
        h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (o, lse, dq, dk, dv)]
        d_in = [[torch.empty_like(t) for t in (q, k, v, do)] for _ in range(2)]
        d_out = [[torch.empty_like(t) for t in (o, lse, dq, dk, dv)] for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        h2d = sum(t.numel() * t.element_size() for t in h_in)
        d2h = sum(t.numel() * t.element_size() for t in h_out)

        def e2e_run(steps, start_ev=None, end_ev=None):
            ev = lambda: torch.cuda.Event()  # noqa: E731
            # per step: Q, K, V in (the forward's inputs) and dO in (the backward's) as two events;
            # O, LSE out as soon as the merge is done and dQ, dK, dV after the backward
            qkv_ready, do_ready = [ev() for _ in range(steps)], [ev() for _ in range(steps)]
            in_free = [ev() for _ in range(steps)]
            fwd_done, bwd_done, out_free = [ev() for _ in range(steps)], [ev() for _ in range(steps)], \
                [ev() for _ in range(steps)]
            if start_ev is not None:
                start_ev.record(stream)
            s_in.wait_stream(stream)
            s_out.wait_stream(stream)

            def copy_in(i):
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(in_free[i - 2])   # step i-2 no longer reads this set
                    for j, (dst, src) in enumerate(zip(d_in[i % 2], h_in)):
                        dst.copy_(src, non_blocking=True)
                        if j == 2:
                            qkv_ready[i].record(s_in)
                    do_ready[i].record(s_in)

            copy_in(0)
            for i in range(steps):
                if i + 1 < steps:
                    copy_in(i + 1)
                stream.wait_event(qkv_ready[i])
                if i >= 2:
                    stream.wait_event(out_free[i - 2])    # step i-2's results have left this set
                qi, ki, vi, doi = d_in[i % 2]
                oi, lsei, dqi, dki, dvi = d_out[i % 2]
                sap.sap_attn_fwd(plan, qi, ki, vi, scale, oi, lsei, ws_f, stream)
                sap.sap_merge(plan, ws_f, hq, d, oi, lsei, stream)
                fwd_done[i].record(stream)
                stream.wait_event(do_ready[i])
                sap.sap_attn_bwd(plan, qi, ki, vi, oi, lsei, doi, scale, dqi, dki, dvi, ws_b, stream)
                in_free[i].record(stream)
                bwd_done[i].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(fwd_done[i])
                    for dst, src in zip(h_out[:2], d_out[i % 2][:2]):  # O, LSE
                        dst.copy_(src, non_blocking=True)
                    s_out.wait_event(bwd_done[i])
                    for dst, src in zip(h_out[2:], d_out[i % 2][2:]):  # dQ, dK, dV
                        dst.copy_(src, non_blocking=True)
                    out_free[i].record(s_out)
            stream.wait_stream(s_in)
            stream.wait_stream(s_out)
            if end_ev is not None:
                end_ev.record(stream)

        e2e_run(2)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_run(args.steps, s2, e2)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(s2.elapsed_time(e2), dist if world > 1 else None, dev)
        status = sap.sap_device_status()
        if status != 0:
            raise RuntimeError(f"device error word {status} after the end-to-end steps")
        if not torch.equal(h_out[0], o.cpu()):  # the forward is deterministic; the gradients' fp32 sums are not
            raise RuntimeError("end-to-end O differs from the device-resident run on the same inputs")
        e2e = {"value": round(job_throughput(f_step, args.steps, world, e2e_ms), 2), "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(e2e_ms / args.steps, 3),
               "tokens_per_s": round(world * n * args.steps / (e2e_ms / 1e3), 1),
               "overlap": "double-buffered: step s+1's inputs in and step s's results out on two copy "
                          "streams while step s+1 computes; dO in while the forward runs, O and LSE out "
                          "while the backward runs"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, secs, desc = run_oracle_sample(b, args.cpu_budget)
        import oracle
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": oracle.max_threads(), "kind": "oracle", "sample": desc,
               "seconds": round(secs, 2)}

    if rank == 0:
        achieved = f_bwd / (t_bwd / 1e3) / 1e12
        line = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_step, 3),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded packed documents, bf16 N(0,1) Q/K/V/dO)",
            "config": {"workload": w.name, "tokens": n, "docs": int(len(b.cu_seqlens) - 1), "hq": hq, "hkv": hkv,
                       "head_dim": d, "chunks": w.p, "tiles": n_items, "unmasked_pairs_per_head": pairs,
                       "flops_per_step": f_step, "parallelism": f"dp{world}" if world > 1 else "single",
                       "fused_merge": bool(args.fused_merge), "fwd_variant": args.fwd_variant,
                       "l2": "inputs larger than L2 (Q, dO, O 1 GiB each); no flush"},
            "tokens_per_s": round(tokens_s, 1),
            "pct_bf16_peak": round(100 * value / world / burst, 2),
            "pct_bf16_peak_sustained": round(100 * value / world / sustained, 2),
            "peak_source": peak_src,
            "hbm": {"merge_kernel": {"bytes": int(merge_bytes), "ms": round(t_merge, 3),
                                     "gbs": round(merge_bytes / (t_merge / 1e3) / 1e9, 1) if t_merge > 0 else None,
                                     "frac_of_measured": round(merge_bytes / (t_merge / 1e3) / 1e9 / hbm, 3)
                                     if t_merge > 0 else None, "peak_gbs": hbm}},
            "kernels_ms": {"fwd": round(t_fwd, 3), "merge": round(t_merge, 3), "bwd": round(t_bwd, 3),
                           "fwd_tflops": round(f_fwd / (t_fwd / 1e3) / 1e12, 1),
                           "bwd_tflops": round(f_bwd / (t_bwd / 1e3) / 1e12, 1),
                           "plan_host_ms": round(1e3 * t_plan, 2)},
            "roofline": {"bound": "tensor", "kernel": "sap_attn_bwd (bwd_pre + sap_bwd_kernel + bwd_post)",
                         "achieved": round(achieved, 1), "peak": sustained, "unit": "TFLOP/s",
                         "frac": round(achieved / sustained, 4), "frac_of_burst_peak": round(achieved / burst, 4),
                         "traffic": None if args.tokens else measured_traffic(w.name),
                         "traffic_unit": "bytes per sap_bwd_kernel launch (dram__bytes_read + dram__bytes_write)"},
            "clocks": clocks,
            "energy": energy,
            "gpu_launches": launches_per_step * args.steps,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def _split_ranks(w, b, nranks, balanced):
    from packed_sequence_causal_b200 import sap_dist
    return [sap_dist.SapAttention(b.cu_seqlens, w.n, w.hq, w.hkv, w.d, c, nranks, balanced=balanced)
            for c in range(nranks)]


def run_emulated_ranks(args, w):
    """The rank plans of a W-way sequence-parallel split, run one after another on this GPU.

    Per step and rank: the forward (sap_attn_fwd + sap_merge on the rank's windowed buffers) and the
    backward (sap_attn_bwd, then sap_attn_bwd_kv_add of the partials later ranks computed for its
    tokens), each timed with CUDA events on the launching stream.  The key/value windows are
    assembled once from the batch (what the exchange delivers); the partial dK/dV rows are handed
    over by device copies, outside the per-rank times.  Reported: the slowest rank's time per step
    (the step time of W GPUs if the transfers were free) and the whole job's TFLOP/s at that time,
    each rank's time and the bytes it would receive, for the balanced or the equal cut."""
    import torch

    import packed_sequence_causal_b200 as sap

    W = args.emulate_ranks
    balanced = not args.equal_chunks
    torch.cuda.set_device(0)
    b = workloads.make_batch(w, args.seed, device="cuda", with_do=True)
    ranks = _split_ranks(w, b, W, balanced)
    q, k, v, do = b.q, b.k, b.v, b.do
    wins = []
    for r in ranks:
        wd = r.window
        kv0, q0, q1, s0 = wd["kv_begin"], wd["q_begin"], wd["q_end"], wd["span_begin"]
        k_win = torch.zeros((q1 - kv0, w.hkv, w.d), dtype=k.dtype, device="cuda")
        v_win = torch.zeros_like(k_win)
        k_win[s0 - kv0:] = k[s0:q1]
        v_win[s0 - kv0:] = v[s0:q1]
        wins.append((q[q0:q1].contiguous(), k_win, v_win, do[q0:q1].contiguous()))
    stream = torch.cuda.current_stream()

    def step(times=None):
        received = {c: [] for c in range(W)}
        for c, (r, (qr, kw, vw, dor)) in enumerate(zip(ranks, wins)):
            e = [torch.cuda.Event(enable_timing=True) for _ in range(2)] if times is not None else None
            if e:
                e[0].record(stream)
            r.attend(qr, kw, vw)
            r.local_backward(dor)
            if e:
                e[1].record(stream)
                times[c].append(e)
        for r in ranks:
            kv0 = r.window["kv_begin"]
            for src, lo, hi in r.recv:
                received[src].append((lo, hi, r._dk_acc[lo - kv0:hi - kv0].clone(),
                                      r._dv_acc[lo - kv0:hi - kv0].clone()))
        for c, r in enumerate(ranks):
            e = [torch.cuda.Event(enable_timing=True) for _ in range(2)] if times is not None else None
            if e:
                e[0].record(stream)
            r.add_partials(received[c])
            if e:
                e[1].record(stream)
                times[c].append(e)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if sap.sap_device_status() != 0:
        raise RuntimeError("device error word set after warm-up")
    times = [[] for _ in range(W)]
    for _ in range(args.steps):
        step(times)
    torch.cuda.synchronize()
    if sap.sap_device_status() != 0:
        raise RuntimeError("device error word set after the timed steps")
    per_rank = [sum(e[0].elapsed_time(e[1]) for e in t) / args.steps for t in times]
    pairs = sap.sap_plan_stats(ranks[0].full)["unmasked_pairs"]
    f_fwd, f_bwd = _flops(w, pairs)
    row = 2 * w.hkv * w.d * 2
    recv_bytes = [sum(int(hi - lo) for _, lo, hi in r.recv) * row for r in ranks]
    items = sap.sap_plan_chunk_stats(ranks[0].full)["items"]
    slow = max(per_rank)
    line = {
        "metric": METRIC + " (emulated sequence split: slowest rank)", "value": round((f_fwd + f_bwd) / (slow / 1e3) / 1e12, 2),
        "unit": "TFLOP/s", "n_gpus_emulated": W, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step_slowest_rank": round(slow, 3), "ms_per_rank": [round(t, 3) for t in per_rank],
        "max_over_mean": round(slow / (sum(per_rank) / W), 4), "cut": "balanced" if balanced else "equal",
        "chunk_bounds": ranks[0].bounds.tolist(), "items_per_rank": items.tolist(),
        "kv_bytes_received_per_rank": recv_bytes, "ring_kv_bytes": _ring(ranks[0].bounds, row),
        "dtype": "bf16", "data": "synthetic (seeded packed documents, bf16 N(0,1) Q/K/V/dO)",
        "config": {"workload": w.name, "tokens": w.n, "hq": w.hq, "hkv": w.hkv, "head_dim": w.d},
        "note": "all ranks on one GPU in turn; transfers not timed",
    }
    print(json.dumps(line), flush=True)


def _ring(bounds, row):
    from packed_sequence_causal_b200 import sap_dist
    return sap_dist.ring_bytes(bounds, row)


def run_split(args, w, rank, world, local_rank):
    """One packed batch split across the ranks: SAP (chunk per rank) or HSAP (Ulysses groups of
    --ulysses ranks, SAP across them).  Every rank builds the same seeded batch and takes its token
    block; one step = HsapAttention.forward + backward with their NCCL exchanges.  Whole-job
    TFLOP/s = the batch's unmasked FLOPs / the slowest rank's time (strong scaling: the work is
    fixed as the ranks grow).  Unmeasured on hardware in this repository: every GPU call it had
    was a single GPU."""
    import torch
    import torch.distributed as dist

    import packed_sequence_causal_b200 as sap
    from packed_sequence_causal_b200 import sap_dist

    U = args.ulysses if args.parallelism == "hsap" else 1
    if world % U:
        raise SystemExit("--ulysses must divide the number of ranks")
    S = world // U
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    b = workloads.make_batch(w, args.seed, device=str(dev), with_do=True)
    ug = sap_dist.make_hsap_groups(S, U) if world > 1 else None
    h = sap_dist.HsapAttention(b.cu_seqlens, w.n, w.hq, w.hkv, w.d, S, U, rank=rank, ulysses_group=ug,
                               balanced=not args.equal_chunks)
    lo, hi = h.block
    q, k, v, do = (t[lo:hi].contiguous() for t in (b.q, b.k, b.v, b.do))
    stream = torch.cuda.current_stream()

    def step():
        h.forward(q, k, v)
        h.backward(do)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize()
    elapsed = max_over_ranks(start.elapsed_time(end), dist if world > 1 else None, dev)
    if sap.sap_device_status() != 0:
        raise RuntimeError("device error word set after the timed steps")
    pairs = sap.sap_plan_stats(h.sap.full)["unmasked_pairs"]
    f_fwd, f_bwd = _flops(w, pairs)
    value = (f_fwd + f_bwd) * args.steps / (elapsed / 1e3) / 1e12
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(elapsed / args.steps, 3), "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded packed documents, bf16 N(0,1) Q/K/V/dO)",
            "config": {"workload": w.name, "tokens": w.n, "hq": w.hq, "hkv": w.hkv, "head_dim": w.d,
                       "parallelism": f"sap{S}" + (f"xulysses{U}" if U > 1 else ""),
                       "cut": "equal" if args.equal_chunks else "balanced"},
            "kv_bytes_received_rank0": h.sap.bytes["kv_received"], "gpu_launches": None}), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args, w, rank, world):
    """The oracle as the reference arm: fp64 on the host cores, bounded sample per step."""
    if rank != 0:
        return
    import oracle
    b = workloads.make_batch(w, args.seed, device="cpu", with_do=True)
    budget = args.cpu_budget / 3
    for _ in range(args.warmup):
        run_oracle_sample(b, budget / 4)
    times, desc, tf_all = [], "", []
    for _ in range(args.steps):
        tf, secs, desc = run_oracle_sample(b, budget)
        times.append(secs)
        tf_all.append(tf)
    _, _, flops, _ = _doc_sample(b, budget)
    value = flops * len(times) / sum(times) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * sum(times) / len(times), 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded packed documents, bf16 N(0,1) Q/K/V/dO)",
        "config": {"workload": w.name, "tokens": w.n, "hq": w.hq, "hkv": w.hkv, "head_dim": w.d, "chunks": w.p},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
