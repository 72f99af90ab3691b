#!/usr/bin/env python
"""Benchmark of the B200 MoBA prefill forward pass (one layer-forward = one step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--variant forced|shared|prefix] [--pass forward|backward|decode]
                    [--queries N]

A step runs the whole path -- block mean-pool, gate/top-k, regrouping,
history and own-block attention, merge -- on seeded synthetic inputs of the
named workload (default: the scaling-law shape, batch 4 x 8192 tokens, 16
heads, d=128, B=512, k=3, bf16). Inputs stay resident in HBM; they are larger
than the 126 MB L2, so no flush is needed between steps.

Metric: useful TFLOP/s (only QK^T and PV over the selected keys, 4*d per
query-key pair), with ms per layer-forward beside it. Under torchrun every
rank runs the same workload on its own GPU (weak scaling, no collective on
the data path); `value` is the sum of all ranks' useful FLOPs divided by the
slowest rank's time. Prints one JSON line on rank 0.

--impl reference times the fp64 CPU oracle (the only reference this method
has) on a bounded sample of the same workload on the host cores.

--variant picks the gate: forced own block (default, the headline), shared
(one choice per kv head's group, by the group's mean score) or prefix (the
own block scored by the mean of its keys up to the query). Useful FLOPs of
the prefix variant are counted from the gate's own index rows. --pass
backward times moba_backward (dq, dk, dv through the chosen blocks, on the
forward's indices): useful FLOPs 2.5x the forward's (five contractions per
query-key pair against two). --pass decode times one decode step
(moba_decode: every request's last --queries positions against its cache,
the workload's K/V) in microseconds, with the bytes it must read (the chosen
keys' K and V, the scored block means, q and out) against the HBM peak.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moba_inputs import WORKLOADS, make_inputs, sample_rows  # noqa: E402

METRIC = "moba_prefill_fwd_useful_tflops"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0}


# ------------------------------------------------------------ accounting
def flop_counts(w):
    """(useful, history part, own-block part, dense causal) FLOPs of one layer-forward."""
    useful = hist = cur = dense = 0
    d, B, k, H = w.head_dim, w.block_size, w.topk, w.num_q_heads
    for n in w.lengths:
        p = np.arange(n, dtype=np.int64)
        c = p // B
        h = np.minimum(k - 1, c)
        hist += int((4 * d * B * h).sum()) * H
        cur += int((4 * d * (p - c * B + 1)).sum()) * H
        dense += int((4 * d * (p + 1)).sum()) * H
    useful = hist + cur
    return useful, hist, cur, dense


def gate_flops(w):
    """Gate scoring FLOPs of one layer-forward, reported apart from the useful
    attention FLOPs: 2*d per (query, head, complete earlier block scored)."""
    total = 0
    for n in w.lengths:
        c = np.arange(n, dtype=np.int64) // w.block_size
        total += int(c.sum()) * 2 * w.head_dim * w.num_q_heads
    return total


def flops_from_indices(idx, cu, B, d):
    """(history, own-block) useful FLOPs of index rows idx [T, Hq, k] (device
    tensor): every chosen earlier block gives B keys, the own block, when
    chosen, keys cB..p."""
    T = idx.shape[0]
    cu64 = cu.to(idx.device, torch.int64)
    t = torch.arange(T, device=idx.device)
    b = torch.searchsorted(cu64[1:], t, right=True)
    p = t - cu64[b]
    c = (p // B)[:, None, None]
    hist = ((idx >= 0) & (idx < c)).sum().item() * B
    own = (idx == c).any(dim=2)  # [T, Hq]
    own_keys = ((p - (p // B) * B + 1)[:, None] * own).sum().item()
    return 4 * d * int(hist), 4 * d * int(own_keys)


def row_flops(w, rows):
    """Useful FLOPs of the sampled rows (row = t * Hq + h)."""
    cu = np.concatenate([[0], np.cumsum(w.lengths)])
    t = np.asarray(rows) // w.num_q_heads
    b = np.searchsorted(cu, t, side="right") - 1
    p = t - cu[b]
    c = p // w.block_size
    nkeys = np.minimum(w.topk - 1, c) * w.block_size + (p - c * w.block_size + 1)
    return int((4 * w.head_dim * nkeys).sum())


def rank_workload(w, rank: int):
    """Rank r of a weak-scaling run processes its own batch: same shapes, its
    own seed (independent problems, no collective on the data path)."""
    import dataclasses

    return dataclasses.replace(w, seed=w.seed + 7919 * rank) if rank else w


def reduce_max(x: float, world: int, device) -> float:
    """Max over ranks (slowest rank's time)."""
    if world == 1:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def profile_traffic(kernel_src: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel; else None."""
    path = os.path.join(ROOT, "profiles", f"attn_history_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    s = re.search(r"kernel_source_sha256:\s*([0-9a-f]+)", text)
    if not m or not s:
        return None
    sha = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()
    return float(m.group(1)) if sha.startswith(s.group(1)) else None


# ------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampled every 200 ms from before the warm-up to after the
    timed region; summarise() keeps the samples inside a wall-clock window."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.proc = None
        self.rows = []
        self.path = tempfile.mktemp(suffix=".csv")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={index}",
                                          f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def wait_first_sample(self, timeout=5.0):
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < timeout:
            if os.path.getsize(self.path) > 0:
                return
            time.sleep(0.05)

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        for line in open(self.path).read().strip().splitlines():
            r = [x.strip() for x in line.split(",")]
            try:
                ts = time.mktime(time.strptime(r[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + r[0].split(".")[1]) if "." in r[0] else 0.0
                self.rows.append((ts, float(r[2]), float(r[3]), r[6:10]))
            except (ValueError, IndexError):
                continue
        os.unlink(self.path)

    def summarise(self, t_lo: float, t_hi: float):
        if not self.rows:
            return None
        inside = [r for r in self.rows if t_lo - 0.25 <= r[0] <= t_hi + 0.25]
        window = "timed region"
        if not inside:
            inside, window = self.rows, "whole run (timed region shorter than the 200 ms period)"
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({nm for r in inside for nm, val in zip(names, r[3])
                          if val.lower() == "active"})
        return {"sm_mhz": float(np.median([r[1] for r in inside])),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "samples": len(inside), "window": window}


# ------------------------------------------------------------ CPU oracle leg
def time_oracle(w, q, k, v, cu, budget_s: float, seed: int = 7, n_rows=None):
    """Time the oracle on a bounded sample of rows (about budget_s seconds, or
    n_rows rows when given); returns (tflops, rows, seconds, threads)."""
    import oracle

    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    total_rows = w.total_tokens * w.num_q_heads
    if n_rows is None:
        n, dt = 64, 0.0
        while True:  # grow the sample until one call takes a measurable time
            rows = sample_rows(total_rows, n, seed).numpy()
            t0 = time.perf_counter()
            oracle.forward_rows(qc, kc, vc, cu, w.block_size, w.topk, rows)
            dt = time.perf_counter() - t0
            if dt > 0.05 * budget_s or n >= total_rows:
                break
            n = min(total_rows, n * 8)
        n2 = int(min(total_rows, max(n, n * budget_s / max(dt, 1e-3))))
    else:
        n2 = int(min(total_rows, n_rows))
    rows = sample_rows(total_rows, n2, seed + 1).numpy()
    t0 = time.perf_counter()
    oracle.forward_rows(qc, kc, vc, cu, w.block_size, w.topk, rows)
    dt = time.perf_counter() - t0
    return row_flops(w, rows) / dt / 1e12, len(rows), dt, oracle.num_threads()


# ------------------------------------------------------------ main
def bench_backward(args, w, moba, q, k, v, cu, dev, world, rank, config, shared, prefix):
    """--pass backward: moba_backward on the forward's output, lse and index rows."""
    cu_d = cu.to(dev)
    out, lse = moba.moba_forward(q, k, v, cu_d, w.block_size, w.topk, max_seqlen=w.max_seqlen,
                                 return_lse=True, shared_routing=shared, prefix_mean=prefix)
    idx = moba.moba_gate_topk(q, k, cu_d, w.block_size, w.topk, max_seqlen=w.max_seqlen,
                              shared_routing=shared, prefix_mean=prefix)
    gen = torch.Generator(device=dev).manual_seed(w.seed + 17)
    dout = (torch.randn(q.shape, generator=gen, device=dev) * 0.5).to(q.dtype)
    if prefix:
        hist, cur = flops_from_indices(idx, cu, w.block_size, w.head_dim)
    else:
        _, hist, cur, _ = flop_counts(w)
    useful = 2.5 * (hist + cur)
    p = moba.make_params(q, k, cu, w.block_size, w.topk, w.max_seqlen, shared, prefix)
    L = moba.lib()
    P = ctypes.byref(p)
    L.moba_backward_workspace_size.argtypes = [ctypes.POINTER(moba.MobaParams), ctypes.c_int]
    L.moba_backward_workspace_size.restype = ctypes.c_size_t
    fn = L.moba_backward
    fn.argtypes = [ctypes.POINTER(moba.MobaParams)] + [ctypes.c_void_p] * 12 + [ctypes.c_size_t,
                                                                              ctypes.c_void_p]
    fn.restype = ctypes.c_int
    ws = torch.empty(max(int(L.moba_backward_workspace_size(P, 1)), 256), dtype=torch.uint8,
                     device=dev)
    dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
    dk = torch.empty(k.shape, dtype=torch.float32, device=dev)
    dv = torch.empty(v.shape, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = ctypes.c_void_p(stream.cuda_stream)
    ptr = lambda x: ctypes.c_void_p(x.data_ptr())

    def step(qq=q, kk=k, vv=v, oo=out, ll=lse, dd=dout, ii=idx):
        rc = fn(P, ptr(qq), ptr(kk), ptr(vv), ptr(cu_d), ptr(oo), ptr(ll), ptr(dd), ptr(ii),
                ptr(dq), ptr(dk), ptr(dv), ptr(ws), ws.numel(), sp)
        if rc:
            raise RuntimeError(f"moba_backward failed: {rc}")

    clocks = ClockSampler(dev.index) if rank == 0 else None
    if clocks:
        clocks.wait_first_sample()
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    if moba.moba_device_status(dev) != 0:
        raise RuntimeError("device status error after warm-up")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t_lo = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    t_hi = time.time()
    if world > 1:
        torch.distributed.barrier()
    if clocks:
        clocks.stop()
    clock_info = clocks.summarise(t_lo, t_hi) if clocks else None
    ms = reduce_max(e0.elapsed_time(e1) / args.steps, world, dev)

    # end to end: the step's inputs from pinned host memory, the gradients back
    host_in = [x.cpu().pin_memory() for x in (q, k, v, out, lse, dout, idx)]
    dev_in = [torch.empty_like(x) for x in (q, k, v, out, lse, dout, idx)]
    host_out = [torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in (dq, dk, dv)]

    def e2e_step():
        for d_, h_ in zip(dev_in, host_in):
            d_.copy_(h_, non_blocking=True)
        step(*dev_in)
        for h_, d_ in zip(host_out, (dq, dk, dv)):
            h_.copy_(d_, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    erep = max(3, min(args.steps, 10))
    e0.record(stream)
    for _ in range(erep):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = reduce_max(e0.elapsed_time(e1) / erep, world, dev)
    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    value = useful * world / (ms * 1e-3) / 1e12
    line = {
        "metric": "moba_prefill_bwd_useful_tflops", "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": dict(config, **{"pass": "backward"}),
        "roofline": {"bound": "tensor", "achieved": value / world, "peak": peak,
                     "unit": "TFLOP/s", "frac": value / world / peak, "traffic": None,
                     "kernel": "moba_backward, all launches (a lower bound for each kernel)",
                     "peak_source": f"{peak_src} bf16 burst"},
        "cpu_baseline": None,
        "e2e": {"value": useful * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in host_in),
                "d2h_bytes_per_step": sum(x.numel() * x.element_size() for x in host_out)},
        # regroup (4), D = dO . O, the history and own-block kernels
        "gpu_launches": 7 * args.steps,
        "clocks": clock_info,
        "useful_flop_per_step": useful,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def bench_decode(args, w, moba, q_all, k, v, cu, dev, world, rank, config, shared):
    """--pass decode: one decode step = every request's last --queries positions against its
    cache (the workload's K/V), through moba_decode; the block means are built once, as a
    serving loop keeps them up to date incrementally."""
    nq_r = args.queries
    lens = np.diff(cu.numpy())
    if (lens < nq_r).any():
        raise ValueError("--queries exceeds a sequence length")
    Hq, d = q_all.shape[1], q_all.shape[2]
    tok = torch.cat([torch.arange(int(cu[r + 1]) - nq_r, int(cu[r + 1])) for r in range(w.batch)])
    q = q_all[tok.to(dev)].contiguous()
    del q_all
    cu_d = cu.to(dev)
    cu_q = torch.arange(0, (w.batch + 1) * nq_r, nq_r, dtype=torch.int32)
    kbar = moba.moba_meanpool(k, cu_d, w.block_size, max_seqlen=w.max_seqlen)
    p = moba.decode_params(q, k, cu, w.block_size, w.topk, w.max_seqlen, shared)
    L = moba.lib()
    L.moba_decode_workspace_size.argtypes = [ctypes.POINTER(moba.MobaParams), ctypes.c_int]
    L.moba_decode_workspace_size.restype = ctypes.c_size_t
    n = q.shape[0]
    ws = torch.empty(max(int(L.moba_decode_workspace_size(ctypes.byref(p), n)), 256),
                     dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    idx = torch.empty((n, Hq, w.topk), dtype=torch.int32, device=dev)
    cu_qd = cu_q.to(dev)
    stream = torch.cuda.current_stream(dev)
    sp = ctypes.c_void_p(stream.cuda_stream)
    fn = L.moba_decode
    V = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(moba.MobaParams), V, V, V, V, V, ctypes.c_int, V, V, V, V, V,
                   ctypes.c_size_t, V]
    fn.restype = ctypes.c_int
    P = ctypes.byref(p)
    ptr = lambda x: ctypes.c_void_p(x.data_ptr())

    def step(qq=q, oo=out):
        rc = fn(P, ptr(qq), ptr(k), ptr(v), ptr(cu_d), ptr(cu_qd), n, ptr(kbar), ptr(oo), None,
                ptr(idx), ptr(ws), ws.numel(), sp)
        if rc:
            raise RuntimeError(f"moba_decode failed: {rc}")

    clocks = ClockSampler(dev.index) if rank == 0 else None
    if clocks:
        clocks.wait_first_sample()
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    if moba.moba_device_status(dev) != 0:
        raise RuntimeError("device status error after warm-up")
    # bytes the step must read: the chosen keys' K and V rows of every (query, q head), the
    # block means it scores and the query rows (output written once)
    pos = (torch.as_tensor(lens, device=dev).repeat_interleave(nq_r) - nq_r
           + torch.arange(nq_r, device=dev).repeat(w.batch))  # [n] positions
    c = (pos // w.block_size)[:, None, None]
    nkeys = (((idx >= 0) & (idx < c)).sum() * w.block_size
             + (((pos - (pos // w.block_size) * w.block_size + 1)[:, None]) * (idx == c).any(2)).sum())
    esz = k.element_size()
    kv_bytes = int(nkeys.item()) * 2 * d * esz
    gate_bytes = int((pos // w.block_size).sum().item()) * (Hq if not shared else w.num_kv_heads) * d * 4
    io_bytes = 2 * q.numel() * esz
    alg_bytes = kv_bytes + gate_bytes + io_bytes
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t_lo = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    t_hi = time.time()
    if world > 1:
        torch.distributed.barrier()
    if clocks:
        clocks.stop()
    clock_info = clocks.summarise(t_lo, t_hi) if clocks else None
    ms = reduce_max(e0.elapsed_time(e1) / args.steps, world, dev)
    # end to end: the step's query rows in from pinned memory, the outputs back
    hq = q.cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dq = torch.empty_like(q)

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        step(dq, out)
        hout.copy_(out, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    erep = max(3, min(args.steps, 20))
    e0.record(stream)
    for _ in range(erep):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = reduce_max(e0.elapsed_time(e1) / erep, world, dev)
    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    peaks, peak_src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    achieved = alg_bytes / (ms * 1e-3) / 1e9
    line = {
        "metric": "moba_decode_step_us", "value": ms * 1e3, "unit": "us",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": dict(config, **{"pass": "decode", "queries_per_request": nq_r}),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": None,
                     "kernel": "moba_decode, all launches (gate, split-K attention with the merge)",
                     "algorithmic_bytes": alg_bytes, "peak_source": f"{peak_src} HBM copy"},
        "cpu_baseline": None,
        "e2e": {"value": e2e_ms * 1e3, "unit": "us", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": hq.numel() * hq.element_size(),
                "d2h_bytes_per_step": hout.numel() * hout.element_size()},
        "gpu_launches": 2 * args.steps,
        "clocks": clock_info,
        "queries_per_step": n,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="scaling_8k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--variant", default="forced", choices=["forced", "shared", "prefix"])
    ap.add_argument("--pass", dest="pass_", default="forward",
                    choices=["forward", "backward", "decode"])
    ap.add_argument("--queries", type=int, default=1, help="decode: queries per request")
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    useful, hist_flops, cur_flops, dense_flops = flop_counts(w)
    elem = 2 if w.dtype == torch.bfloat16 else 4
    in_bytes = w.total_tokens * (w.num_q_heads + 2 * w.num_kv_heads) * w.head_dim * elem
    l2_note = ("inputs exceed L2 (q+k+v > 126 MB), no flush" if in_bytes > 126 * 2**20 else
               f"inputs ({in_bytes / 2**20:.1f} MiB) fit in L2 and stay warm between steps")
    config = {"workload": w.name, "batch": w.batch, "seq_lens": list(w.lengths),
              "q_heads": w.num_q_heads, "kv_heads": w.num_kv_heads, "head_dim": w.head_dim,
              "block_size": w.block_size, "topk": w.topk, "l2": l2_note}
    if args.variant != "forced":
        config["variant"] = args.variant
    dtype_name = "bf16" if w.dtype == torch.bfloat16 else "f32"

    if args.impl == "reference":
        if rank != 0:
            return
        q, k, v, cu = make_inputs(w, "cpu")
        per_step = []
        # about two minutes of oracle work for the whole run, at most 2 s a step;
        # the first step sizes the row sample, the others reuse its size
        n_steps = args.warmup + args.steps
        budget = min(2.0, max(0.05, 120.0 / max(1, n_steps)))
        n_rows = None
        for _ in range(n_steps):
            tf, nrows, dt, thr = time_oracle(w, q, k, v, cu, budget_s=budget, n_rows=n_rows)
            n_rows = nrows
            per_step.append((tf, nrows, dt))
        per_step = per_step[args.warmup:]
        tf = float(np.mean([x[0] for x in per_step]))
        ms = float(np.mean([x[2] for x in per_step])) * 1e3
        line = {"impl": "reference", "metric": METRIC, "value": tf, "unit": "TFLOP/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "cpu_baseline": {"kind": "oracle", "value": tf, "unit": "TFLOP/s", "cores": thr,
                                 "sample": f"{per_step[0][1]} seeded (token, head) rows per step "
                                           f"of {w.name}, useful FLOPs of those rows"},
                "e2e": {"value": tf, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import long_context_prefill_block_b200 as moba

    if world > 1:
        import torch.distributed as dist
        import datetime

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    q, k, v, cu = make_inputs(rank_workload(w, rank), dev)
    cu_d = cu.to(dev)
    shared, prefix = args.variant == "shared", args.variant == "prefix"
    if args.pass_ == "backward":
        return bench_backward(args, w, moba, q, k, v, cu, dev, world, rank, config, shared, prefix)
    if args.pass_ == "decode":
        if prefix:
            raise ValueError("the decode step takes the forced own block only")
        return bench_decode(args, w, moba, q, k, v, cu, dev, world, rank, config, shared)
    p = moba.make_params(q, k, cu, w.block_size, w.topk, w.max_seqlen, shared, prefix)
    ws = moba.workspace(p, dev)
    if prefix:
        idx0 = moba.moba_gate_topk(q, k, cu_d, w.block_size, w.topk, max_seqlen=w.max_seqlen,
                                   prefix_mean=True)
        hist_flops, cur_flops = flops_from_indices(idx0, cu, w.block_size, w.head_dim)
        useful = hist_flops + cur_flops
        del idx0
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)
    L = moba.lib()
    P = ctypes.byref(p)
    sp = ctypes.c_void_p(stream.cuda_stream)

    def step():
        rc = L.moba_forward(P, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                            ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(cu_d.data_ptr()),
                            ctypes.c_void_p(out.data_ptr()), None, ctypes.c_void_p(ws.data_ptr()),
                            ws.numel(), sp)
        if rc:
            raise RuntimeError(f"moba_forward failed: {rc}")

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, world, dev)

    clocks = ClockSampler(dev.index) if rank == 0 else None
    if clocks:
        clocks.wait_first_sample()
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    if moba.moba_device_status(dev) != 0:
        raise RuntimeError("device status error after warm-up")

    # ---- timed region: K steps, barrier + sync on both sides
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    t_lo = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    t_hi = time.time()
    barrier()
    if clocks:
        clocks.stop()
    clock_info = clocks.summarise(t_lo, t_hi) if clocks else None
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
    value = useful * world / (ms * 1e-3) / 1e12

    # ---- per-stage timing (same stream, CUDA events recorded by the library)
    n_pass = L.moba_num_passes(P)
    n_ev = 3 + 4 * n_pass
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    for e in evs:  # torch creates the CUDA event on first record
        e.record(stream)
    torch.cuda.synchronize(dev)
    ev_arr = (ctypes.c_void_p * n_ev)(*[ctypes.c_void_p(e.cuda_event) for e in evs])
    stage_ms = {"meanpool": 0.0, "gate_topk": 0.0, "regroup": 0.0, "attn_history": 0.0,
                "attn_current": 0.0, "merge": 0.0}
    reps = max(3, min(args.steps, 10))
    for _ in range(reps):
        rc = L.moba_forward_staged(P, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                   ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(cu_d.data_ptr()),
                                   ctypes.c_void_p(out.data_ptr()), None,
                                   ctypes.c_void_p(ws.data_ptr()), ws.numel(), ev_arr, n_ev, sp)
        if rc:
            raise RuntimeError(f"moba_forward_staged failed: {rc}")
        torch.cuda.synchronize(dev)
        stage_ms["meanpool"] += evs[0].elapsed_time(evs[1]) / reps
        stage_ms["gate_topk"] += evs[1].elapsed_time(evs[2]) / reps
        prev = evs[2]
        for j in range(n_pass):
            a, b_, c_, d_ = evs[3 + 4 * j: 7 + 4 * j]
            stage_ms["regroup"] += prev.elapsed_time(a) / reps
            stage_ms["attn_history"] += a.elapsed_time(b_) / reps
            stage_ms["attn_current"] += b_.elapsed_time(c_) / reps
            stage_ms["merge"] += c_.elapsed_time(d_) / reps
            prev = d_

    # ---- dense causal comparison at the same shape
    # (seconds-long dense passes, as at the million-token shape: one warm-up, one timed)
    long_dense = ms > 200.0
    dense_out = torch.empty_like(q)
    for _ in range(1 if long_dense else 2):
        moba.dense_causal_forward(q, k, v, cu, max_seqlen=w.max_seqlen, out=dense_out)
    torch.cuda.synchronize(dev)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dreps = 1 if long_dense else 3
    d0.record(stream)
    for _ in range(dreps):
        moba.dense_causal_forward(q, k, v, cu, max_seqlen=w.max_seqlen, out=dense_out)
    d1.record(stream)
    torch.cuda.synchronize(dev)
    dense_ms = d0.elapsed_time(d1) / dreps
    del dense_out

    # ---- end to end through the public API with host buffers
    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    hout = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def e2e_step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        rc = L.moba_forward(P, ctypes.c_void_p(dq.data_ptr()), ctypes.c_void_p(dk.data_ptr()),
                            ctypes.c_void_p(dv.data_ptr()), ctypes.c_void_p(cu_d.data_ptr()),
                            ctypes.c_void_p(out.data_ptr()), None, ctypes.c_void_p(ws.data_ptr()),
                            ws.numel(), sp)
        if rc:
            raise RuntimeError(f"moba_forward failed: {rc}")
        hout.copy_(out, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    erep = max(3, min(args.steps, 10))
    barrier()
    e0.record(stream)
    for _ in range(erep):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / erep)
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
    d2h = hout.numel() * hout.element_size()

    peaks, peak_src = load_peaks()
    hist_launch_ms = stage_ms["attn_history"] / n_pass
    hist_launch_flops = hist_flops / n_pass
    achieved = hist_launch_flops / (hist_launch_ms * 1e-3) / 1e12 if hist_launch_ms > 0 else 0.0
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    # the attention kernels together: history, own block (with its merge), merge
    attn_ms = stage_ms["attn_history"] + stage_ms["attn_current"] + stage_ms["merge"]
    attn_tflops = useful / (attn_ms * 1e-3) / 1e12 if attn_ms > 0 else 0.0
    traffic = profile_traffic(os.path.join(ROOT, "long_context_prefill_block_b200", "csrc",
                                           "attn_tc.cu"), w.name)
    tc_path = w.dtype == torch.bfloat16 and w.head_dim == 128 and w.block_size % 128 == 0
    # mean-pool, gate; per pass: 4 regroup kernels, history, own-block (+ merge on the SIMT path)
    launches_per_step = 2 + (6 if tc_path else 7) * n_pass
    if prefix:  # the own-block scores: chunk key sums, then the dot products
        launches_per_step += 2

    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline and args.variant == "forced":
        tf, nrows, dt, thr = time_oracle(w, q, k, v, cu, args.cpu_budget)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
               "sample": f"{nrows} seeded (token, head) rows of {w.name} ({dt:.1f} s), "
                         "useful FLOPs of those rows"}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype_name,
        "data": "synthetic", "config": config,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "attn_history", "peak_source": f"{peak_src} bf16 burst"},
        "cpu_baseline": cpu,
        "e2e": {"value": useful * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clock_info,
        "stage_ms": stage_ms,
        "useful_flop_per_step": useful,
        "gate_flop_per_step": gate_flops(w),
        "dense_causal_ms": dense_ms,
        "speedup_vs_dense": dense_ms / ms,
        "frac_of_peak_end_to_end": value / world / peak,
        "attn_kernels_tflops": attn_tflops,
        "attn_kernels_frac_of_peak": attn_tflops / peak,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
