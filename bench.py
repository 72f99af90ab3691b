#!/usr/bin/env python
"""Benchmark of the B200 MoBA prefill forward pass (one layer-forward = one step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--variant forced|shared|prefix] [--pass forward|backward|decode]
                    [--queries N]

A step runs the whole path -- block mean-pool, gate/top-k, regrouping,
history and own-block attention, merge -- on seeded synthetic inputs of the
named workload (default: the Llama-3.1-8B million-token prefill shape, 1 x
1,048,576 tokens, 32 q / 8 kv heads, d=128, B=4096, k=12, bf16: the largest
workload that fits one GPU). Inputs stay resident in HBM; they are larger
than the 126 MB L2, so no flush is needed between steps.

Metric: useful TFLOP/s (only QK^T and PV over the selected keys, 4*d per
query-key pair), with ms per layer-forward beside it. Under torchrun every
rank runs the same workload on its own GPU (weak scaling, no collective on
the data path); `value` is the sum of all ranks' useful FLOPs divided by the
slowest rank's time. Prints one JSON line on rank 0.

The roofline fraction divides by the measured bf16 peak: the sustained
figure when the timed region lasts a second or more (the kernel then runs
under the power cap), else the burst figure; both fractions are reported.

--impl reference times the fp64 CPU oracle (the only reference this method
has) on a bounded sample of the same workload on the host cores, with the
same input bits as the GPU arm (drawn on the GPU when one is present; only
K, V and the sampled q rows are copied to the host).

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
import concurrent.futures as cf
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
SIDE_WORKLOADS = ("long_32k", "micro_32k")
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
DEFAULT_WORKLOAD = "llama_1m"
TIE_GAP = 1e-4  # near-tie band of the block indices (relative score gap)


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


def history_pairs(w):
    """(query, head, chosen earlier block) entries of one forward with the forced own block."""
    total = 0
    for n in w.lengths:
        c = np.arange(n, dtype=np.int64) // w.block_size
        total += int(np.minimum(w.topk - 1, c).sum()) * w.num_q_heads
    return total


def stage_bytes(w):
    """Algorithmic HBM bytes of the memory-bound stages of one forward:
    mean-pool reads K once and writes the block means; the gate reads Q once
    and writes the index rows; regroup reads the index rows twice (count and
    scatter passes) and writes one 4-byte entry per history pair."""
    esz = 2 if w.dtype == torch.bfloat16 else 4
    T, Hq, Hkv, d, k = w.total_tokens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.topk
    nb = sum((n + w.block_size - 1) // w.block_size for n in w.lengths)
    idx_bytes = T * Hq * k * 4
    return {"meanpool": T * Hkv * d * esz + nb * Hkv * d * 4,
            "gate_topk": T * Hq * d * esz + idx_bytes,
            "regroup": 2 * idx_bytes + 4 * history_pairs(w)}


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


def tensor_peak(peaks, timed_s: float):
    """(peak TFLOP/s, which one): the sustained bf16 figure for a timed region
    of a second or more (the GPU then runs under its power cap), else the
    burst figure."""
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    return (sustained, "sustained") if timed_s >= 1.0 else (burst, "burst")


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


def sha256_of(t: torch.Tensor) -> str:
    """SHA-256 of a host tensor's stored bytes."""
    x = t.detach().contiguous()
    if x.dtype == torch.bfloat16:
        x = x.view(torch.int16)
    return hashlib.sha256(memoryview(x.numpy()).cast("B")).hexdigest()


def input_hashes(named):
    """{name: sha256} of host tensors, hashed in parallel (hashlib releases the GIL)."""
    with cf.ThreadPoolExecutor(max_workers=len(named)) as ex:
        futs = {n: ex.submit(sha256_of, t) for n, t in named.items()}
        return {n: f.result() for n, f in futs.items()}


def pinned_copy(x: torch.Tensor) -> torch.Tensor:
    h = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    h.copy_(x)
    return h


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
def q_rows_from(q: torch.Tensor):
    """Function rows -> the host copy of those q rows (row = t * Hq + h) of q,
    which may live on the GPU: only the sampled rows cross to the host."""
    flat = q.reshape(-1, q.shape[-1])

    def take(rows):
        sel = torch.as_tensor(np.asarray(rows, dtype=np.int64), device=q.device)
        return flat[sel].cpu()

    return take


def time_oracle(w, kc, vc, cu, q_rows_of, budget_s: float, seed: int = 7, n_rows=None):
    """Time the oracle on a bounded sample of rows (about budget_s seconds, or
    n_rows rows when given). kc, vc: host K and V; q_rows_of(rows): host q rows.
    Returns dict(tflops, rows, seconds, threads, result=(out, lse, idx, gap), q_rows)."""
    import oracle

    total_rows = w.total_tokens * w.num_q_heads

    def run(rows):
        qr = q_rows_of(rows)
        t0 = time.perf_counter()
        res = oracle.forward_rows(None, kc, vc, cu, w.block_size, w.topk, rows, q_rows=qr,
                                  num_q_heads=w.num_q_heads)
        return res, qr, time.perf_counter() - t0

    if n_rows is None:
        n = 64
        while True:  # grow the sample until one call takes a measurable time
            _, _, dt = run(sample_rows(total_rows, n, seed).numpy())
            if dt > 0.05 * budget_s or n >= total_rows:
                break
            n = min(total_rows, n * 8)
        n2 = int(min(total_rows, max(n, n * budget_s / max(dt, 1e-3))))
    else:
        n2 = int(min(total_rows, n_rows))
    rows = sample_rows(total_rows, n2, seed + 1).numpy()
    res, qr, dt = run(rows)
    return {"tflops": row_flops(w, rows) / dt / 1e12, "rows": rows, "seconds": dt,
            "threads": oracle.num_threads(), "result": res, "q_rows": qr}


def parity_stats(w, leg, kc, vc, cu, got_out, got_lse, got_idx):
    """The GPU forward against the oracle on the CPU leg's sampled rows:
    output and lse errors, index mismatches (and how many fall outside the
    near-tie band), near-tie count and a histogram of the top-k margins (the
    oracle's relative score gap between the last chosen and the first rejected
    earlier block; "none" where no earlier block was rejected)."""
    import oracle

    ref, ref_lse, ref_idx, gap = (np.array(x) for x in leg["result"])
    rows = leg["rows"]
    mism = np.nonzero((got_idx != ref_idx).any(axis=1))[0]
    beyond = int((gap[mism] >= TIE_GAP).sum())
    if len(mism):
        # near-tie rows: the oracle with the GPU's own choice
        o2, l2, _, _ = oracle.forward_rows(None, kc, vc, cu, w.block_size, w.topk, rows[mism],
                                           indices=got_idx[mism], q_rows=leg["q_rows"][mism],
                                           num_q_heads=w.num_q_heads)
        ref[mism] = o2
        ref_lse[mism] = l2
    err = np.abs(got_out.astype(np.float64) - ref)
    lerr = np.abs(got_lse.astype(np.float64) - ref_lse)
    finite = gap[np.isfinite(gap)]
    edges = [0.0, 1e-6, 1e-5, 1e-4, 1e-3, 1e-2, 1e-1, np.inf]
    names = ["<1e-6", "1e-6..1e-5", "1e-5..1e-4", "1e-4..1e-3", "1e-3..1e-2", "1e-2..1e-1",
             ">=1e-1"]
    counts, _ = np.histogram(finite, bins=edges)
    hist = {n: int(c) for n, c in zip(names, counts)}
    hist["none"] = int((~np.isfinite(gap)).sum())
    tol = (2e-2, 2e-3) if w.dtype == torch.bfloat16 else (1e-4, 1e-4)
    return {"rows": int(len(rows)), "max_abs_err": float(err.max()),
            "mean_abs_err": float(err.mean()), "lse_max_abs_err": float(lerr.max()),
            "index_mismatch_rows": int(len(mism)), "index_mismatch_beyond_tie": beyond,
            "near_tie_rows": int((gap < TIE_GAP).sum()), "topk_margin_hist": hist,
            "tolerance": {"max_abs": tol[0], "mean_abs": tol[1], "tie_gap": TIE_GAP},
            "pass": bool(beyond == 0 and err.max() <= tol[0] and err.mean() <= tol[1])}


def reference_inputs(w):
    """Inputs of the reference arm with the GPU arm's bits: drawn on the GPU
    when one is present (then only K, V and sampled q rows go to the host),
    else on the host."""
    if torch.cuda.is_available():
        dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
        torch.cuda.set_device(dev)
        q, k, v, cu = make_inputs(w, dev)
        kc, vc = k.cpu(), v.cpu()
        del k, v
        return q, kc, vc, cu, "drawn on the GPU (the GPU arm's bits)"
    q, k, v, cu = make_inputs(w, "cpu")
    return q, k, v, cu, "drawn on the host (no GPU present)"


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
    host_in = [pinned_copy(x) for x in (q, k, v, out, lse, dout, idx)]
    dev_in = [torch.empty_like(x) for x in (q, k, v, out, lse, dout, idx)]
    host_out = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in (dq, dk, dv)]

    def e2e_step():
        for d_, h_ in zip(dev_in, host_in):
            d_.copy_(h_, non_blocking=True)
        step(*dev_in)
        for h_, d_ in zip(host_out, (dq, dk, dv)):
            h_.copy_(d_, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    erep = 3 if ms > 100 else max(3, min(args.steps, 10))
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
    peak, which = tensor_peak(peaks, ms * args.steps * 1e-3)
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
                     "peak_source": f"{peak_src} bf16 {which}"},
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
    hm = args.kv_layout == "head"
    lens = np.diff(cu.numpy())
    if (lens < nq_r).any():
        raise ValueError("--queries exceeds a sequence length")
    Hq, d = q_all.shape[1], q_all.shape[2]
    tok = torch.cat([torch.arange(int(cu[r + 1]) - nq_r, int(cu[r + 1])) for r in range(w.batch)])
    q = q_all[tok.to(dev)].contiguous()
    del q_all
    cu_d = cu.to(dev)
    cu_q = torch.arange(0, (w.batch + 1) * nq_r, nq_r, dtype=torch.int32)
    if hm:  # the cache laid out head by head: [Hkv, T, d]
        k, v = k.transpose(0, 1).contiguous(), v.transpose(0, 1).contiguous()
    kbar = moba.moba_meanpool(k, cu_d, w.block_size, max_seqlen=w.max_seqlen, kv_head_major=hm)
    p = moba.decode_params(q, k, cu, w.block_size, w.topk, w.max_seqlen, shared, kv_head_major=hm)
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
    hq = pinned_copy(q)
    hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
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
        "config": dict(config, **{"pass": "decode", "queries_per_request": nq_r,
                                  "kv_layout": "head-major [Hkv, T, d]" if hm else
                                  "packed [T, Hkv, d]"}),
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


def stage_times(L, P, bufs, stream, dev, reps: int):
    """Per-stage milliseconds of moba_forward_staged: CUDA events the library
    records on the launching stream between its stages, mean of `reps` calls."""
    q, k, v, cu_d, out, ws = bufs
    vp = lambda x: ctypes.c_void_p(x.data_ptr())
    n_pass = L.moba_num_passes(P)
    n_ev = 3 + 4 * n_pass
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    for e in evs:  # torch creates the CUDA event on first record
        e.record(stream)
    torch.cuda.synchronize(dev)
    ev_arr = (ctypes.c_void_p * n_ev)(*[ctypes.c_void_p(e.cuda_event) for e in evs])
    stage_ms = {"meanpool": 0.0, "gate_topk": 0.0, "regroup": 0.0, "attn_history": 0.0,
                "attn_current": 0.0, "merge": 0.0}
    sp = ctypes.c_void_p(stream.cuda_stream)
    for _ in range(reps):
        rc = L.moba_forward_staged(P, vp(q), vp(k), vp(v), vp(cu_d), vp(out), None, vp(ws),
                                   ws.numel(), ev_arr, n_ev, sp)
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
    return stage_ms


def side_workload(name: str, moba, dev, burst: float):
    """The forward at another workload, timed like the headline one (CUDA events,
    3 warm-up steps, about a second of timed steps; inputs larger than L2), with
    its attention-kernel fraction of the burst peak and the dense causal time, so
    that the 32K shapes sit beside the million-token line in one run."""
    w = WORKLOADS[name]
    q, k, v, cu = make_inputs(w, dev)
    cu_d = cu.to(dev)
    p = moba.make_params(q, k, cu, w.block_size, w.topk, w.max_seqlen)
    ws = moba.workspace(p, dev)
    out = torch.empty_like(q)
    L, P = moba.lib(), ctypes.byref(p)
    stream = torch.cuda.current_stream(dev)
    sp = ctypes.c_void_p(stream.cuda_stream)
    vp = lambda x: ctypes.c_void_p(x.data_ptr())

    def step():
        rc = L.moba_forward(P, vp(q), vp(k), vp(v), vp(cu_d), vp(out), None, vp(ws), ws.numel(),
                            sp)
        if rc:
            raise RuntimeError(f"moba_forward failed: {rc}")

    t_w = time.perf_counter()
    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    warm_s = (time.perf_counter() - t_w) / 3
    steps = int(min(200, max(5, round(1.0 / max(warm_s, 1e-4)))))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if moba.moba_device_status(dev) != 0:
        raise RuntimeError(f"device status error at {name}")
    ms = e0.elapsed_time(e1) / steps
    useful, hist_flops, _, _ = flop_counts(w)
    st = stage_times(L, P, (q, k, v, cu_d, out, ws), stream, dev, 5)
    attn_ms = st["attn_history"] + st["attn_current"] + st["merge"]
    dense = torch.empty_like(q)
    moba.dense_causal_forward(q, k, v, cu, max_seqlen=w.max_seqlen, out=dense)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for _ in range(3):
        moba.dense_causal_forward(q, k, v, cu, max_seqlen=w.max_seqlen, out=dense)
    d1.record(stream)
    torch.cuda.synchronize(dev)
    dense_ms = d0.elapsed_time(d1) / 3
    return {"ms_per_step": ms, "steps": steps, "useful_tflops": useful / (ms * 1e-3) / 1e12,
            "attn_kernels_frac_of_burst": useful / (attn_ms * 1e-3) / 1e12 / burst,
            "history_frac_of_burst": hist_flops / (st["attn_history"] * 1e-3) / 1e12 / burst,
            "stage_ms": st, "dense_causal_ms": dense_ms, "speedup_vs_dense": dense_ms / ms}


def run_reference(args, w, config):
    """--impl reference: the fp64 oracle on the host cores, each step a
    bounded seeded row sample of the workload, same input bits as the GPU arm."""
    q, kc, vc, cu, origin = reference_inputs(w)
    take = q_rows_from(q)
    per_step = []
    # about two minutes of oracle work for the whole run, at most 2 s a step;
    # the first step sizes the row sample, the others reuse its size
    n_steps = args.warmup + args.steps
    budget = min(2.0, max(0.05, 120.0 / max(1, n_steps)))
    n_rows = None
    thr = 0
    for i in range(n_steps):
        leg = time_oracle(w, kc, vc, cu, take, budget_s=budget, n_rows=n_rows, seed=7 + i)
        n_rows = len(leg["rows"])
        thr = leg["threads"]
        per_step.append((leg["tflops"], n_rows, leg["seconds"]))
    per_step = per_step[args.warmup:]
    tf = float(np.mean([x[0] for x in per_step]))
    ms = float(np.mean([x[2] for x in per_step])) * 1e3
    line = {"impl": "reference", "metric": METRIC, "value": tf, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "cpu_baseline": {"kind": "oracle", "value": tf, "unit": "TFLOP/s", "cores": thr,
                             "sample": f"{per_step[0][1]} seeded (token, head) rows per step "
                                       f"of {w.name} (inputs {origin}), useful FLOPs of those "
                                       "rows"},
            "e2e": {"value": tf, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: about 10 s of work, 3..400 steps)")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-hash", action="store_true", help="skip the input SHA-256s")
    ap.add_argument("--no-side", action="store_true",
                    help="skip the forward at the 32K shapes beside the headline workload")
    ap.add_argument("--variant", default="forced", choices=["forced", "shared", "prefix"])
    ap.add_argument("--pass", dest="pass_", default="forward",
                    choices=["forward", "backward", "decode"])
    ap.add_argument("--queries", type=int, default=1, help="decode: queries per request")
    ap.add_argument("--kv-layout", default="packed", choices=["packed", "head"],
                    help="decode: the KV cache packed [T, Hkv, d] or head-major [Hkv, T, d]")
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
        if args.steps is None:
            args.steps = 10
        return run_reference(args, w, config)

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
        args.steps = args.steps or 20
        return bench_backward(args, w, moba, q, k, v, cu, dev, world, rank, config, shared, prefix)
    if args.pass_ == "decode":
        if prefix:
            raise ValueError("the decode step takes the forced own block only")
        args.steps = args.steps or 200
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
    vp = lambda x: ctypes.c_void_p(x.data_ptr())

    def forward(qq, kk, vv, oo, s=sp):
        rc = L.moba_forward(P, vp(qq), vp(kk), vp(vv), vp(cu_d), vp(oo), None, vp(ws),
                            ws.numel(), s)
        if rc:
            raise RuntimeError(f"moba_forward failed: {rc}")

    def step():
        forward(q, k, v, out)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, world, dev)

    clocks = ClockSampler(dev.index) if rank == 0 else None
    if clocks:
        clocks.wait_first_sample()
    t_w = time.perf_counter()
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    warm_s = (time.perf_counter() - t_w) / max(args.warmup, 3)
    if moba.moba_device_status(dev) != 0:
        raise RuntimeError("device status error after warm-up")
    if args.steps is None:  # about ten seconds of timed work, 3 to 400 steps
        args.steps = int(min(400, max(3, round(10.0 / max(warm_s, 1e-4)))))
        args.steps = int(max_over_ranks(args.steps))

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
    long_step = ms > 100.0

    # ---- per-stage timing (same stream, CUDA events recorded by the library)
    n_pass = L.moba_num_passes(P)
    reps = 3 if long_step else max(3, min(args.steps, 10))
    stage_ms = stage_times(L, P, (q, k, v, cu_d, out, ws), stream, dev, reps)

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

    # ---- end to end through the C ABI with host buffers: every step copies
    # its q, k, v in from pinned host memory and its output back. Two device
    # buffer sets let step i+1's input copies and step i-1's output copy run
    # on their own streams while step i computes.
    hq, hk, hv = (pinned_copy(x) for x in (q, k, v))
    hout = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    bufs = [(q, k, v, out), tuple(torch.empty_like(x) for x in (q, k, v, out))]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_fwd = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    started = [False, False]

    def e2e_steps(n):
        for i in range(n):
            s = i % 2
            bq, bk, bv, bo = bufs[s]
            if i == 0:
                s_in.wait_stream(stream)  # the copies start after the timing event
            if started[s]:
                s_in.wait_event(ev_fwd[s])  # the forward that last read this buffer set
            with torch.cuda.stream(s_in):
                bq.copy_(hq, non_blocking=True)
                bk.copy_(hk, non_blocking=True)
                bv.copy_(hv, non_blocking=True)
                ev_in[s].record(s_in)
            stream.wait_event(ev_in[s])
            if started[s]:
                stream.wait_event(ev_out[s])  # the output copy that last read this buffer
            forward(bq, bk, bv, bo)
            ev_fwd[s].record(stream)
            s_out.wait_event(ev_fwd[s])
            with torch.cuda.stream(s_out):
                hout.copy_(bo, non_blocking=True)
                ev_out[s].record(s_out)
            started[s] = True
        stream.wait_stream(s_out)

    e2e_steps(2)
    torch.cuda.synchronize(dev)
    erep = 3 if long_step else max(3, min(args.steps, 10))
    barrier()
    e0.record(stream)
    e2e_steps(erep)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / erep)
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
    d2h = hout.numel() * hout.element_size()
    del bufs

    peaks, peak_src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    peak, which = tensor_peak(peaks, ms * args.steps * 1e-3)
    hist_launch_ms = stage_ms["attn_history"] / n_pass
    hist_launch_flops = hist_flops / n_pass
    achieved = hist_launch_flops / (hist_launch_ms * 1e-3) / 1e12 if hist_launch_ms > 0 else 0.0
    # the attention kernels together: history, own block (with its merge), merge
    attn_ms = stage_ms["attn_history"] + stage_ms["attn_current"] + stage_ms["merge"]
    attn_tflops = useful / (attn_ms * 1e-3) / 1e12 if attn_ms > 0 else 0.0
    traffic = profile_traffic(os.path.join(ROOT, "long_context_prefill_block_b200", "csrc",
                                           "attn_tc.cu"), w.name)
    sb = stage_bytes(w)
    stage_hbm = {}
    for name, nbytes in sb.items():
        t_ms = stage_ms[name]
        gbs = nbytes / (t_ms * 1e-3) / 1e9 if t_ms > 0 else 0.0
        stage_hbm[name] = {"algorithmic_bytes": nbytes, "gbs": gbs, "frac_of_hbm": gbs / hbm}
    tc_path = w.dtype == torch.bfloat16 and w.head_dim == 128 and w.block_size % 128 == 0
    # mean-pool, gate; per pass: 4 regroup kernels, history, own-block (+ merge on the SIMT path)
    launches_per_step = 2 + (6 if tc_path else 7) * n_pass
    if prefix:  # the own-block scores: chunk key sums, then the dot products
        launches_per_step += 2

    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    cpu = parity = None
    if world == 1 and not args.no_cpu_baseline and args.variant == "forced":
        # the oracle on the host cores, on the GPU arm's bits: host K and V
        # (the pinned e2e copies) and only the sampled q rows
        leg = time_oracle(w, hk, hv, cu, q_rows_from(q), args.cpu_budget)
        cpu = {"value": leg["tflops"], "unit": "TFLOP/s", "cores": leg["threads"],
               "kind": "oracle",
               "sample": f"{len(leg['rows'])} seeded (token, head) rows of {w.name} "
                         f"({leg['seconds']:.1f} s), useful FLOPs of those rows"}
        # parity of this run's GPU forward on the same rows
        out_c, lse_c = moba.moba_forward(q, k, v, cu_d, w.block_size, w.topk,
                                         max_seqlen=w.max_seqlen, return_lse=True)
        idx_c = moba.moba_gate_topk(q, k, cu_d, w.block_size, w.topk, max_seqlen=w.max_seqlen)
        sel = torch.as_tensor(leg["rows"], device=dev)
        got_out = out_c.reshape(-1, w.head_dim)[sel].float().cpu().numpy()
        got_lse = lse_c.reshape(-1)[sel].cpu().numpy()
        got_idx = idx_c.reshape(-1, w.topk)[sel].cpu().numpy()
        del out_c, lse_c, idx_c
        parity = parity_stats(w, leg, hk, hv, cu, got_out, got_lse, got_idx)
    hashes = None if args.no_hash else input_hashes({"q": hq, "k": hk, "v": hv, "cu_seqlens": cu})
    side = None
    if world == 1 and not args.no_side and args.variant == "forced":
        # the 32K shapes beside the headline one, measured in the same run
        side = {n: side_workload(n, moba, dev, burst) for n in SIDE_WORKLOADS if n != w.name}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype_name,
        "data": "synthetic", "config": config,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "attn_history", "peak_source": f"{peak_src} bf16 {which}",
                     "frac_of_burst": achieved / burst, "frac_of_sustained": achieved / sustained},
        "cpu_baseline": cpu,
        "e2e": {"value": useful * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "copies on their own streams, overlapped with the previous and next "
                        "steps' compute (two device buffer sets)"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clock_info,
        "stage_ms": stage_ms,
        "stage_hbm": stage_hbm,
        "useful_flop_per_step": useful,
        "gate_flop_per_step": gate_flops(w),
        "dense_causal_ms": dense_ms,
        "speedup_vs_dense": dense_ms / ms,
        "frac_of_peak_end_to_end": value / world / peak,
        "attn_kernels_tflops": attn_tflops,
        "attn_kernels_frac_of_peak": attn_tflops / peak,
        "attn_kernels_frac_of_burst": attn_tflops / burst,
        "parity": parity,
        "input_sha256": hashes,
        "side_workloads": side,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
