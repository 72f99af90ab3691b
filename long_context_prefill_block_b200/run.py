"""Runs calls of the MoBA path on a seeded synthetic workload (a profiling aid).

    python -m long_context_prefill_block_b200.run --workload long_32k --iters 3
    python -m long_context_prefill_block_b200.run --workload llama_1m --tokens 131072 \\
        --block-size 512 --call gate

Draws the workload's inputs on cuda:0, then makes --iters calls of one entry
point through the public binding (forward, gate, backward or decode) and
prints the mean time per call (CUDA events) and the device status word. The
shape options override the named workload, so that a profiler can capture a
kernel on a case a few GB in size that keeps the per-row work of the full
workload (e.g. the million-token gate's 256 blocks at 131,072 tokens with
B = 512). Inputs are drawn before the first call: a profiler that skips the
first launches of our kernels sees only the calls.
"""
from __future__ import annotations

import argparse
import dataclasses
import os
import sys

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import long_context_prefill_block_b200 as moba  # noqa: E402
from moba_inputs import WORKLOADS, make_inputs  # noqa: E402


def workload(name: str, tokens: int | None, block_size: int | None, topk: int | None):
    w = WORKLOADS[name]
    kw = {}
    if tokens is not None:
        kw["lengths"] = (int(tokens),)
    if block_size is not None:
        kw["block_size"] = int(block_size)
    if topk is not None:
        kw["topk"] = int(topk)
    return dataclasses.replace(w, **kw) if kw else w


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="long_32k", choices=sorted(WORKLOADS))
    ap.add_argument("--tokens", type=int, default=None, help="one sequence of this length")
    ap.add_argument("--block-size", type=int, default=None)
    ap.add_argument("--topk", type=int, default=None)
    ap.add_argument("--call", default="forward", choices=["forward", "gate", "backward", "decode"])
    ap.add_argument("--iters", type=int, default=2)
    args = ap.parse_args()
    w = workload(args.workload, args.tokens, args.block_size, args.topk)
    dev = torch.device("cuda", 0)
    q, k, v, cu = make_inputs(w, dev)
    cu_d = cu.to(dev)
    B, K, S = w.block_size, w.topk, w.max_seqlen
    if args.call == "forward":
        call = lambda: moba.moba_forward(q, k, v, cu_d, B, K, max_seqlen=S)
    elif args.call == "gate":
        call = lambda: moba.moba_gate_topk(q, k, cu_d, B, K, max_seqlen=S)
    elif args.call == "backward":
        out, lse = moba.moba_forward(q, k, v, cu_d, B, K, max_seqlen=S, return_lse=True)
        idx = moba.moba_gate_topk(q, k, cu_d, B, K, max_seqlen=S)
        dout = torch.randn(out.shape, generator=torch.Generator(device=dev).manual_seed(5),
                           device=dev, dtype=torch.float32).to(out.dtype)
        call = lambda: moba.moba_backward(q, k, v, cu_d, out, lse, dout, B, K, idx=idx,
                                          max_seqlen=S)
    else:
        # one query per request: the last position of each sequence
        last = (cu_d[1:] - 1).long()
        qd = q[last].contiguous()
        cu_q = torch.arange(w.batch + 1, dtype=torch.int32, device=dev)
        kbar = moba.moba_meanpool(k, cu_d, B, max_seqlen=S)
        call = lambda: moba.moba_decode(qd, k, v, cu_d, cu_q, kbar, B, K, max_seqlen=S)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.iters):
        call()
    e1.record()
    torch.cuda.synchronize(dev)
    status = moba.moba_device_status(dev)
    print(f"{args.call} {w.name} tokens={w.total_tokens} B={B} k={K}: "
          f"{e0.elapsed_time(e1) / max(args.iters, 1):.3f} ms per call, status {status}")
    if status != 0:
        raise SystemExit(1)


if __name__ == "__main__":
    main()
