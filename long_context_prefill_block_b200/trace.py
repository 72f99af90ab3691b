"""Phase traces of one CTA of a tensor-core kernel (a measuring aid).

    python -m long_context_prefill_block_b200.build --trace
    python -m long_context_prefill_block_b200.trace --workload llama_1m --kernel gate [--cta 0]

Runs the chosen workload once through the trace build (libmoba_trace.so,
the library compiled with MOBA_TRACE; include/moba_trace.h), with lane 0 of
every warp of one CTA recording the SM clock at the kernel's phase
boundaries, and prints, per warp role, the time between consecutive events
(count, median and mean, in SM cycles and in microseconds at --mhz). The
ordinary library carries none of this code.
"""
from __future__ import annotations

import argparse
import ctypes
import os
import sys
from collections import defaultdict

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import long_context_prefill_block_b200 as moba  # noqa: E402
from long_context_prefill_block_b200 import build  # noqa: E402
from moba_inputs import WORKLOADS, make_inputs  # noqa: E402

KERNELS = {"gate": 1, "hist": 2, "cur": 3, "dense": 4}
MAX_WARPS = 16

# event ids of each kernel, as the kernel sources list them
EVENTS = {
    "gate": {1: "item", 2: "q buffer free", 3: "q tile stored", 4: "scores free",
             5: "q tile ready", 6: "mma issued", 10: "scores ready", 11: "scores in regs",
             12: "list sorted", 13: "lists merged", 14: "row written"},
}
EVENTS["hist"] = EVENTS["cur"] = EVENTS["dense"] = {
    20: "K issued", 21: "V issued", 30: "unit", 31: "QK issued", 32: "P lo ready",
    33: "PV issued", 40: "Q half loaded", 50: "S ready", 51: "row max", 52: "P lo written",
    53: "P written", 54: "O ready", 55: "row written", 56: "S in regs", 57: "P lo computed",
    58: "P hi computed"}


def run(workload: str, kernel: str, cta: int, cap: int, mhz: float, shared: bool):
    L = moba.use_library(build.LIB_TRACE)
    L.moba_trace_arm.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                 ctypes.c_int]
    L.moba_trace_arm.restype = ctypes.c_int
    L.moba_trace_disarm.restype = ctypes.c_int
    w = WORKLOADS[workload]
    dev = torch.device("cuda", 0)
    q, k, v, cu = make_inputs(w, dev)
    call = (lambda: moba.moba_gate_topk(q, k, cu, w.block_size, w.topk, max_seqlen=w.max_seqlen,
                                        shared_routing=shared)) if kernel == "gate" else \
        (lambda: moba.moba_forward(q, k, v, cu, w.block_size, w.topk, max_seqlen=w.max_seqlen,
                                   shared_routing=shared))
    if kernel == "dense":
        call = lambda: moba.dense_causal_forward(q, k, v, cu, max_seqlen=w.max_seqlen)
    call()  # warm-up, untraced
    torch.cuda.synchronize(dev)
    buf = torch.zeros((MAX_WARPS, cap, 2), dtype=torch.int64, device=dev)
    counts = torch.zeros(MAX_WARPS, dtype=torch.int32, device=dev)
    rc = L.moba_trace_arm(KERNELS[kernel], cta, buf.data_ptr(), counts.data_ptr(), cap)
    if rc:
        raise RuntimeError(f"moba_trace_arm failed: {rc}")
    call()
    torch.cuda.synchronize(dev)
    L.moba_trace_disarm()
    if moba.moba_device_status(dev) != 0:
        raise RuntimeError("device status error")
    return buf.cpu().numpy(), counts.cpu().numpy()


def summarise(buf, counts, kernel: str, mhz: float):
    names = EVENTS[kernel]
    lines = []
    t0 = min(int(buf[wi, 0, 0]) for wi in range(MAX_WARPS) if counts[wi] > 0)
    t1 = max(int(buf[wi, min(counts[wi], buf.shape[1]) - 1, 0]) for wi in range(MAX_WARPS)
             if counts[wi] > 0)
    lines.append(f"CTA span {t1 - t0} cycles = {(t1 - t0) / mhz:.1f} us at {mhz:.0f} MHz")
    for wi in range(MAX_WARPS):
        n = int(min(counts[wi], buf.shape[1]))
        if n == 0:
            continue
        clk = buf[wi, :n, 0].astype(np.int64)
        ids = (buf[wi, :n, 1] & 0xFFFFFFFF).astype(np.int64)
        pairs = defaultdict(list)
        for i in range(1, n):
            pairs[(int(ids[i - 1]), int(ids[i]))].append(int(clk[i] - clk[i - 1]))
        lines.append(f"warp {wi}: {n} events"
                     + (f" ({counts[wi] - n} dropped)" if counts[wi] > n else ""))
        for (a, b), d in sorted(pairs.items(), key=lambda kv: -sum(kv[1])):
            d = np.asarray(d)
            lines.append(f"  {names.get(a, a):>16} -> {names.get(b, b):<16} n={len(d):6d} "
                         f"median {np.median(d):8.0f} cyc ({np.median(d) / mhz:6.2f} us)  "
                         f"mean {d.mean():8.0f}  total {d.sum() / mhz / 1e3:7.3f} ms")
    return "\n".join(lines)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="llama_1m", choices=sorted(WORKLOADS))
    ap.add_argument("--kernel", default="gate", choices=sorted(KERNELS))
    ap.add_argument("--cta", type=int, default=0)
    ap.add_argument("--cap", type=int, default=1 << 16, help="records per warp")
    ap.add_argument("--mhz", type=float, default=1900.0, help="SM clock for the us figures")
    ap.add_argument("--shared", action="store_true", help="shared routing")
    args = ap.parse_args()
    buf, counts = run(args.workload, args.kernel, args.cta, args.cap, args.mhz, args.shared)
    print(summarise(buf, counts, args.kernel, args.mhz))


if __name__ == "__main__":
    main()
