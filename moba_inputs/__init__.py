"""Seeded synthetic inputs for the MoBA prefill forward pass.

Shared by the tests, the bench and the smoke check: both the CUDA path and
the oracle consume the tensors made here, bit for bit. This module draws
random numbers only; it contains none of the method's arithmetic.

Layout: packed THD, like flash-attn varlen. q [T, Hq, d], k and v [T, Hkv, d],
cu_seqlens int32 [batch + 1] with sequence b at rows cu[b] .. cu[b+1]-1.

Distributions follow the workload table: q, k, v ~ N(0, s^2) and every key of
block i of sequence b and kv head g gets the same offset vector
delta[b, g, i] ~ N(0, sigma^2 I), so block means differ and routing is not
trivial. Draws are made in float32 with a seeded torch.Generator and then
cast to the input dtype.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    lengths: tuple          # per-sequence token counts
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    topk: int
    dtype: torch.dtype
    seed: int
    value_scale: float      # standard deviation of q, k, v
    offset_sigma: float     # standard deviation of the per-block key offset
    needles: int = 0        # planted needle blocks per head (long-context workload)
    needle_rows: int = 256  # query rows aligned with each needle

    @property
    def batch(self) -> int:
        return len(self.lengths)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.lengths))

    @property
    def max_seqlen(self) -> int:
        return int(max(self.lengths)) if self.lengths else 0


_S2 = 1.0 / math.sqrt(2.0)

WORKLOADS = {
    # N=1024, one head, d=64, B=128 (8 blocks), top-k 3, fp32.
    "tiny_fp32": Workload("tiny_fp32", (1024,), 1, 1, 64, 128, 3, torch.float32, 1001, 1.0, 0.5),
    # Scaling-law shape: batch 4 x N=8192, 16 heads MHA, d=128, B=512, k=3.
    "scaling_8k": Workload("scaling_8k", (8192,) * 4, 16, 16, 128, 512, 3, torch.bfloat16, 1002,
                           _S2, 0.3),
    # Long-context shape: N=32768, 32 heads MHA, B=512, k=3, 8 needle blocks per head.
    "long_32k": Workload("long_32k", (32768,), 32, 32, 128, 512, 3, torch.bfloat16, 1003, _S2, 0.3,
                         needles=8),
    # Kernel microbench shape: N=32768, 1 head, B=2048, k=3.
    "micro_32k": Workload("micro_32k", (32768,), 1, 1, 128, 2048, 3, torch.bfloat16, 1004, _S2, 0.3),
    # Llama-3.1-8B 1M prefill attention shape: 32 q heads / 8 kv heads, B=4096, k=12.
    "llama_1m": Workload("llama_1m", (1048576,), 32, 8, 128, 4096, 12, torch.bfloat16, 1005, _S2,
                         0.3),
}


def varlen_scaling_8k(seed: int = 1012) -> Workload:
    """Varlen variant of the scaling shape: 4 lengths ~ U[2048, 8192], rounded to 512."""
    g = torch.Generator().manual_seed(seed)
    raw = torch.randint(2048, 8193, (4,), generator=g).tolist()
    lengths = tuple(int(round(x / 512.0)) * 512 for x in raw)
    return dataclasses.replace(WORKLOADS["scaling_8k"], name="scaling_8k_varlen", lengths=lengths,
                               seed=seed)


def cu_seqlens_of(lengths: Sequence[int]) -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32)


def make_inputs(w: Workload, device: str | torch.device = "cpu"):
    """(q, k, v, cu_seqlens) for workload w, drawn on `device` (cu_seqlens on CPU).

    Draws depend only on (seed, device type): the same call on the same kind
    of device gives the same bits.
    """
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(w.seed)
    T, Hq, Hkv, d, B = w.total_tokens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size
    q = torch.randn((T, Hq, d), generator=g, device=dev, dtype=torch.float32).mul_(w.value_scale)
    k = torch.randn((T, Hkv, d), generator=g, device=dev, dtype=torch.float32).mul_(w.value_scale)
    v = torch.randn((T, Hkv, d), generator=g, device=dev, dtype=torch.float32).mul_(w.value_scale)
    start = 0
    for n in w.lengths:
        nb = (n + B - 1) // B
        off = torch.randn((nb, Hkv, d), generator=g, device=dev, dtype=torch.float32)
        off.mul_(w.offset_sigma)
        if w.needles:
            _plant_needles(w, g, q, off, start, n)
        blk = torch.arange(n, device=dev) // B
        k[start:start + n] += off[blk]
        start += n
    cast = lambda x: x.to(w.dtype).contiguous()
    return cast(q), cast(k), cast(v), cu_seqlens_of(w.lengths)


def _plant_needles(w: Workload, g: torch.Generator, q: torch.Tensor, off: torch.Tensor, start: int,
                   n: int) -> None:
    """Per head: `needles` distinct history blocks (index >= 1, not among the
    last two) get offset 0.3*sqrt(d)*u for a unit vector u; `needle_rows`
    query rows after that block are replaced by |q| (0.8 u + 0.6 w), w a unit
    vector orthogonal to u (cosine 0.8 with u). Needs Hq == Hkv."""
    dev = q.device
    d, B = w.head_dim, w.block_size
    nb = (n + B - 1) // B
    assert w.num_q_heads == w.num_kv_heads, "needles are planted per MHA head"
    for h in range(w.num_q_heads):
        blocks = torch.randperm(nb - 3, generator=g, device=dev)[: w.needles] + 1
        for blk in blocks.tolist():
            u = torch.randn(d, generator=g, device=dev)
            u /= u.norm()
            off[blk, h] = 0.3 * math.sqrt(d) * u
            lo = (blk + 1) * B
            rows = torch.randint(lo, n, (w.needle_rows,), generator=g, device=dev)
            r = torch.randn((w.needle_rows, d), generator=g, device=dev)
            r -= (r @ u)[:, None] * u[None, :]
            r /= r.norm(dim=1, keepdim=True)
            qr = q[start + rows, h]
            norm = qr.norm(dim=1, keepdim=True)
            q[start + rows, h] = norm * (0.8 * u[None, :] + 0.6 * r)


def small_case(lengths: Sequence[int], num_q_heads: int, num_kv_heads: int, head_dim: int,
               block_size: int, topk: int, dtype: torch.dtype = torch.bfloat16, seed: int = 0,
               value_scale: float = _S2, offset_sigma: float = 0.3, device="cpu"):
    """Inputs for an arbitrary small shape (parity sweeps and edge cases)."""
    w = Workload(f"case{seed}", tuple(int(x) for x in lengths), num_q_heads, num_kv_heads, head_dim,
                 block_size, topk, dtype, seed, value_scale, offset_sigma)
    return make_inputs(w, device)


def sample_rows(total_rows: int, n: int, seed: int) -> torch.Tensor:
    """n distinct seeded row ids in [0, total_rows) (row = token * Hq + head), sorted."""
    g = torch.Generator().manual_seed(seed)
    n = min(n, total_rows)
    if total_rows <= 4 * n:
        return torch.randperm(total_rows, generator=g)[:n].sort().values
    picks = torch.unique(torch.randint(0, total_rows, (2 * n,), generator=g, dtype=torch.int64))
    picks = picks[torch.randperm(len(picks), generator=g)[:n]]
    return picks.sort().values
