"""Query-head-parallel MoBA forward over several GPUs (the route the pages
give for 10M-token prefill: tensor parallelism extended to the query heads,
K/V sent to every GPU that holds heads reading them -- agihunt digest of
arXiv 2502.13189, efficiency paragraph).

Every rank starts with a contiguous token shard of the packed batch (all
heads), as a sequence-parallel producer of Q, K, V leaves it. One exchange
step turns token shards into head shards: rank j receives, for every token
of the batch, its q heads [j*Hq/G, (j+1)*Hq/G) and the kv heads those heads
read (a kv head read by several ranks is sent to each of them: the K/V
broadcast). Each rank then runs the whole single-GPU path on its heads --
the problem separates by kv-head group, so nothing else crosses GPUs -- and
a second exchange returns each rank's tokens with all heads. Both exchanges
are all-to-all calls on the process group (NCCL over NVLink / NVSwitch on
GPUs, gloo on CPU), into each rank's own memory.

Memory per rank: T * (Hq/G + 2 * kv heads of the rank) * d elements, instead
of the whole batch's Q.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

import torch
import torch.distributed as dist


def head_ranges(num_q_heads: int, num_kv_heads: int, world: int):
    """Per rank: (first q head, q heads, first kv head, kv heads)."""
    if num_q_heads % world:
        raise ValueError(f"{num_q_heads} q heads do not split over {world} ranks")
    if num_q_heads % num_kv_heads:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    grp = num_q_heads // num_kv_heads
    per = num_q_heads // world
    if per % grp and grp % per:
        raise ValueError(f"{per} q heads per rank must hold whole groups of {grp} or divide one")
    out = []
    for j in range(world):
        h0 = j * per
        g0 = h0 // grp
        g1 = (h0 + per - 1) // grp + 1
        out.append((h0, per, g0, g1 - g0))
    return out


def _all_to_all(chunks: List[torch.Tensor], recv_rows: Sequence[int], tail, group):
    """Send chunks[j] (rows x tail) to rank j; return the chunks received from every rank."""
    flat = [c.reshape(-1, *tail) for c in chunks]
    send = torch.cat(flat, dim=0).contiguous()
    recv = send.new_empty((sum(recv_rows), *tail))
    dist.all_to_all_single(recv, send, list(recv_rows), [c.shape[0] for c in flat], group=group)
    return list(torch.split(recv, list(recv_rows), dim=0))


def moba_forward_head_parallel(q_shard: torch.Tensor, k_shard: torch.Tensor,
                               v_shard: torch.Tensor, cu_seqlens: torch.Tensor, block_size: int,
                               topk: int, shard_tokens: Sequence[int],
                               max_seqlen: Optional[int] = None, return_lse: bool = False,
                               group=None, forward_fn: Optional[Callable] = None):
    """MoBA forward of a token-sharded batch, computed head-parallel.

    q_shard [T_r, Hq, d], k_shard / v_shard [T_r, Hkv, d]: this rank's tokens (the ranks'
    shards in rank order make up the packed batch); shard_tokens: T_r of every rank;
    cu_seqlens: the whole batch's sequence offsets (the same on every rank). Returns this
    rank's tokens of the output [T_r, Hq, d] (and lse [T_r, Hq]).

    forward_fn(q, k, v, cu_seqlens, block_size, topk, max_seqlen) -> (out, lse) runs the
    single-GPU path on the rank's heads; the default is the CUDA library."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    T_r, Hq, d = q_shard.shape
    Hkv = k_shard.shape[1]
    if len(shard_tokens) != world or shard_tokens[rank] != T_r:
        raise ValueError("shard_tokens must list every rank's token count")
    if forward_fn is None:
        from . import moba_forward

        def forward_fn(q, k, v, cu, B, kk, ms):
            return moba_forward(q, k, v, cu, B, kk, max_seqlen=ms, return_lse=True)

    ranges = head_ranges(Hq, Hkv, world)
    h0, nh, g0, ng = ranges[rank]
    # tokens of every rank, heads of rank j
    q_parts = _all_to_all([q_shard[:, a:a + n] for a, n, _, _ in ranges],
                          [t * nh for t in shard_tokens], (d,), group)
    k_parts = _all_to_all([k_shard[:, a:a + n] for _, _, a, n in ranges],
                          [t * ng for t in shard_tokens], (d,), group)
    v_parts = _all_to_all([v_shard[:, a:a + n] for _, _, a, n in ranges],
                          [t * ng for t in shard_tokens], (d,), group)
    q = torch.cat([p.reshape(t, nh, d) for p, t in zip(q_parts, shard_tokens)], dim=0)
    k = torch.cat([p.reshape(t, ng, d) for p, t in zip(k_parts, shard_tokens)], dim=0)
    v = torch.cat([p.reshape(t, ng, d) for p, t in zip(v_parts, shard_tokens)], dim=0)
    out, lse = forward_fn(q.contiguous(), k.contiguous(), v.contiguous(), cu_seqlens, block_size,
                          topk, max_seqlen)
    # back: rank i's tokens, this rank's heads
    offs = [0]
    for t in shard_tokens:
        offs.append(offs[-1] + t)
    o_parts = _all_to_all([out[offs[i]:offs[i + 1]] for i in range(world)],
                          [T_r * n for _, n, _, _ in ranges], (d,), group)
    out_r = torch.cat([p.reshape(T_r, n, d) for p, (_, n, _, _) in zip(o_parts, ranges)], dim=1)
    if not return_lse:
        return out_r
    lse = lse.to(torch.float32)
    l_parts = _all_to_all([lse[offs[i]:offs[i + 1]].reshape(-1, 1) for i in range(world)],
                          [T_r * n for _, n, _, _ in ranges], (1,), group)
    lse_r = torch.cat([p.reshape(T_r, n) for p, (_, n, _, _) in zip(l_parts, ranges)], dim=1)
    return out_r, lse_r
