"""GPU gate/top-k against the oracle across every top-k width of the gate
kernels (the tensor-core gates for bf16, d = 128 and at most 256 blocks per
sequence -- the sorting-network form for 5 to 15 history slots, the
insertion form otherwise -- and the SIMT gate for the rest), candidate
counts that span several column groups of the score tile, and exact ties
between blocks."""
import numpy as np
import pytest
import torch

import long_context_prefill_block_b200 as moba
import oracle
from moba_inputs import small_case
from parity import check_mismatch_band, index_mismatches, network_gate

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    # lengths, Hq, Hkv, d, B, topk
    ((5000,), 2, 1, 128, 128, 9),          # 40 blocks: two 32-column chunks, top-8 lists
    ((16384,), 1, 1, 128, 128, 17),        # 128 blocks (largest tensor-core gate), top-16
    ((16512,), 1, 1, 128, 128, 2),         # 129 blocks: SIMT gate, top-1
    ((4200, 900), 4, 2, 128, 128, 32),     # top-32 lists (k = 32, the largest), two sequences, GQA
    ((3000,), 2, 2, 128, 64, 2),           # block size 64, 47 blocks
    ((70, 0, 200), 2, 1, 128, 128, 3),     # sequences shorter than a block, an empty one
    # sorting-network gate (k - 1 = 5 .. 15 history slots, forced own block)
    ((32768,), 2, 1, 128, 128, 12),        # 256 blocks, the full score tile
    ((9000, 0, 1, 3000), 8, 2, 128, 128, 6),   # varlen, empty and one-token sequences, GQA
    ((20000, 700), 4, 4, 128, 256, 16),    # k = 16 (15 slots), B = 256
    ((2100,) * 40, 4, 4, 128, 128, 8),     # 160 groups: a CTA takes several, restaging kbar
]


@pytest.mark.parametrize("case", CASES)
def test_gate_widths(case):
    lengths, Hq, Hkv, d, B, topk = case
    q, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=torch.bfloat16, seed=211)
    idx = moba.moba_gate_topk(q.to(DEV), k.to(DEV), cu, B, topk).cpu().numpy()
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    ref, gap = oracle.gate_topk(q, k, cu, B, topk)
    bad = index_mismatches(idx, ref, gap)
    nb = -(-max(lengths) // B)
    check_mismatch_band(bad, gap, ref.shape[0] * ref.shape[1],
                        network_gate(torch.bfloat16, d, nb, topk))


@pytest.mark.parametrize("n_blocks", [12, 70, 130])
def test_gate_exact_ties_take_lower_block(n_blocks):
    # blocks 1, 2 and 3 hold identical keys, so their means -- and every
    # query's scores against them -- are bit-identical: the lower block wins
    B, topk = 128, 3
    q, k, v, cu = small_case((n_blocks * B,), 2, 1, 128, B, topk, dtype=torch.bfloat16, seed=212)
    # every query leans along dimension 0, and the tied blocks lie far along
    # it, so they are every later query's best history candidates
    q[..., 0] = q[..., 0].abs() + 2.0
    k[B:2 * B, :, 0] += 10.0
    k[2 * B:3 * B] = k[B:2 * B]
    k[3 * B:4 * B] = k[B:2 * B]
    idx = moba.moba_gate_topk(q.to(DEV), k.to(DEV), cu, B, topk).cpu().numpy()
    ref, _ = oracle.gate_topk(q, k, cu, B, topk)
    rows = np.arange(4 * B, n_blocks * B)  # queries that see all three tied blocks
    assert (idx[rows] == ref[rows]).all()
    # the tie is real and resolved to the lower indices 1 and 2
    assert (idx[rows, :, 0] == 1).all() and (idx[rows, :, 1] == 2).all()


@pytest.mark.parametrize("shared", [False, True])
def test_network_gate_million_token_geometry(shared):
    # the million-token shape's selection geometry (256 blocks of a 4096-token
    # block size is too big here; 256 blocks of 128 tokens instead), GQA 4:1,
    # k = 12, per-head and shared routing
    lengths, Hq, Hkv, B, topk = (32768, 5000), 8, 2, 128, 12
    q, k, v, cu = small_case(lengths, Hq, Hkv, 128, B, topk, dtype=torch.bfloat16, seed=215)
    idx = moba.moba_gate_topk(q.to(DEV), k.to(DEV), cu, B, topk, shared_routing=shared)
    idx = idx.cpu().numpy()
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    ref, gap = oracle.gate_topk(q, k, cu, B, topk, shared_routing=shared)
    bad = index_mismatches(idx, ref, gap)
    check_mismatch_band(bad, gap, ref.shape[0] * ref.shape[1], True)


def test_network_gate_exact_ties_take_lower_block():
    # as above, with k = 8: blocks 1 .. 7 hold identical keys, so seven tied
    # candidates compete for the seven history slots of every later query,
    # and blocks 8 .. 10 too (ten tied blocks in all): the lower ones win
    B, topk, n_blocks = 128, 8, 40
    q, k, v, cu = small_case((n_blocks * B,), 2, 1, 128, B, topk, dtype=torch.bfloat16, seed=216)
    q[..., 0] = q[..., 0].abs() + 2.0
    k[B:2 * B, :, 0] += 10.0
    for blk in range(2, 11):
        k[blk * B:(blk + 1) * B] = k[B:2 * B]
    idx = moba.moba_gate_topk(q.to(DEV), k.to(DEV), cu, B, topk).cpu().numpy()
    ref, _ = oracle.gate_topk(q, k, cu, B, topk)
    rows = np.arange(11 * B, n_blocks * B)  # queries that see all ten tied blocks
    assert (idx[rows] == ref[rows]).all()
    assert (idx[rows, :, :7] == np.arange(1, 8)).all()
