"""GPU gate/top-k against the oracle across every top-k width of both gate
kernels (the tensor-core gate for bf16, d = 128 and at most 128 blocks per
sequence; the SIMT gate otherwise), candidate counts that span several
32-column chunks of the score tile, and exact ties between blocks."""
import numpy as np
import pytest
import torch

import long_context_prefill_block_b200 as moba
import oracle
from moba_inputs import small_case
from parity import index_mismatches

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
    assert len(bad) <= 1e-4 * ref.shape[0] * ref.shape[1] + 2


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
