"""Edge shapes of the forward against the oracle: block size 1 (every token its own block),
the largest top-k, block sizes that are multiples of the 128-key tile but not powers of two,
sequences of exactly whole blocks, one-token sequences and a single-block batch."""
import pytest
import torch

import long_context_prefill_block_b200 as moba
from moba_inputs import small_case
from parity import check_forward

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    # lengths, Hq, Hkv, d, B, topk, dtype
    ((200, 57), 2, 1, 64, 1, 3, torch.float32),          # B = 1: a block per token (SIMT)
    ((150,), 2, 2, 64, 1, 32, torch.bfloat16),           # B = 1, the largest k (SIMT, bf16)
    ((4608, 1152), 4, 2, 128, 384, 3, torch.bfloat16),   # B = 3 x 128 (tensor-core path)
    ((6144,), 2, 1, 128, 1024, 2, torch.bfloat16),       # B = 1024: 8 KV tiles per unit
    ((8192,), 2, 2, 128, 128, 32, torch.bfloat16),       # k = 32 over 64 blocks
    ((1024, 512, 2048), 2, 1, 128, 512, 3, torch.bfloat16),  # whole blocks only
    ((1, 1, 129), 2, 1, 128, 128, 3, torch.bfloat16),    # one-token sequences
    ((128,), 1, 1, 128, 128, 3, torch.bfloat16),         # a single block: own block only
]


@pytest.mark.parametrize("case", CASES)
def test_edge_forward(case):
    lengths, Hq, Hkv, d, B, topk, dtype = case
    q, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=dtype, seed=661)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out, lse = moba.moba_forward(qd, kd, vd, cu, B, topk, return_lse=True)
    idx = moba.moba_gate_topk(qd, kd, cu, B, topk)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    check_forward(q, k, v, cu, B, topk, out, lse, idx)
