"""GPU shared routing (the q heads of a kv head's group share the blocks of
their mean score) against the oracle's shared-routing mode: gate indices on
both gate kernels, and the full forward."""
import pytest
import torch

import long_context_prefill_block_b200 as moba
import oracle
from moba_inputs import small_case
from parity import check_forward, check_mismatch_band, index_mismatches, network_gate

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    # lengths, Hq, Hkv, d, B, topk, dtype
    ((2048, 700), 8, 2, 128, 128, 3, torch.bfloat16),   # tensor-core gate, GQA 4:1
    ((5000,), 8, 1, 128, 128, 9, torch.bfloat16),       # tensor-core gate, 8:1, 40 blocks
    ((1100, 300), 4, 2, 64, 64, 4, torch.bfloat16),     # SIMT gate (d = 64)
    ((1024,), 6, 2, 64, 128, 3, torch.float32),         # SIMT gate, fp32, 3 heads per group
]


@pytest.mark.parametrize("case", CASES)
def test_shared_gate(case):
    lengths, Hq, Hkv, d, B, topk, dtype = case
    q, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=dtype, seed=311)
    idx = moba.moba_gate_topk(q.to(DEV), k.to(DEV), cu, B, topk, shared_routing=True)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    idx = idx.cpu().numpy()
    grp = Hq // Hkv
    for h in range(Hq):
        assert (idx[:, h] == idx[:, (h // grp) * grp]).all()
    ref, gap = oracle.gate_topk(q, k, cu, B, topk, shared_routing=True)
    bad = index_mismatches(idx, ref, gap)
    check_mismatch_band(bad, gap, ref.shape[0] * ref.shape[1],
                        network_gate(dtype, d, -(-max(lengths) // B), topk))


@pytest.mark.parametrize("case", CASES)
def test_shared_forward(case):
    lengths, Hq, Hkv, d, B, topk, dtype = case
    if dtype == torch.bfloat16 and d == 128 and B % 128:
        pytest.skip("covered by the other cases")
    q, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=dtype, seed=312)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out, lse = moba.moba_forward(qd, kd, vd, cu, B, topk, return_lse=True, shared_routing=True)
    idx = moba.moba_gate_topk(qd, kd, cu, B, topk, shared_routing=True)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    check_forward(q, k, v, cu, B, topk, out, lse, idx, shared_routing=True)
