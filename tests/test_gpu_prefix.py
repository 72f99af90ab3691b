"""GPU prefix-mean own-block gate (the own block scored by the mean of its
keys up to the query, competing for the k slots; PaperTrace "2.1.3 MoBA",
section 5.2) against the oracle's prefix-mean mode: gate indices, the full
forward on both attention paths (tensor-core and SIMT), the backward, and a
sampled check at the 8K scaling workload's size."""
import numpy as np
import pytest
import torch

import long_context_prefill_block_b200 as moba
import oracle
from moba_inputs import WORKLOADS, make_inputs, small_case
from parity import check_forward, check_rows, index_mismatches

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    # lengths, Hq, Hkv, d, B, topk, dtype, shared
    ((2048, 700), 4, 2, 128, 128, 3, torch.bfloat16, False),   # tensor-core attention, GQA
    ((5000,), 2, 1, 128, 128, 9, torch.bfloat16, False),       # 40 blocks, top-9
    ((1100, 300, 0), 4, 2, 64, 64, 4, torch.bfloat16, False),  # d = 64, an empty sequence
    ((1024, 77), 2, 2, 64, 40, 3, torch.float32, False),       # fp32 SIMT path, ragged blocks
    ((2048,), 8, 2, 128, 128, 4, torch.bfloat16, True),        # with shared routing
    ((640,), 2, 1, 128, 128, 1, torch.bfloat16, False),        # k = 1: one block per query
    ((512,), 2, 1, 128, 64, 8, torch.bfloat16, False),         # k >= blocks: dense causal
]


def _own_lost_share(idx, cu, B):
    T = idx.shape[0]
    c = np.zeros(T, dtype=np.int64)
    cu = np.asarray(cu)
    for b in range(len(cu) - 1):
        c[cu[b]:cu[b + 1]] = np.arange(cu[b + 1] - cu[b]) // B
    return float((~(idx == c[:, None, None]).any(axis=2)).mean())


@pytest.mark.parametrize("case", CASES)
def test_prefix_gate(case):
    lengths, Hq, Hkv, d, B, topk, dtype, shared = case
    q, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=dtype, seed=621)
    idx = moba.moba_gate_topk(q.to(DEV), k.to(DEV), cu, B, topk, shared_routing=shared,
                              prefix_mean=True)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    idx = idx.cpu().numpy()
    ref, gap = oracle.gate_topk(q, k, cu, B, topk, shared_routing=shared, prefix_mean=True)
    bad = index_mismatches(idx, ref, gap)
    assert len(bad) <= 1e-4 * ref.shape[0] * ref.shape[1] + 2
    if topk > 1 and topk < 8:
        # the variant is exercised: some own blocks lose, most win
        assert 0.0 < _own_lost_share(ref, cu, B) < 0.9


@pytest.mark.parametrize("case", CASES)
def test_prefix_forward(case):
    lengths, Hq, Hkv, d, B, topk, dtype, shared = case
    q, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=dtype, seed=622)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out, lse = moba.moba_forward(qd, kd, vd, cu, B, topk, return_lse=True, shared_routing=shared,
                                 prefix_mean=True)
    idx = moba.moba_gate_topk(qd, kd, cu, B, topk, shared_routing=shared, prefix_mean=True)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    check_forward(q, k, v, cu, B, topk, out, lse, idx, shared_routing=shared, prefix_mean=True)


def test_prefix_forward_with_given_indices():
    # rows that leave out their own block, fed directly: the own-block kernel
    # skips them and the merge gives their history alone
    q, k, v, cu = small_case((1500,), 2, 1, 128, 128, 3, dtype=torch.bfloat16, seed=623)
    idx, _ = oracle.gate_topk(q, k, cu, 128, 3, prefix_mean=True)
    idx_t = torch.from_numpy(idx)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out, lse = moba.moba_forward_with_indices(qd, kd, vd, cu, idx_t.to(DEV), 128, return_lse=True,
                                              prefix_mean=True)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    check_forward(q, k, v, cu, 128, 3, out, lse, indices=idx_t, prefix_mean=True)
    # the same rows under the forced-block contract are not canonical
    moba.moba_forward_with_indices(qd, kd, vd, cu, idx_t.to(DEV), 128)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == moba.MOBA_ERR_BAD_INDICES


@pytest.mark.parametrize("case", [CASES[0], CASES[3]])
def test_prefix_backward(case):
    lengths, Hq, Hkv, d, B, topk, dtype, shared = case
    q, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=dtype, seed=624)
    dO = (torch.randn(q.shape, generator=torch.Generator().manual_seed(625)) * 0.5).to(dtype)
    qd, kd, vd, dOd = (x.to(DEV) for x in (q, k, v, dO))
    out, lse = moba.moba_forward(qd, kd, vd, cu, B, topk, return_lse=True, prefix_mean=True)
    idx = moba.moba_gate_topk(qd, kd, cu, B, topk, prefix_mean=True)
    dq, dk, dv = moba.moba_backward(qd, kd, vd, cu, out, lse, dOd, B, topk, idx=idx,
                                    prefix_mean=True)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    rq, rk, rv = oracle.backward(q, k, v, dO, cu, B, topk, indices=idx.cpu(), prefix_mean=True)
    for gpu, ref, what in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        g = gpu.float().cpu().numpy().astype(np.float64)
        scale = max(1.0, np.abs(ref).max())
        err = np.abs(g - ref)
        if dtype == torch.bfloat16:
            assert err.max() <= 2e-2 * scale and err.mean() <= 2e-3 * scale, what
        else:
            assert err.max() <= 1e-4 * scale, what


def test_prefix_forward_sampled_at_scaling_size():
    w = WORKLOADS["scaling_8k"]
    q, k, v, cu = make_inputs(w, DEV)
    out, lse = moba.moba_forward(q, k, v, cu, w.block_size, w.topk, max_seqlen=w.max_seqlen,
                                 return_lse=True, prefix_mean=True)
    idx = moba.moba_gate_topk(q, k, cu, w.block_size, w.topk, max_seqlen=w.max_seqlen,
                              prefix_mean=True)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    T, Hq = q.shape[:2]
    rows = np.random.default_rng(626).choice(T * Hq, size=192, replace=False)
    check_rows(q, k, v, cu, w.block_size, w.topk, rows, out, idx, lse, prefix_mean=True)
