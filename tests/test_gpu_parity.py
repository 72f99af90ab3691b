"""GPU parity of every kernel of the path against the fp64 oracle, through
the C ABI (Python binding), on seeded synthetic inputs. Small shapes span
several tiles, ragged tails, empty sequences, GQA ratios and the degenerate
budgets (k = 1, k >= number of blocks)."""
import numpy as np
import pytest
import torch

import long_context_prefill_block_b200 as moba
import oracle
from moba_inputs import cu_seqlens_of, small_case
from parity import TIE_GAP, assert_close, check_forward, index_mismatches

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    # lengths, Hq, Hkv, d, B, topk, dtype
    ((1000, 333, 0, 2048), 4, 2, 128, 128, 3, torch.bfloat16),
    ((1024,), 1, 1, 64, 128, 3, torch.float32),
    ((700, 1300), 8, 2, 128, 256, 4, torch.bfloat16),
    ((517, 64, 1), 2, 1, 64, 128, 2, torch.bfloat16),
    ((300, 95), 4, 4, 64, 20, 3, torch.float32),
    ((640,), 8, 1, 128, 128, 5, torch.bfloat16),
]


def to_dev(*ts):
    return [t.to(DEV) for t in ts]


@pytest.mark.parametrize("case", CASES)
def test_meanpool(case):
    lengths, Hq, Hkv, d, B, topk, dtype = case
    q, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=dtype, seed=101)
    kbar = moba.moba_meanpool(k.to(DEV), cu, B).cpu().numpy()
    ref = oracle.meanpool(k, cu, B)
    assert kbar.shape == ref.shape
    assert (np.abs(kbar - ref) <= 1e-5 * np.maximum(1.0, np.abs(ref))).all()


@pytest.mark.parametrize("case", CASES)
def test_gate_topk(case):
    lengths, Hq, Hkv, d, B, topk, dtype = case
    q, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=dtype, seed=102)
    idx = moba.moba_gate_topk(q.to(DEV), k.to(DEV), cu, B, topk).cpu().numpy()
    ref, gap = oracle.gate_topk(q, k, cu, B, topk)
    index_mismatches(idx, ref, gap)


@pytest.mark.parametrize("case", CASES)
def test_forward(case):
    lengths, Hq, Hkv, d, B, topk, dtype = case
    q, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=dtype, seed=103)
    qd, kd, vd = to_dev(q, k, v)
    out, lse = moba.moba_forward(qd, kd, vd, cu, B, topk, return_lse=True)
    idx = moba.moba_gate_topk(qd, kd, cu, B, topk)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    check_forward(q, k, v, cu, B, topk, out, lse, idx)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_topk_one_and_full_budget(dtype):
    lengths, B = (900, 257), 128
    q, k, v, cu = small_case(lengths, 2, 1, 128, B, 1, dtype=dtype, seed=104)
    qd, kd, vd = to_dev(q, k, v)
    out1 = moba.moba_forward(qd, kd, vd, cu, B, 1)
    check_forward(q, k, v, cu, B, 1, out1)
    full = max(lengths) // B + 1
    outf = moba.moba_forward(qd, kd, vd, cu, B, full)
    dense, _ = oracle.dense_causal(q, k, v, cu)
    assert_close(outf.float().cpu().numpy(), dense, dtype, "full budget vs dense")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_dense_causal(dtype):
    lengths = (700, 0, 301)
    q, k, v, cu = small_case(lengths, 4, 2, 128, 128, 1, dtype=dtype, seed=105)
    out, lse = moba.dense_causal_forward(*to_dev(q, k, v), cu, return_lse=True)
    ref, ref_lse = oracle.dense_causal(q, k, v, cu)
    assert_close(out.float().cpu().numpy(), ref, dtype)
    assert np.abs(lse.cpu().numpy() - ref_lse).max() < 1e-3


def test_window_and_sink_indices():
    lengths, B, topk = (1024, 384), 128, 3
    q, k, v, cu = small_case(lengths, 2, 2, 128, B, topk, dtype=torch.bfloat16, seed=106)
    idx = np.full((sum(lengths), 2, topk), -1, np.int32)
    pos = np.concatenate([np.arange(n) for n in lengths])
    for t, p in enumerate(pos):
        c = p // B
        row = sorted({0, c - 1, c}) if c >= 1 else [c]
        idx[t, :, :len(row)] = row
    idx_t = torch.from_numpy(idx)
    out = moba.moba_forward_with_indices(*to_dev(q, k, v), cu, idx_t.to(DEV), B)
    assert moba.moba_device_status() == 0
    check_forward(q, k, v, cu, B, topk, out, indices=idx_t)


def test_non_canonical_indices_are_reported():
    lengths, B, topk = (512,), 128, 3
    q, k, v, cu = small_case(lengths, 1, 1, 128, B, topk, dtype=torch.bfloat16, seed=107)
    idx = torch.full((512, 1, topk), -1, dtype=torch.int32)
    idx[:, 0, 0] = torch.arange(512) // B        # canonical: own block only
    idx[300, 0, :] = torch.tensor([2, 1, 2])     # descending history: not canonical
    moba.moba_device_status()                    # clear
    moba.moba_forward_with_indices(*to_dev(q, k, v), cu, idx.to(DEV), B)
    assert moba.moba_device_status() == moba.MOBA_ERR_BAD_INDICES
    assert moba.moba_device_status() == 0


def test_gqa_ratios():
    for Hq, Hkv in ((8, 8), (8, 4), (8, 2), (8, 1)):
        q, k, v, cu = small_case((600, 200), Hq, Hkv, 128, 128, 3, dtype=torch.bfloat16,
                                 seed=108 + Hq * 10 + Hkv)
        qd, kd, vd = to_dev(q, k, v)
        out = moba.moba_forward(qd, kd, vd, cu, 128, 3)
        idx = moba.moba_gate_topk(qd, kd, cu, 128, 3)
        check_forward(q, k, v, cu, 128, 3, out, idx_gpu=idx)


def test_repeat_calls_are_deterministic():
    q, k, v, cu = small_case((1500,), 4, 2, 128, 128, 3, dtype=torch.bfloat16, seed=109)
    qd, kd, vd = to_dev(q, k, v)
    a = moba.moba_forward(qd, kd, vd, cu, 128, 3)
    b = moba.moba_forward(qd, kd, vd, cu, 128, 3)
    assert torch.equal(a, b)
