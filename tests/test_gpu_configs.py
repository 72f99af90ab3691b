"""GPU parity at the workloads' full sizes, in the launch configuration the
bench times (moba_forward through the C ABI): block indices, outputs and lse
compared with the oracle on every row of the 8K, 8K-varlen, 32K and
kernel-microbench workloads, and on 4,096 seeded sampled rows of the
million-token shape (the oracle gets only those q rows)."""
import numpy as np
import pytest
import torch

import long_context_prefill_block_b200 as moba
import oracle
from moba_inputs import WORKLOADS, make_inputs, sample_rows, varlen_scaling_8k
from parity import assert_close, check_forward, index_mismatches

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run(w):
    q, k, v, cu = make_inputs(w, "cpu")
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out, lse = moba.moba_forward(qd, kd, vd, cu, w.block_size, w.topk, max_seqlen=w.max_seqlen,
                                 return_lse=True)
    idx = moba.moba_gate_topk(qd, kd, cu, w.block_size, w.topk, max_seqlen=w.max_seqlen)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    return q, k, v, cu, out, lse, idx


def test_tiny_fp32_full():
    w = WORKLOADS["tiny_fp32"]
    q, k, v, cu, out, lse, idx = run(w)
    check_forward(q, k, v, cu, w.block_size, w.topk, out, lse, idx)


@pytest.mark.parametrize("name", ["scaling_8k", "scaling_8k_varlen", "long_32k", "micro_32k"])
def test_workload_every_row(name):
    # the oracle computes every (token, head) row: indices, outputs and lse of
    # the whole forward (tens of seconds of fp64 work on the host cores)
    w = varlen_scaling_8k() if name == "scaling_8k_varlen" else WORKLOADS[name]
    q, k, v, cu, out, lse, idx = run(w)
    ref_idx, gap = oracle.gate_topk(q, k, cu, w.block_size, w.topk)
    bad = index_mismatches(idx.cpu().numpy(), ref_idx, gap)
    # near-tie rows stay rare
    assert len(bad) <= 1e-4 * ref_idx.shape[0] * ref_idx.shape[1] + 4
    check_forward(q, k, v, cu, w.block_size, w.topk, out, lse, idx)


def test_llama_1m_sampled():
    w = WORKLOADS["llama_1m"]
    q, k, v, cu = make_inputs(w, DEV)
    out = torch.empty_like(q)
    out, lse = moba.moba_forward(q, k, v, cu, w.block_size, w.topk, max_seqlen=w.max_seqlen,
                                 return_lse=True, out=out)
    idx = moba.moba_gate_topk(q, k, cu, w.block_size, w.topk, max_seqlen=w.max_seqlen)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    rows = sample_rows(w.total_tokens * w.num_q_heads, 4096, seed=11)
    Hq, d = w.num_q_heads, w.head_dim
    rd = rows.to(DEV)
    q_rows = q.reshape(-1, d)[rd].cpu()
    got = out.reshape(-1, d)[rd].float().cpu().numpy()
    got_lse = lse.reshape(-1)[rd].cpu().numpy()
    got_idx = idx.reshape(-1, w.topk)[rd].cpu().numpy()
    del q, out, lse, idx
    kc, vc = k.cpu(), v.cpu()
    del k, v
    torch.cuda.empty_cache()
    ref, ref_lse, ref_idx, gap = oracle.forward_rows(None, kc, vc, cu, w.block_size, w.topk,
                                                     rows.numpy(), q_rows=q_rows, num_q_heads=Hq)
    bad = index_mismatches(got_idx, ref_idx, gap)
    if len(bad):
        o2, l2, _, _ = oracle.forward_rows(None, kc, vc, cu, w.block_size, w.topk,
                                           rows.numpy()[bad], indices=got_idx[bad],
                                           q_rows=q_rows[torch.as_tensor(bad)], num_q_heads=Hq)
        ref[bad] = o2
        ref_lse[bad] = l2
    assert_close(got, ref, torch.bfloat16)
    assert np.abs(got_lse - ref_lse).max() <= 1e-3
