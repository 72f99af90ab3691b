"""GPU backward (dq, dk, dv through the chosen blocks) against the oracle
backward, on the gate's own choice and on given indices.

Tolerance: the GPU takes P from the forward's lse and D = dO . O from the
forward's output (rounded to the input dtype), and accumulates in fp32; the
oracle is exact fp64. Errors are compared with the largest reference
magnitude of each gradient: bf16 inputs max 2e-2 and mean 2e-3 of it, fp32
inputs max 1e-4 of it."""
import numpy as np
import pytest
import torch

import long_context_prefill_block_b200 as moba
import oracle
from moba_inputs import small_case

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    # lengths, Hq, Hkv, d, B, topk, dtype
    ((1000, 333, 0, 700), 4, 2, 128, 128, 3, torch.bfloat16),
    ((1024,), 2, 1, 64, 128, 3, torch.float32),
    ((300, 95), 4, 4, 64, 20, 3, torch.float32),     # block size below the 64-key tile
    ((700, 1300), 8, 2, 128, 256, 4, torch.bfloat16),
    ((640,), 2, 2, 128, 128, 1, torch.bfloat16),     # k = 1: own block only
    ((512,), 2, 1, 128, 64, 8, torch.bfloat16),      # k >= blocks: dense causal
]


def _close(gpu, ref, dtype, what):
    gpu = gpu.float().cpu().numpy().astype(np.float64)
    scale = max(1.0, np.abs(ref).max())
    err = np.abs(gpu - ref)
    if dtype == torch.bfloat16:
        assert err.max() <= 2e-2 * scale, f"{what}: max err {err.max():.3e} (scale {scale:.3e})"
        assert err.mean() <= 2e-3 * scale, f"{what}: mean err {err.mean():.3e}"
    else:
        assert err.max() <= 1e-4 * scale, f"{what}: max err {err.max():.3e} (scale {scale:.3e})"


@pytest.mark.parametrize("case", CASES)
def test_backward_matches_oracle(case):
    lengths, Hq, Hkv, d, B, topk, dtype = case
    q, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=dtype, seed=411)
    dO = (torch.randn(q.shape, generator=torch.Generator().manual_seed(412)) * 0.5).to(dtype)
    qd, kd, vd, dOd = (x.to(DEV) for x in (q, k, v, dO))
    out, lse = moba.moba_forward(qd, kd, vd, cu, B, topk, return_lse=True)
    idx = moba.moba_gate_topk(qd, kd, cu, B, topk)
    dq, dk, dv = moba.moba_backward(qd, kd, vd, cu, out, lse, dOd, B, topk, idx=idx)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    rq, rk, rv = oracle.backward(q, k, v, dO, cu, B, topk, indices=idx.cpu())
    _close(dq, rq, dtype, "dq")
    _close(dk, rk, dtype, "dk")
    _close(dv, rv, dtype, "dv")


def test_backward_runs_the_gate_when_no_indices():
    q, k, v, cu = small_case((900, 500), 4, 2, 128, 128, 3, dtype=torch.bfloat16, seed=413)
    dO = torch.randn(q.shape, generator=torch.Generator().manual_seed(414)).to(q.dtype)
    qd, kd, vd, dOd = (x.to(DEV) for x in (q, k, v, dO))
    out, lse = moba.moba_forward(qd, kd, vd, cu, 128, 3, return_lse=True)
    idx = moba.moba_gate_topk(qd, kd, cu, 128, 3)
    a = moba.moba_backward(qd, kd, vd, cu, out, lse, dOd, 128, 3, idx=idx)
    b = moba.moba_backward(qd, kd, vd, cu, out, lse, dOd, 128, 3)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        # the same blocks; only the order of the fp32 atomic additions may differ
        assert torch.allclose(x, y, rtol=1e-5, atol=1e-6)
