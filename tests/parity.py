"""Comparison helpers for GPU-vs-oracle parity tests.

Tolerances (written here, used by every GPU test):
  bf16 inputs (fp32 accumulation): max |gpu - oracle| <= 2e-2 and mean <= 2e-3;
  fp32 inputs:                     max |gpu - oracle| <= 1e-4.
  block indices: bit-exact, except rows whose oracle score gap between the
  last chosen and the first rejected history block is below 1e-4 relative;
  such rows are re-checked against the oracle run with the GPU's indices.
  The sorting-network gate ranks by 32-bit keys that keep a score's top 24
  order bits, so its mismatches must lie inside a tighter band, a relative
  gap below 4e-5 (2^-15 plus fp32 rounding of the scores); the other gates
  compare exact fp32 scores, so their (near-tie) mismatches must stay rare.
  block means: |gpu - oracle| <= 1e-5 * max(1, |oracle|).
"""
import numpy as np
import torch

import oracle

TOL = {torch.bfloat16: dict(max_abs=2e-2, mean_abs=2e-3), torch.float32: dict(max_abs=1e-4,
                                                                              mean_abs=1e-4)}
TIE_GAP = 1e-4
KEY_GAP = 4e-5


def network_gate(dtype, head_dim, n_blocks, topk, prefix_mean=False):
    """Whether the sorting-network tensor-core gate serves this shape (bf16,
    d = 128, at most 256 blocks per sequence, 5 to 15 history slots beside
    the forced own block)."""
    return (dtype == torch.bfloat16 and head_dim == 128 and n_blocks <= 256 and not prefix_mean
            and 5 <= topk - 1 <= 15)


def check_mismatch_band(bad, gap, n_rows, network):
    """Mismatching rows (from index_mismatches): inside the 2^-15 key band
    for the network gate, else rare (at most 1e-4 of the rows, plus 2)."""
    gp = np.asarray(gap).reshape(-1)
    if network:
        assert (gp[bad] < KEY_GAP).all(), f"mismatch outside the key band: gaps {gp[bad].max():.3e}"
    else:
        assert len(bad) <= 1e-4 * n_rows + 2, f"{len(bad)} near-tie mismatches"


def assert_close(gpu, ref, dtype, what="output"):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    if gpu.size == 0:
        return
    assert np.isfinite(gpu).all(), f"{what}: non-finite values"
    err = np.abs(gpu - ref)
    tol = TOL[dtype]
    assert err.max() <= tol["max_abs"], f"{what}: max abs err {err.max():.3e} > {tol['max_abs']}"
    assert err.mean() <= tol["mean_abs"], f"{what}: mean abs err {err.mean():.3e} > {tol['mean_abs']}"


def index_mismatches(gpu_idx, ref_idx, gap):
    """Rows (flattened) where indices differ; asserts each is a near-tie."""
    g = np.asarray(gpu_idx).reshape(-1, gpu_idx.shape[-1])
    r = np.asarray(ref_idx).reshape(-1, ref_idx.shape[-1])
    bad = np.nonzero((g != r).any(axis=1))[0]
    gp = np.asarray(gap).reshape(-1)
    not_tie = bad[gp[bad] >= TIE_GAP]
    assert len(not_tie) == 0, (f"{len(not_tie)} index rows differ beyond the near-tie band, "
                               f"first row {not_tie[0]}: gpu {g[not_tie[0]]} oracle {r[not_tie[0]]}")
    return bad


def check_forward(q, k, v, cu, B, topk, out_gpu, lse_gpu=None, idx_gpu=None, indices=None,
                  shared_routing=False, prefix_mean=False):
    """Full oracle comparison of a forward result (small shapes)."""
    dtype = q.dtype
    ref, ref_lse, ref_idx, _ = oracle.forward(q.cpu(), k.cpu(), v.cpu(), cu.cpu(), B, topk,
                                              indices=None if indices is None else indices.cpu(),
                                              shared_routing=shared_routing,
                                              prefix_mean=prefix_mean)
    out = out_gpu.float().cpu().numpy()
    T, Hq = q.shape[:2]
    if idx_gpu is not None and indices is None:
        _, gap = oracle.gate_topk(q.cpu(), k.cpu(), cu.cpu(), B, topk,
                                  shared_routing=shared_routing, prefix_mean=prefix_mean)
        bad = index_mismatches(idx_gpu.cpu().numpy(), ref_idx, gap)
        if len(bad):
            # near-tie rows: the oracle with the GPU's own choice
            gi = idx_gpu.cpu().numpy().reshape(T * Hq, topk)[bad]
            o2, l2, _, _ = oracle.forward_rows(q.cpu(), k.cpu(), v.cpu(), cu.cpu(), B, topk, bad,
                                               indices=gi, prefix_mean=prefix_mean)
            ref = ref.reshape(T * Hq, -1).copy()
            ref[bad] = o2
            ref = ref.reshape(out.shape)
            ref_lse = ref_lse.reshape(-1).copy()
            ref_lse[bad] = l2
            ref_lse = ref_lse.reshape(T, Hq)
    assert_close(out, ref, dtype)
    if lse_gpu is not None:
        assert np.abs(lse_gpu.cpu().numpy() - ref_lse).max() <= (1e-3 if dtype == torch.bfloat16
                                                                 else 1e-4)
    return ref


def check_rows(q, k, v, cu, B, topk, rows, out_gpu, idx_gpu=None, lse_gpu=None,
               prefix_mean=False):
    """Sampled oracle comparison on flattened rows (row = t * Hq + h)."""
    dtype = q.dtype
    T, Hq, d = q.shape
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    rows = np.asarray(rows, dtype=np.int64)
    ref, ref_lse, ref_idx, gap = oracle.forward_rows(qc, kc, vc, cu.cpu(), B, topk, rows,
                                                     prefix_mean=prefix_mean)
    if idx_gpu is not None:
        gi = idx_gpu.reshape(T * Hq, topk)[torch.as_tensor(rows, device=idx_gpu.device)].cpu().numpy()
        bad = index_mismatches(gi, ref_idx, gap)
        if len(bad):
            o2, l2, _, _ = oracle.forward_rows(qc, kc, vc, cu.cpu(), B, topk, rows[bad],
                                               indices=gi[bad], prefix_mean=prefix_mean)
            ref[bad] = o2
            ref_lse[bad] = l2
    sel = torch.as_tensor(rows, device=out_gpu.device)
    out = out_gpu.reshape(T * Hq, d)[sel].float().cpu().numpy()
    assert_close(out, ref, dtype)
    if lse_gpu is not None:
        l = lse_gpu.reshape(-1)[sel].cpu().numpy()
        assert np.abs(l - ref_lse).max() <= (1e-3 if dtype == torch.bfloat16 else 1e-4)
