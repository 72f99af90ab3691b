"""GPU decode step (the last few positions of each request against its KV
cache; PaperTrace "2.1.3 MoBA", sections 5.1 and 5.4) and the incremental
block means, against the oracle: a decode query must get exactly the prefill
forward's result for its position, so the reference is the oracle's sampled
forward on those rows of the cache."""
import numpy as np
import pytest
import torch

import long_context_prefill_block_b200 as moba
import oracle
from moba_inputs import WORKLOADS, make_inputs, small_case
from parity import assert_close, index_mismatches

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _decode_rows(cu, n_new, Hq):
    """Flattened (token * Hq + head) rows of each request's last n_new[r] positions, in the
    order moba_decode returns them."""
    rows = []
    for r in range(len(cu) - 1):
        for j in range(n_new[r]):
            t = int(cu[r + 1]) - n_new[r] + j
            rows.extend(t * Hq + h for h in range(Hq))
    return np.asarray(rows, dtype=np.int64)


def _run_decode(q_all, k, v, cu, n_new, B, topk, shared=False):
    """Decode the last n_new[r] positions of each request, with q taken from q_all."""
    Hq = q_all.shape[1]
    rows = _decode_rows(cu, n_new, Hq)
    tok = rows[::Hq] // Hq
    q = q_all[torch.as_tensor(tok)].contiguous()
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum(n_new)]), dtype=torch.int32)
    kd, vd = k.to(DEV), v.to(DEV)
    kbar = moba.moba_meanpool(kd, cu.to(DEV), B)
    out, lse, idx = moba.moba_decode(q.to(DEV), kd, vd, cu, cu_q, kbar, B, topk,
                                     shared_routing=shared, return_lse=True, return_idx=True)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    return rows, out.cpu(), lse.cpu(), idx.cpu()


def _check(q_all, k, v, cu, B, topk, rows, out, lse, idx, shared=False):
    dtype = q_all.dtype
    Hq, d = q_all.shape[1], q_all.shape[2]
    if shared:
        ref_idx_all, gap_all = oracle.gate_topk(q_all, k, cu, B, topk, shared_routing=True)
        ref_idx = ref_idx_all.reshape(-1, topk)[rows]
        gap = gap_all.reshape(-1)[rows]
        ref, ref_lse, _, _ = oracle.forward_rows(q_all, k, v, cu, B, topk, rows, indices=ref_idx)
    else:
        ref, ref_lse, ref_idx, gap = oracle.forward_rows(q_all, k, v, cu, B, topk, rows)
    gi = idx.numpy().reshape(-1, topk)
    bad = index_mismatches(gi, ref_idx, gap)
    if len(bad):
        o2, l2, _, _ = oracle.forward_rows(q_all, k, v, cu, B, topk, rows[bad], indices=gi[bad])
        ref[bad] = o2
        ref_lse[bad] = l2
    assert_close(out.float().numpy().reshape(-1, d), ref, dtype)
    tol = 1e-3 if dtype == torch.bfloat16 else 1e-4
    assert np.abs(lse.numpy().reshape(-1) - ref_lse).max() <= tol


CASES = [
    # lengths, Hq, Hkv, d, B, topk, dtype, queries per request
    ((5000, 1300, 700), 4, 2, 128, 128, 3, torch.bfloat16, (1, 1, 1)),
    ((4096, 2000), 2, 1, 128, 512, 4, torch.bfloat16, (3, 5)),          # speculative drafts
    ((3000, 40, 900), 8, 2, 128, 256, 9, torch.bfloat16, (2, 0, 1)),    # a request with no query
    ((1500, 777), 2, 2, 64, 64, 5, torch.float32, (1, 4)),              # fp32, d = 64
    ((2500,), 4, 4, 64, 100, 3, torch.bfloat16, (7,)),                  # B not a multiple of 32
    ((9000,), 2, 1, 128, 1024, 3, torch.bfloat16, (1,)),                # two 512-key splits per block
]


@pytest.mark.parametrize("case", CASES)
def test_decode_matches_oracle(case):
    lengths, Hq, Hkv, d, B, topk, dtype, n_new = case
    q, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=dtype, seed=631)
    rows, out, lse, idx = _run_decode(q, k, v, cu, n_new, B, topk)
    _check(q, k, v, cu, B, topk, rows, out, lse, idx)


def test_decode_shared_routing():
    q, k, v, cu = small_case((3000, 1800), 8, 2, 128, 128, 4, dtype=torch.bfloat16, seed=632)
    rows, out, lse, idx = _run_decode(q, k, v, cu, (2, 1), 128, 4, shared=True)
    i = idx.numpy()
    for h in range(8):
        assert (i[:, h] == i[:, (h // 4) * 4]).all()
    _check(q, k, v, cu, 128, 4, rows, out, lse, idx, shared=True)


def test_decode_equals_prefill_rows():
    # the decode of the last position is the prefill forward's last row
    q, k, v, cu = small_case((4000, 2500), 4, 2, 128, 256, 3, dtype=torch.bfloat16, seed=633)
    rows, out, lse, idx = _run_decode(q, k, v, cu, (1, 1), 256, 3)
    full, full_lse = moba.moba_forward(q.to(DEV), k.to(DEV), v.to(DEV), cu, 256, 3,
                                       return_lse=True)
    gidx = moba.moba_gate_topk(q.to(DEV), k.to(DEV), cu, 256, 3).cpu().reshape(-1, 3)
    same = (gidx[torch.as_tensor(rows)] == idx.reshape(-1, 3)).all(dim=1)
    assert same.float().mean() > 0.99
    ref = full.cpu().reshape(-1, 128)[torch.as_tensor(rows)][same].float()
    got = out.reshape(-1, 128)[same].float()
    assert (ref - got).abs().max() <= 2e-2


def test_meanpool_update_is_the_full_mean_of_touched_blocks():
    lengths, Hkv, d, B = (3000, 700, 1030), 2, 128, 128
    _, k, _, cu = small_case(lengths, 2, Hkv, d, B, 3, dtype=torch.bfloat16, seed=634)
    n_new = (1, 200, 3)  # the last tokens of each request were just appended
    before = torch.tensor(np.concatenate([[0], np.cumsum([n - a for n, a in zip(lengths, n_new)])]),
                          dtype=torch.int32)
    keep = torch.cat([torch.arange(int(cu[r]), int(cu[r + 1]) - n_new[r]) for r in range(3)])
    kd = k.to(DEV)
    max_len = max(lengths)
    old = moba.moba_meanpool(k[keep].contiguous().to(DEV), before.to(DEV), B, max_seqlen=max_len)
    kbar = old.clone()
    cu_new = torch.tensor(np.concatenate([[0], np.cumsum(n_new)]), dtype=torch.int32)
    moba.moba_meanpool_update(kd, cu, cu_new, kbar, B, max(n_new), max_seqlen=max_len)
    full = moba.moba_meanpool(kd, cu.to(DEV), B, max_seqlen=max_len)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    for r in range(3):
        L, n = lengths[r], n_new[r]
        touched = set(range((L - n) // B, (L - 1) // B + 1))
        for i in range(kbar.shape[1]):
            if i in touched:
                assert torch.equal(kbar[r, i], full[r, i]), (r, i)
            else:
                assert torch.equal(kbar[r, i], old[r, i]), (r, i)
    ref = oracle.meanpool(k, cu, B)
    nb = ref.shape[1]
    assert np.abs(kbar[:, :nb].cpu().numpy() - ref).max() <= 1e-5 * max(1.0, np.abs(ref).max())


def test_decode_at_scaling_size():
    w = WORKLOADS["scaling_8k"]
    q_all, k, v, cu = make_inputs(w, DEV)
    n_new = (1,) * w.batch
    T, Hq = q_all.shape[:2]
    rows = _decode_rows(cu, n_new, Hq)
    q = q_all[torch.as_tensor(rows[::Hq] // Hq, device=DEV)].contiguous()
    kbar = moba.moba_meanpool(k, cu.to(DEV), w.block_size, max_seqlen=w.max_seqlen)
    cu_q = torch.arange(w.batch + 1, dtype=torch.int32)
    out, lse, idx = moba.moba_decode(q, k, v, cu, cu_q, kbar, w.block_size, w.topk,
                                     max_seqlen=w.max_seqlen, return_lse=True, return_idx=True)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    _check(q_all.cpu(), k.cpu(), v.cpu(), cu, w.block_size, w.topk, rows, out.cpu(), lse.cpu(),
           idx.cpu())


@pytest.mark.parametrize("case", CASES[:4])
def test_decode_head_major_cache(case):
    # the same caches laid out head by head ([Hkv, T, d], moba_params.kv_layout = 1): the
    # block means and the decode results are bit-identical to the packed cache's, and the
    # oracle agrees; an append refreshes the means in the head-major layout too
    lengths, Hq, Hkv, d, B, topk, dtype, n_new = case
    q_all, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=dtype, seed=441)
    rows, out, lse, idx = _run_decode(q_all, k, v, cu, n_new, B, topk)
    tok = torch.as_tensor(rows[::Hq] // Hq)
    q = q_all[tok].contiguous().to(DEV)
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum(n_new)]), dtype=torch.int32)
    kh = k.transpose(0, 1).contiguous().to(DEV)
    vh = v.transpose(0, 1).contiguous().to(DEV)
    kbar_p = moba.moba_meanpool(k.to(DEV), cu.to(DEV), B)
    kbar_h = moba.moba_meanpool(kh, cu.to(DEV), B, kv_head_major=True)
    out_h, lse_h, idx_h = moba.moba_decode(q, kh, vh, cu, cu_q, kbar_h, B, topk, return_lse=True,
                                           return_idx=True, kv_head_major=True)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
    assert torch.equal(kbar_h, kbar_p)
    assert torch.equal(idx_h.cpu(), idx) and torch.equal(lse_h.cpu(), lse)
    assert torch.equal(out_h.cpu(), out)
    _check(q_all, k, v, cu, B, topk, rows, out_h.cpu(), lse_h.cpu(), idx_h.cpu())
    # incremental block means: recompute the blocks of each request's last positions
    kbar_u = kbar_h.clone()
    kbar_u[:] = 0
    cu_new = torch.tensor(np.concatenate([[0], np.cumsum(n_new)]), dtype=torch.int32)
    moba.moba_meanpool_update(kh, cu.to(DEV), cu_new, kbar_u, B, max(max(n_new), 1),
                              kv_head_major=True)
    torch.cuda.synchronize()
    for r, n in enumerate(n_new):
        L = int(cu[r + 1] - cu[r])
        for blk in sorted({(L - 1 - j) // B for j in range(n)}):
            assert torch.equal(kbar_u[r, blk], kbar_p[r, blk])


def test_prefill_refuses_head_major_kv():
    q, k, v, cu = small_case((300,), 2, 2, 128, 128, 3, dtype=torch.bfloat16, seed=442)
    p = moba.make_params(q, k, cu, 128, 3)
    p.kv_layout = 1
    ws = moba.workspace(p, DEV)
    L = moba.lib()
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out = torch.empty_like(qd)
    cu_d = cu.to(DEV)
    ptr = lambda x: moba.ctypes.c_void_p(x.data_ptr())
    rc = L.moba_forward(moba.ctypes.byref(p), ptr(qd), ptr(kd), ptr(vd), ptr(cu_d), ptr(out), None,
                        ptr(ws), ws.numel(), None)
    assert rc == moba.MOBA_ERR_UNSUPPORTED
    p.kv_layout = 2
    assert moba.moba_workspace_size(p) == 0  # invalid layout value
