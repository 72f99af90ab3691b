"""Pins for the fp64 oracle: values the pages print, closed forms, textbook
special cases and brute force on tiny inputs. Nothing here compares the
oracle with itself or with the CUDA path.

Pages: PaperTrace knowledge page "2.1.3 MoBA" (sections 1-3.1, 5.2, 5.5, the
worked example of section 2 and Figure 1), and the translated MoBA README
(moba_naive = attention-mask view).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from moba_inputs import cu_seqlens_of, small_case

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers
def sdpa_with_mask(q, k, v, cu, allowed):
    """Library reference: torch SDPA (float64) per sequence and head with the
    boolean mask allowed(p, j) (positions relative to the sequence)."""
    q64, k64, v64 = (x.to(torch.float64) for x in (q, k, v))
    T, Hq, d = q.shape
    grp = Hq // k.shape[1]
    out = torch.zeros((T, Hq, d), dtype=torch.float64)
    cu = [int(x) for x in cu]
    for b in range(len(cu) - 1):
        s, e = cu[b], cu[b + 1]
        n = e - s
        if n == 0:
            continue
        m = torch.tensor([[allowed(p, j) for j in range(n)] for p in range(n)], dtype=torch.bool)
        qs = q64[s:e].permute(1, 0, 2)                                   # [Hq, n, d]
        ks = k64[s:e].repeat_interleave(grp, dim=1).permute(1, 0, 2)
        vs = v64[s:e].repeat_interleave(grp, dim=1).permute(1, 0, 2)
        out[s:e] = F.scaled_dot_product_attention(qs, ks, vs, attn_mask=m).permute(1, 0, 2)
    return out.numpy()


def worked_example_inputs(k6=7.0, v_unprinted=(-3.0, 5.0, 11.0)):
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    keys = [g["keys_1indexed"][str(i)] for i in range(1, 6)] + [k6]
    vals = [v_unprinted[0], v_unprinted[1]] + [g["values_1indexed"][str(i)] for i in (3, 4, 5)] + \
           [v_unprinted[2]]
    qs = [0.5, -1.0, 2.0, 0.25, g["q_at_query"], 1.5]  # only position 5 (1-indexed) is checked
    t = lambda a: torch.tensor(a, dtype=torch.float32).reshape(6, 1, 1)
    return g, t(qs), t(keys), t(vals), cu_seqlens_of([6])


# ------------------------------------------------------- worked example
def test_worked_example_gate_and_output():
    g, q, k, v, cu = worked_example_inputs()
    B, topk = g["block_size"], g["topk"]
    p = g["query_position_1indexed"] - 1
    kbar = oracle.meanpool(k, cu, B)
    assert kbar[0, :2, 0, 0].tolist() == g["block_mean_scores"]  # q = 1, so scores = means
    out, lse, idx, nkeys = oracle.forward(q, k, v, cu, B, topk)
    hist = g["selected_history_block_1indexed"] - 1
    assert idx[p, 0].tolist() == [hist, p // B]
    cand = [c - 1 for c in g["candidates_1indexed"]]
    assert nkeys[p, 0] == len(cand)
    w = [math.exp(float(k[j, 0, 0]) * 1.0 - lse[p, 0]) for j in cand]
    tol = 0.5 * 10 ** -g["weights_printed_decimals"]
    assert np.allclose(w, g["weights"], atol=tol)
    assert abs(out[p, 0, 0] - g["output"]) <= 0.5 * 10 ** -g["output_printed_decimals"]


def test_worked_example_unprinted_entries_do_not_matter():
    g, q, k, v, cu = worked_example_inputs()
    p = g["query_position_1indexed"] - 1
    base = oracle.forward(q, k, v, cu, g["block_size"], g["topk"])[0][p, 0, 0]
    _, q2, k2, v2, _ = worked_example_inputs(k6=-40.0, v_unprinted=(100.0, -7.0, 1e3))
    alt = oracle.forward(q2, k2, v2, cu, g["block_size"], g["topk"])[0][p, 0, 0]
    assert base == alt


def test_worked_example_two_branch_merge_and_naive_sum():
    g, q, k, v, cu = worked_example_inputs()
    p = g["query_position_1indexed"] - 1
    merged = oracle.forward_two_branch(q, k, v, cu, g["block_size"], g["topk"])[p, 0, 0]
    assert abs(merged - g["output"]) <= 0.5e-4
    # Adding two separately normalised branch outputs gives the current value a
    # whole unit of weight: 30 + (10 + 20 e^-2)/(1 + e^-2) -- far from 11.98.
    naive = oracle.forward_two_branch(q, k, v, cu, g["block_size"], g["topk"], naive_sum=True)[p, 0, 0]
    assert abs(naive - (30.0 + (10 + 20 * math.exp(-2)) / (1 + math.exp(-2)))) < 1e-12
    assert abs(naive - g["output"]) > 1.0


def test_worked_example_mask_view():
    g, q, k, v, cu = worked_example_inputs()
    p = g["query_position_1indexed"] - 1
    assert abs(oracle.forward_mask(q, k, v, cu, g["block_size"], g["topk"])[p, 0, 0] - g["output"]) <= 0.5e-4


# ------------------------------------------------ textbook special cases
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_full_budget_equals_dense_causal(dtype):
    # k covering every legal block recovers full causal attention (section 4).
    lengths, B = (37, 64, 20), 8
    q, k, v, cu = small_case(lengths, 4, 2, 8, B, 1, dtype=dtype, seed=3)
    topk = max(lengths) // B + 1
    ref = sdpa_with_mask(q, k, v, cu, lambda p, j: j <= p)
    out = oracle.forward(q, k, v, cu, B, topk)[0]
    dense, lse = oracle.dense_causal(q, k, v, cu)
    assert np.abs(out - ref).max() < 1e-12
    assert np.abs(dense - ref).max() < 1e-12


def test_topk_one_is_block_diagonal_causal():
    lengths, B = (40, 33), 8
    q, k, v, cu = small_case(lengths, 2, 1, 4, B, 1, dtype=torch.float32, seed=4)
    ref = sdpa_with_mask(q, k, v, cu, lambda p, j: j <= p and j // B == p // B)
    out, _, idx, _ = oracle.forward(q, k, v, cu, B, 1)
    assert np.abs(out - ref).max() < 1e-12
    T = q.shape[0]
    pos = np.concatenate([np.arange(n) for n in lengths])
    assert (idx[:, :, 0] == (pos // B)[:, None]).all()


def test_uniform_logits_closed_form():
    # q = 0: every logit and every gate score is 0, so ties go to the lowest
    # block indices, the output is the plain mean of V over the candidates
    # and lse = log(number of candidates).
    n, B, topk, d = 50, 4, 3, 4
    _, k, v, cu = small_case((n,), 1, 1, d, B, topk, dtype=torch.float32, seed=5)
    q = torch.zeros((n, 1, d))
    out, lse, idx, nkeys = oracle.forward(q, k, v, cu, B, topk)
    v64 = v.double().numpy()
    for p in range(n):
        c = p // B
        hist = list(range(min(topk - 1, c)))
        assert idx[p, 0].tolist() == hist + [c] + [-1] * (topk - 1 - len(hist))
        J = [j for i in hist for j in range(i * B, (i + 1) * B)] + list(range(c * B, p + 1))
        assert nkeys[p, 0] == len(J)
        assert abs(lse[p, 0] - math.log(len(J))) < 1e-12
        assert np.abs(out[p, 0] - v64[J, 0].mean(0)).max() < 1e-12


def test_window_and_sink_as_forced_gates():
    # A gate that always picks the previous block gives a blocked sliding
    # window; adding block 0 gives sink + window (section 3).
    n, B, topk = 48, 4, 3
    q, k, v, cu = small_case((n,), 2, 2, 8, B, topk, dtype=torch.float32, seed=6)
    win = np.full((n, 2, topk), -1, np.int32)
    sink = np.full((n, 2, topk), -1, np.int32)
    for p in range(n):
        c = p // B
        win[p, :, :2] = [c - 1, c] if c >= 1 else [c, -1]
        row = sorted({0, c - 1, c} if c >= 1 else {c})
        sink[p, :, :len(row)] = row
    ref_w = sdpa_with_mask(q, k, v, cu, lambda p, j: j <= p and p // B - 1 <= j // B)
    ref_s = sdpa_with_mask(q, k, v, cu, lambda p, j: j <= p and (p // B - 1 <= j // B or j // B == 0))
    assert np.abs(oracle.forward(q, k, v, cu, B, topk, indices=win)[0] - ref_w).max() < 1e-12
    assert np.abs(oracle.forward(q, k, v, cu, B, topk, indices=sink)[0] - ref_s).max() < 1e-12


# ------------------------------------------------------ gate pins
def test_meanpool_closed_forms():
    # keys that are constant per block average to that constant; a linear
    # ramp averages to the mid-point; a trailing partial block averages the
    # tokens present.
    B, n, d = 4, 14, 3
    k = torch.zeros((n, 2, d))
    for j in range(n):
        k[j, 0, :] = float(j // B) * 2.0 - 1.0
        k[j, 1, :] = float(j)
    kbar = oracle.meanpool(k, cu_seqlens_of([n]), B)
    for i in range(4):
        j0, j1 = i * B, min(n, (i + 1) * B)
        assert (kbar[0, i, 0] == 2.0 * i - 1.0).all()
        assert (kbar[0, i, 1] == (j0 + j1 - 1) / 2.0).all()


def test_mean_dilution_example():
    # Section 5.2: one key scoring 8 among 255 scoring 0 -> block mean 8/256 =
    # 0.03125; 256 keys scoring 0.05 -> 0.05. The gate must pick the latter.
    B = 256
    k = torch.zeros((3 * B, 1, 1))
    k[17, 0, 0] = 8.0
    k[B:2 * B, 0, 0] = 0.05
    q = torch.ones((3 * B, 1, 1))
    v = torch.zeros((3 * B, 1, 1))
    cu = cu_seqlens_of([3 * B])
    kbar = oracle.meanpool(k, cu, B)
    assert kbar[0, 0, 0, 0] == 8.0 / 256.0 == 0.03125
    assert abs(kbar[0, 1, 0, 0] - 0.05) < 1e-9
    idx, gap = oracle.gate_topk(q, k, cu, B, 2)
    assert (idx[2 * B:, 0].tolist() == [[1, 2]] * B)


def test_routing_counterexample_planted():
    # Section 5.5: 64 blocks x 256 tokens, a single evidence key in block 7,
    # a block of moderately similar keys in block 31. Mean routing prefers
    # block 31; forcing block 7 lets exact attention find the evidence.
    B, nb, d = 256, 64, 16
    g = torch.Generator().manual_seed(11)
    k = torch.randn((nb * B, 1, d), generator=g) * 0.01
    k[:, 0, 0] = 0.0
    e = torch.zeros(d)
    e[0] = 1.0
    k[7 * B + 100, 0] = 60.0 * e      # block mean 60/256 ~ 0.23
    k[31 * B:32 * B, 0, 0] = 0.5      # block mean 0.5
    v = torch.zeros((nb * B, 1, d))
    v[7 * B + 100, 0, 1] = 1.0
    q = torch.zeros((nb * B, 1, d))
    q[:, 0, 0] = 1.0
    cu = cu_seqlens_of([nb * B])
    p = nb * B - 1
    out, _, idx, _ = oracle.forward_rows(q, k, v, cu, B, 2, [p])
    assert idx[0].tolist() == [31, nb - 1]
    assert abs(out[0, 1]) < 1e-6                 # evidence missed
    forced = np.array([[7, nb - 1]], np.int32)
    out7 = oracle.forward_rows(q, k, v, cu, B, 2, [p], indices=forced)[0]
    assert out7[0, 1] > 0.9                      # evidence found once block 7 is read


def test_tie_break_lower_index():
    # identical block means: every history score ties, the lowest indices win.
    B, n, topk = 4, 40, 4
    k = torch.ones((n, 1, 2))
    q = torch.randn((n, 1, 2), generator=torch.Generator().manual_seed(2))
    idx, gap = oracle.gate_topk(q, k, cu_seqlens_of([n]), B, topk)
    for p in range(n):
        c = p // B
        h = min(topk - 1, c)
        assert idx[p, 0, :h + 1].tolist() == list(range(h)) + [c]


def test_current_block_mean_never_competes():
    # Make the current block's full mean (which includes future keys) score
    # far above everything; it must neither be chosen as history nor change
    # the choice. Only earlier, complete blocks are scored.
    B, n, topk = 4, 24, 2
    g = torch.Generator().manual_seed(9)
    k = torch.randn((n, 1, 2), generator=g) * 0.1
    q = torch.ones((n, 1, 2))
    k[20:24, 0, :] = 100.0         # block 5 (the last)
    k[8:12, 0, :] = 1.0            # block 2: best history block
    idx, _ = oracle.gate_topk(q, k, cu_seqlens_of([n]), B, topk)
    for p in range(12, 20):
        assert idx[p, 0].tolist() == [2, p // B]
    for p in range(20, 24):
        assert idx[p, 0].tolist() == [2, 5]


def brute_force_moba(q, k, v, cu, B, topk):
    """Independent brute force: block means by torch.mean, all score sums over
    every subset of h history blocks, the best subset, then torch SDPA with
    the resulting boolean mask. Continuous random inputs (no ties)."""
    q64, k64, v64 = (x.to(torch.float64) for x in (q, k, v))
    T, Hq, d = q.shape
    grp = Hq // k.shape[1]
    out = torch.zeros((T, Hq, d), dtype=torch.float64)
    idx = np.full((T, Hq, topk), -1, np.int32)
    cu = [int(x) for x in cu]
    for b in range(len(cu) - 1):
        s, e = cu[b], cu[b + 1]
        n = e - s
        for h in range(Hq):
            kk = k64[s:e, h // grp]
            mask = torch.zeros((n, n), dtype=torch.bool)
            for p in range(n):
                c = p // B
                means = [kk[i * B:(i + 1) * B].mean(0) for i in range(c)]
                scores = [float(torch.dot(q64[s + p, h], m)) for m in means]
                hn = min(topk - 1, c)
                best = max(itertools.combinations(range(c), hn),
                           key=lambda S: sum(scores[i] for i in S))
                chosen = sorted(best) + [c]
                idx[s + p, h, :len(chosen)] = chosen
                for j in range(p + 1):
                    mask[p, j] = (j // B) in chosen
            qs = q64[s:e, h][None]
            ks = kk[None]
            vs = v64[s:e, h // grp][None]
            out[s:e, h] = F.scaled_dot_product_attention(qs, ks, vs, attn_mask=mask[None])[0]
    return out.numpy(), idx


@pytest.mark.parametrize("seed,lengths,Hq,Hkv,d,B,topk", [
    (21, (33,), 1, 1, 4, 4, 3),
    (22, (29, 40), 4, 2, 8, 4, 2),
    (23, (64, 17, 0, 31), 2, 1, 1, 8, 3),
    (24, (48,), 2, 2, 8, 2, 4),
])
def test_brute_force_tiny(seed, lengths, Hq, Hkv, d, B, topk):
    q, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=torch.float32, seed=seed,
                             offset_sigma=0.5)
    ref, ref_idx = brute_force_moba(q, k, v, cu, B, topk)
    out, lse, idx, _ = oracle.forward(q, k, v, cu, B, topk)
    assert (idx == ref_idx).all()
    assert np.abs(out - ref).max() < 1e-12
    gate_idx, _ = oracle.gate_topk(q, k, cu, B, topk)
    assert (gate_idx == ref_idx).all()
    # other oracle routes agree too
    assert np.abs(oracle.forward_mask(q, k, v, cu, B, topk) - ref).max() < 1e-12
    assert np.abs(oracle.forward_two_branch(q, k, v, cu, B, topk) - ref).max() < 1e-12


# ------------------------------------------------------ invariants
def test_attended_key_count_matches_sparsity_accounting():
    # eq.(9) accounting: a query at position p in block c reads min(k-1, c)
    # full history blocks plus p - cB + 1 keys of its own block.
    lengths, B, topk = (100, 64, 7), 8, 3
    q, k, v, cu = small_case(lengths, 2, 1, 4, B, topk, dtype=torch.float32, seed=8)
    nkeys = oracle.forward(q, k, v, cu, B, topk)[3]
    pos = np.concatenate([np.arange(n) for n in lengths])
    c = pos // B
    expect = np.minimum(topk - 1, c) * B + (pos - c * B + 1)
    assert (nkeys == expect[:, None]).all()


def test_varlen_equals_separate_sequences():
    lengths, B, topk = (24, 40, 9), 8, 2
    q, k, v, cu = small_case(lengths, 2, 1, 4, B, topk, dtype=torch.float32, seed=12)
    out, lse, idx, _ = oracle.forward(q, k, v, cu, B, topk)
    s = 0
    for n in lengths:
        o1, l1, i1, _ = oracle.forward(q[s:s + n], k[s:s + n], v[s:s + n], cu_seqlens_of([n]), B, topk)
        assert (o1 == out[s:s + n]).all() and (i1 == idx[s:s + n]).all()
        s += n


def test_gqa_equals_repeated_kv_heads():
    lengths, B, topk = (40,), 8, 3
    q, k, v, cu = small_case(lengths, 4, 2, 8, B, topk, dtype=torch.float32, seed=13)
    out, _, idx, _ = oracle.forward(q, k, v, cu, B, topk)
    kr, vr = k.repeat_interleave(2, dim=1), v.repeat_interleave(2, dim=1)
    out2, _, idx2, _ = oracle.forward(q, kr, vr, cu, B, topk)
    assert (out == out2).all() and (idx == idx2).all()


def test_rows_mode_matches_full():
    lengths, B, topk = (64, 40), 8, 3
    q, k, v, cu = small_case(lengths, 4, 2, 8, B, topk, dtype=torch.bfloat16, seed=14)
    out, lse, idx, _ = oracle.forward(q, k, v, cu, B, topk)
    rows = np.array([0, 5, 77, 200, 415])
    o, l, i, gap = oracle.forward_rows(q, k, v, cu, B, topk, rows)
    T, Hq = q.shape[:2]
    assert (o == out.reshape(T * Hq, -1)[rows]).all()
    assert (i == idx.reshape(T * Hq, -1)[rows]).all()
    assert (l == lse.reshape(-1)[rows]).all()


def test_rows_mode_with_only_the_sampled_q_rows():
    lengths, B, topk = (64, 40), 8, 3
    q, k, v, cu = small_case(lengths, 4, 2, 8, B, topk, dtype=torch.bfloat16, seed=15)
    rows = np.array([3, 99, 250, 300])
    full = oracle.forward_rows(q, k, v, cu, B, topk, rows)
    q_rows = q.reshape(-1, 8)[torch.as_tensor(rows)]
    part = oracle.forward_rows(None, k, v, cu, B, topk, rows, q_rows=q_rows, num_q_heads=4)
    for a, b in zip(full, part):
        assert (a == b).all()
