"""Pins of the oracle's prefix-mean own-block variant (PaperTrace "2.1.3 MoBA",
section 5.2, the paragraph on causal blocks: a gate must not score the own
block by its full mean, which holds keys after the query; it either forces
the own block in, the default, or scores it by the mean of its keys up to
the query). With the prefix mean the own block competes with the earlier
blocks for the k slots, and a query whose own block loses reads no key of
it, itself included.

The pins: closed forms for a one-dimensional case worked by hand, the tie
rule, brute force over every candidate subset on tiny random inputs (with
textbook masked softmax for the output), the full budget, and the
finite-difference check of the backward."""
import itertools
import math

import numpy as np
import torch

import oracle
from moba_inputs import small_case


def _one_dim(keys, queries, values):
    t = lambda x: torch.tensor(x, dtype=torch.float32).reshape(-1, 1, 1)
    return t(queries), t(keys), t(values), torch.tensor([0, len(keys)], dtype=torch.int32)


def _softmax_avg(logits, vals):
    m = max(logits)
    w = [math.exp(x - m) for x in logits]
    return sum(a * b for a, b in zip(w, vals)) / sum(w)


def test_hand_worked_one_dimensional_case():
    # d = 1 (scale 1), B = 2: block 0 = keys 1, 3 (mean 2); block 1 = keys 1, 5;
    # block 2 = keys 4, 0.
    keys = [1.0, 3.0, 1.0, 5.0, 4.0, 0.0]
    vals = [1.0, 2.0, 4.0, 8.0, 16.0, 32.0]
    queries = [0.5, 2.0, 1.0, 1.0, 1.0, -1.0]
    q, k, v, cu = _one_dim(keys, queries, vals)
    idx, _ = oracle.gate_topk(q, k, cu, 2, 1, prefix_mean=True)
    out, lse, idx2, nkeys = oracle.forward(q, k, v, cu, 2, 1, prefix_mean=True)
    assert (idx == idx2).all()
    # p = 0, 1: block 0 is the only candidate
    assert idx[0, 0, 0] == 0 and idx[1, 0, 0] == 0
    assert out[0, 0, 0] == 1.0
    assert math.isclose(out[1, 0, 0], _softmax_avg([2.0, 6.0], [1.0, 2.0]), rel_tol=1e-14)
    # p = 2: s_0 = 1 * 2 = 2 beats the prefix mean 1 (key 1 alone): block 0 only,
    # and the query does not see itself
    assert idx[2, 0, 0] == 0 and nkeys[2, 0] == 2
    assert math.isclose(out[2, 0, 0], _softmax_avg([1.0, 3.0], [1.0, 2.0]), rel_tol=1e-14)
    # p = 3: prefix mean (1 + 5) / 2 = 3 beats 2: the own block, keys 2 and 3
    assert idx[3, 0, 0] == 1 and nkeys[3, 0] == 2
    assert math.isclose(out[3, 0, 0], _softmax_avg([1.0, 5.0], [4.0, 8.0]), rel_tol=1e-14)
    # p = 4 (block 2, q = 1): means 2, 3 and the prefix mean 4: the own block
    assert idx[4, 0, 0] == 2
    assert math.isclose(out[4, 0, 0], 16.0, rel_tol=1e-14)
    # p = 5 (q = -1): scores -2, -3 and -(4 + 0)/2 = -2: block 0 and the own
    # block tie, the lower index wins
    assert idx[5, 0, 0] == 0
    assert math.isclose(out[5, 0, 0], _softmax_avg([-1.0, -3.0], [1.0, 2.0]), rel_tol=1e-14)
    assert math.isclose(lse[5, 0], math.log(math.exp(-1.0) + math.exp(-3.0)), rel_tol=1e-14)
    # k = 2 at p = 5: block 0 and the own block (score -2 each) beat block 1 (-3)
    idx_k2, _ = oracle.gate_topk(q, k, cu, 2, 2, prefix_mean=True)
    assert list(idx_k2[5, 0]) == [0, 2]
    # the forced gate keeps the own block at every position
    forced, _ = oracle.gate_topk(q, k, cu, 2, 1)
    assert list(forced[:, 0, 0]) == [0, 0, 1, 1, 2, 2]


def _subset_choice(scores, k):
    """The k-subset (k = min(k, n)) of candidates 0..n-1 with the largest score
    sum; distinct random scores make it unique."""
    n = len(scores)
    best, best_sum = None, -math.inf
    for sub in itertools.combinations(range(n), min(k, n)):
        s = sum(scores[i] for i in sub)
        if s > best_sum:
            best, best_sum = sub, s
    return sorted(best)


def test_choice_is_the_best_subset_and_output_is_masked_softmax():
    rng = np.random.default_rng(611)
    for (lens, Hq, Hkv, d, B, topk) in [((37,), 2, 1, 4, 4, 2), ((25, 18), 2, 2, 3, 3, 3),
                                        ((30,), 1, 1, 2, 5, 1)]:
        T = sum(lens)
        q = torch.tensor(rng.standard_normal((T, Hq, d)), dtype=torch.float32)
        k = torch.tensor(rng.standard_normal((T, Hkv, d)), dtype=torch.float32)
        v = torch.tensor(rng.standard_normal((T, Hkv, d)), dtype=torch.float32)
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
        out, _, idx, _ = oracle.forward(q, k, v, cu, B, topk, prefix_mean=True)
        qd, kd, vd = q.double().numpy(), k.double().numpy(), v.double().numpy()
        grp = Hq // Hkv
        for b, n in enumerate(lens):
            s0 = int(cu[b])
            for p in range(n):
                c = p // B
                for h in range(Hq):
                    g = h // grp
                    kk = kd[s0:s0 + n, g]
                    qq = qd[s0 + p, h]
                    scores = [float(qq @ kk[i * B:(i + 1) * B].mean(axis=0)) for i in range(c)]
                    scores.append(float(qq @ kk[c * B:p + 1].mean(axis=0)))
                    chosen = _subset_choice(scores, topk)
                    row = [int(x) for x in idx[s0 + p, h] if x >= 0]
                    assert row == chosen, (b, p, h)
                    keys = [j for j in range(p + 1) if j // B in chosen]
                    logits = np.array([qq @ kk[j] for j in keys]) / math.sqrt(d)
                    w = np.exp(logits - logits.max())
                    ref = (w[:, None] * vd[s0:s0 + n, g][keys]).sum(axis=0) / w.sum()
                    np.testing.assert_allclose(out[s0 + p, h], ref, rtol=0, atol=1e-12)


def test_full_budget_is_dense_causal():
    q, k, v, cu = small_case((130, 75), 4, 2, 8, 16, 9, dtype=torch.float32, seed=612)
    out, lse, idx, _ = oracle.forward(q, k, v, cu, 16, 9, prefix_mean=True)
    ref, ref_lse = oracle.dense_causal(q, k, v, cu)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_unchosen_own_block_is_never_read():
    q, k, v, cu = small_case((400,), 2, 1, 8, 20, 2, dtype=torch.float32, seed=613)
    out, _, idx, _ = oracle.forward(q, k, v, cu, 20, 2, prefix_mean=True)
    T = q.shape[0]
    pos = np.arange(T)
    c = pos // 20
    dropped = ~(idx == c[:, None, None]).any(axis=2)  # [T, Hq]
    assert 0.05 < dropped.mean() < 0.95
    # new values for the own block of every row whose own block lost: block 7
    rows = (c == 7)
    v2 = v.clone()
    v2[torch.tensor(rows)] += 3.0
    out2, _, idx2, _ = oracle.forward(q, k, v2, cu, 20, 2, prefix_mean=True)
    assert (idx2 == idx).all()
    sel = rows[:, None] & dropped
    assert sel.any() and (rows[:, None] & ~dropped).any()
    assert np.array_equal(out2[sel], out[sel])
    assert not np.allclose(out2[rows[:, None] & ~dropped], out[rows[:, None] & ~dropped])


def test_mask_route_and_shared_one_head_groups_agree():
    q, k, v, cu = small_case((150, 90), 3, 3, 8, 12, 3, dtype=torch.float32, seed=614)
    out, _, idx, _ = oracle.forward(q, k, v, cu, 12, 3, prefix_mean=True)
    mask = oracle.forward_mask(q, k, v, cu, 12, 3, prefix_mean=True)
    np.testing.assert_allclose(mask, out, rtol=0, atol=1e-12)
    shared, _ = oracle.gate_topk(q, k, cu, 12, 3, shared_routing=True, prefix_mean=True)
    assert (shared == idx).all()


def _dyadic(rng, shape, scale=64):
    return torch.tensor(np.round(rng.standard_normal(shape) * scale) / 256, dtype=torch.float32)


def test_backward_matches_central_differences():
    rng = np.random.default_rng(615)
    T, Hq, Hkv, d, B, topk = 80, 2, 1, 8, 16, 2
    q, k, v = _dyadic(rng, (T, Hq, d)), _dyadic(rng, (T, Hkv, d)), _dyadic(rng, (T, Hkv, d))
    dO = _dyadic(rng, (T, Hq, d))
    cu = torch.tensor([0, T], dtype=torch.int32)
    idx, gap = oracle.gate_topk(q, k, cu, B, topk, prefix_mean=True)
    c = np.arange(T) // B
    assert not (idx == c[:, None, None]).any(axis=2).all()  # some own blocks lost
    dq, dk, dv = oracle.backward(q, k, v, dO, cu, B, topk, prefix_mean=True)

    def loss(qq, kk, vv):
        out, _, ix, _ = oracle.forward(qq, kk, vv, cu, B, topk, prefix_mean=True)
        return float((out * dO.double().numpy()).sum()), ix

    eps = 2.0 ** -12
    checked = 0
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(10):
            i = tuple(int(rng.integers(0, n)) for n in x.shape)
            args = {"q": q, "k": k, "v": v}
            xp, xm = x.clone(), x.clone()
            xp[i] += eps
            xm[i] -= eps
            args[name] = xp
            lp, ip = loss(args["q"], args["k"], args["v"])
            args[name] = xm
            lm, im = loss(args["q"], args["k"], args["v"])
            if not ((ip == idx).all() and (im == idx).all()):
                continue  # the step moved a block choice: no derivative there
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - g[i]) <= 1e-6 * max(1.0, abs(fd)), (name, i, fd, g[i])
            checked += 1
    assert checked >= 24
