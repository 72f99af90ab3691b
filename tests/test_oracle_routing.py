"""Pins of the oracle's shared-routing variant (PaperTrace "2.1.3 MoBA",
section 5.5, multi-head settings: the query heads of a group share their
candidate blocks, chosen on the group's mean score). Each pin reduces the
variant to the per-head gate, which tests/test_oracle_pins.py pins to the
pages' worked example, brute force and closed forms."""
import numpy as np
import torch

import oracle
from moba_inputs import small_case

TIE = 1e-9  # rows whose per-head gap is below this are not compared


def _gate(q, k, cu, B, topk, shared):
    return oracle.gate_topk(q, k, cu, B, topk, shared_routing=shared)


def test_one_head_per_group_is_per_head_routing():
    q, k, v, cu = small_case((700, 300), 3, 3, 16, 32, 4, dtype=torch.float32, seed=301)
    a, ga = _gate(q, k, cu, 32, 4, False)
    b, gb = _gate(q, k, cu, 32, 4, True)
    assert (a == b).all()
    assert np.array_equal(ga, gb)


def test_identical_heads_share_their_own_choice():
    q, k, v, cu = small_case((900,), 4, 1, 16, 32, 3, dtype=torch.float32, seed=302)
    q[:, 1:] = q[:, :1]  # every head of the group asks the same question
    a, ga = _gate(q, k, cu, 32, 3, False)
    b, _ = _gate(q, k, cu, 32, 3, True)
    keep = ga[:, 0] >= TIE
    assert (a[keep] == b[keep]).all()


def test_group_choice_is_the_choice_of_the_mean_query():
    # q_h = qbar + delta_h with sum_h delta_h = 0, all on a dyadic grid so every
    # stored value and the mean are exact in fp32: the shared choice must be
    # the per-head choice of a one-head problem asking qbar
    rng = np.random.default_rng(303)
    T, grp, d, B, topk = 1200, 4, 16, 40, 4
    qbar = np.round(rng.standard_normal((T, 1, d)) * 256) / 1024
    delta = np.round(rng.standard_normal((T, grp, d)) * 256) / 1024
    delta[:, 0] = -delta[:, 1:].sum(axis=1)
    q = torch.tensor(qbar + delta, dtype=torch.float32)
    assert torch.equal(q.double().mean(dim=1, keepdim=True), torch.tensor(qbar))
    k = torch.tensor(rng.standard_normal((T, 1, d)), dtype=torch.float32)
    cu = torch.tensor([0, T], dtype=torch.int32)
    shared, _ = _gate(q, k, cu, B, topk, True)
    ref, gap = _gate(torch.tensor(qbar, dtype=torch.float32), k, cu, B, topk, False)
    keep = gap[:, 0] >= TIE
    assert keep.mean() > 0.99
    for h in range(grp):
        assert (shared[keep, h] == ref[keep, 0]).all()


def test_shared_choice_is_symmetric_and_common_to_the_group():
    q, k, v, cu = small_case((800, 500), 8, 2, 16, 32, 5, dtype=torch.float32, seed=304)
    a, _ = _gate(q, k, cu, 32, 5, True)
    perm = torch.tensor([3, 1, 0, 2, 7, 4, 6, 5])  # within each group of 4
    b, _ = _gate(q[:, perm].contiguous(), k, cu, 32, 5, True)
    assert (a == b).all()
    for g in range(2):
        for h in range(4 * g + 1, 4 * g + 4):
            assert (a[:, h] == a[:, 4 * g]).all()


def test_shared_forward_attends_the_shared_blocks():
    q, k, v, cu = small_case((300, 200), 4, 2, 16, 32, 3, dtype=torch.float32, seed=305)
    out, lse, idx, _ = oracle.forward(q, k, v, cu, 32, 3, shared_routing=True)
    gate, _ = _gate(q, k, cu, 32, 3, True)
    assert (idx == gate).all()
    out2, lse2, _, _ = oracle.forward(q, k, v, cu, 32, 3, indices=gate)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
