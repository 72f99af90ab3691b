"""Pins of the oracle backward (gradients of sum(dO * O) through the chosen
blocks' keys; the hard top-k passes no gradient, PaperTrace "2.1.3 MoBA"
section 5.3): central finite differences of the oracle forward, and the two
budget limits where MoBA is a textbook attention whose gradients torch's
autograd gives (full budget: dense causal; k = 1: block-diagonal causal)."""
import numpy as np
import torch

import oracle


def _dyadic(rng, shape, scale=64):
    # values on a 1/256 grid: x +- 2^-12 stays exact in fp32
    return torch.tensor(np.round(rng.standard_normal(shape) * scale) / 256, dtype=torch.float32)


def _loss(q, k, v, dO, cu, B, topk):
    out, _, idx, _ = oracle.forward(q, k, v, cu, B, topk)
    return float((out * dO.double().numpy()).sum()), idx


def test_backward_matches_central_differences():
    rng = np.random.default_rng(401)
    T, Hq, Hkv, d, B, topk = 96, 2, 1, 8, 16, 3
    q, k, v = _dyadic(rng, (T, Hq, d)), _dyadic(rng, (T, Hkv, d)), _dyadic(rng, (T, Hkv, d))
    dO = _dyadic(rng, (T, Hq, d))
    cu = torch.tensor([0, T], dtype=torch.int32)
    _, gap = oracle.gate_topk(q, k, cu, B, topk)
    assert gap.min() > 1e-3  # no block choice sits near a tie
    dq, dk, dv = oracle.backward(q, k, v, dO, cu, B, topk)
    eps = 2.0 ** -12
    checked = 0
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            i = tuple(int(rng.integers(0, n)) for n in x.shape)
            xp, xm = x.clone(), x.clone()
            xp[i] += eps
            xm[i] -= eps
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp, ip = _loss(args["q"], args["k"], args["v"], dO, cu, B, topk)
            args[name] = xm
            lm, im = _loss(args["q"], args["k"], args["v"], dO, cu, B, topk)
            assert (ip == im).all()  # the perturbation did not change any block choice
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - g[i]) <= 1e-6 * max(1.0, abs(fd)), (name, i, fd, g[i])
            checked += 1
    assert checked == 36


def _masked_attention_grads(q, k, v, dO, mask):
    """fp64 autograd of softmax(q k^T / sqrt(d) + mask) v, GQA by repeating k, v."""
    T, Hq, d = q.shape
    grp = Hq // k.shape[1]
    qd = q.double().requires_grad_()
    kd = k.double().requires_grad_()
    vd = v.double().requires_grad_()
    kk = kd.repeat_interleave(grp, dim=1)
    vv = vd.repeat_interleave(grp, dim=1)
    s = torch.einsum("thd,jhd->htj", qd, kk) / d ** 0.5
    s = s.masked_fill(~mask, float("-inf"))
    o = torch.einsum("htj,jhd->thd", torch.softmax(s, dim=-1), vv)
    (o * dO.double()).sum().backward()
    return qd.grad.numpy(), kd.grad.numpy(), vd.grad.numpy()


def test_full_budget_backward_is_dense_causal_backward():
    torch.manual_seed(402)
    T, Hq, Hkv, d, B = 120, 4, 2, 8, 16
    q, k, v, dO = (torch.randn(T, h, d) for h in (Hq, Hkv, Hkv, Hq))
    cu = torch.tensor([0, T], dtype=torch.int32)
    nb = (T + B - 1) // B
    dq, dk, dv = oracle.backward(q, k, v, dO, cu, B, nb)
    mask = torch.ones(T, T, dtype=torch.bool).tril()
    rq, rk, rv = _masked_attention_grads(q, k, v, dO, mask)
    for a, b in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.abs(a - b).max() <= 1e-10 * max(1.0, np.abs(b).max())


def test_topk_one_backward_is_block_diagonal_causal_backward():
    torch.manual_seed(403)
    T, Hq, Hkv, d, B = 100, 2, 1, 8, 16
    q, k, v, dO = (torch.randn(T, h, d) for h in (Hq, Hkv, Hkv, Hq))
    cu = torch.tensor([0, T], dtype=torch.int32)
    dq, dk, dv = oracle.backward(q, k, v, dO, cu, B, 1)
    pos = torch.arange(T)
    mask = (pos[None, :] <= pos[:, None]) & (pos[None, :] // B == pos[:, None] // B)
    rq, rk, rv = _masked_attention_grads(q, k, v, dO, mask)
    for a, b in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.abs(a - b).max() <= 1e-10 * max(1.0, np.abs(b).max())


def test_backward_with_given_indices_and_varlen():
    # sequences are independent: the gradient of a two-sequence batch is the
    # two single-sequence gradients side by side
    torch.manual_seed(404)
    Hq, Hkv, d, B, topk = 2, 2, 8, 16, 2
    q, k, v, dO = (torch.randn(150, h, d) for h in (Hq, Hkv, Hkv, Hq))
    cu = torch.tensor([0, 90, 150], dtype=torch.int32)
    dq, dk, dv = oracle.backward(q, k, v, dO, cu, B, topk)
    for a, b in ((0, 90), (90, 150)):
        sl = slice(a, b)
        c1 = torch.tensor([0, b - a], dtype=torch.int32)
        e = oracle.backward(q[sl], k[sl], v[sl], dO[sl], c1, B, topk)
        for x, y in zip((dq, dk, dv), e):
            assert np.array_equal(x[sl], y)
