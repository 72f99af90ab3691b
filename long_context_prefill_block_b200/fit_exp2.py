"""Derivation of the exp2 polynomial used by the attention kernels' softmax.

    python -m long_context_prefill_block_b200.fit_exp2

A share of the softmax exponentials is computed without the exponential
unit: x = j + f with j = round(x) (Cody-Waite range reduction, exact in fp32
for |x| < 2^22) and |f| <= 1/2, 2^x = 2^j * p(f), 2^j applied by adding j to
the exponent field. p is the degree-3 polynomial minimising the maximum
relative error |p(f) / 2^f - 1| on [-1/2, 1/2], found here by Lawson's
iteratively reweighted least squares on Chebyshev nodes (a standard route to
the minimax solution), then rounded to fp32. The kernel's constants are the
printed ones; tests/test_exp2_poly.py re-evaluates them in fp32 arithmetic.
"""
import numpy as np

DEGREE = 3


def fit(degree: int = DEGREE, nodes: int = 4001, iters: int = 400):
    f = 0.5 * np.cos(np.pi * (np.arange(nodes) + 0.5) / nodes)  # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / y[:, None]  # relative-error design matrix
    w = np.full(nodes, 1.0 / nodes)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * sw[:, None], np.ones(nodes) * sw, rcond=None)
        err = np.abs(V @ c - 1.0)
        w = w * err
        w /= w.sum()
    return c


def max_rel_error(c32, n: int = 200001) -> float:
    """Max relative error of p on [-1/2, 1/2], p evaluated by Horner in fp32."""
    f = np.linspace(-0.5, 0.5, n).astype(np.float32)
    p = np.full_like(f, c32[-1])
    for ck in c32[-2::-1]:
        p = (p.astype(np.float64) * f + ck).astype(np.float32)  # one rounding per fused step
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = fit()
    c32 = c.astype(np.float32)
    for k, ck in enumerate(c32):
        print(f"c{k} = {float(ck):.9g}f")
    print(f"max relative error (fp32 Horner) = {max_rel_error(c32):.3e}")
