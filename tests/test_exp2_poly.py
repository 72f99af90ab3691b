"""The attention kernels' polynomial exp2 (csrc/tc_ptx.cuh, ex2_poly2),
checked on the host (CPU): its constants are the ones fit_exp2.py derives
(minimax relative error of a degree-3 polynomial for 2^f on [-1/2, 1/2]),
and the whole evaluation -- the clamp at -125, the Cody-Waite reduction by
adding and subtracting 1.5 * 2^23, Horner's rule with one rounding per fused
multiply-add, and the exponent-field add -- emulated step by step in fp32
stays within 1e-4 relative of 2^x (float64) over the softmax's input range
[-125, 8], and is 2^-125 below it."""
import os
import re

import numpy as np

from long_context_prefill_block_b200 import fit_exp2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "long_context_prefill_block_b200", "csrc", "tc_ptx.cuh")


def kernel_constants():
    text = open(SRC).read()
    body = text[text.index("uint64_t ex2_poly2("):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"f2\(([0-9.e+-]+)f, \1f\)", body)]
    # 1.5 * 2^23, then c3, c2, c1, c0 in Horner order
    return vals[0], vals[1:]


def emulate(x):
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    rnd, (c3, c2, c1, c0) = kernel_constants()
    t = (x + np.float32(rnd)).astype(np.float32)
    j = (t - np.float32(rnd)).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = np.full_like(f, np.float32(c3))
    for ck in (c2, c1, c0):
        p = (p.astype(np.float64) * f + np.float64(np.float32(ck))).astype(np.float32)
    return p.astype(np.float64) * np.exp2(j.astype(np.float64))


def test_constants_are_the_fitted_ones():
    rnd, coefs = kernel_constants()
    assert rnd == 12582912.0
    fitted = fit_exp2.fit().astype(np.float32)[::-1]  # c3 .. c0
    assert np.allclose(np.asarray(coefs, dtype=np.float32), fitted, rtol=0, atol=2e-7)


def test_relative_error_over_the_softmax_range():
    rng = np.random.default_rng(3)
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), rng.uniform(-30.0, 8.0, 200000),
                        np.arange(-125, 9, dtype=np.float64) + 0.5,  # rounding ties
                        np.arange(-125, 9, dtype=np.float64)]).astype(np.float32)
    got = emulate(x)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / ref - 1.0)) < 1e-4


def test_masked_scores_weigh_almost_nothing():
    got = emulate(np.array([-np.inf, -1e30, -126.0, -125.0], dtype=np.float32))
    assert np.all(got > 0) and np.all(got <= 2.0 ** -124.5)
