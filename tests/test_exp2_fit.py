"""The FMA-pipe exp2 of the sparse attention kernel (exp2_poly2 in attn_tc.cuh).

CPU only. The constants in the kernel are the float32 coefficients that
linear_global_attention_b200/exp2_fit.py fits (degree-3 polynomial for 2^f on
[-1/2, 1/2], minimax in relative error), and the kernel's float32 evaluation
(clamp, round-to-nearest split, Horner with fused multiply-adds, exponent add)
stays within 1.5e-4 relative error of 2^x over its whole input range, about
13x below the bf16 rounding (2^-9) that every exponential gets next.
"""
import os
import re

import numpy as np

from linear_global_attention_b200 import exp2_fit as ef

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUH = os.path.join(ROOT, "linear_global_attention_b200", "csrc", "attn_tc.cuh")


def _kernel_coeffs():
    txt = open(CUH).read()
    vals = {}
    for i in range(4):
        m = re.search(rf"EXP2_C{i} = ([0-9.eE+-]+)f", txt)
        assert m, f"EXP2_C{i} not found"
        vals[i] = np.float32(float(m.group(1)))
    return np.array([vals[i] for i in range(4)], np.float32)


def test_kernel_constants_are_the_fit():
    c, bound = ef.fit()
    assert bound < 8e-5
    np.testing.assert_array_equal(_kernel_coeffs(), c)


def test_float32_evaluation_error_bound():
    c = _kernel_coeffs()
    x = np.concatenate([np.linspace(-126.0, 8.0, 4_000_001, dtype=np.float32),
                        np.float32([-126.0, -125.5, -0.5, 0.5, 0.0, 8.0, -1e-8, 7.5])])
    got = ef.exp2_emulated(x, c).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 1.5e-4
    inner = x > -100
    assert rel[inner].max() <= 8e-5


def test_masked_logits_underflow_to_nothing():
    # masked columns carry -inf (and the clamp takes anything below -126 there)
    got = ef.exp2_emulated(np.float32([-np.inf, -1e30, -200.0]), _kernel_coeffs())
    assert (got >= 0).all() and (got < 2e-38).all()
