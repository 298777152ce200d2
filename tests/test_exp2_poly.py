"""The FMA-pipe exp2 of the attention softmax (sparse_attn2.cuh, exp2_poly_x2).

The coefficients in the kernel must be the fp32 roundings of the Remez
minimax fit that exp2_poly.py computes, and the kernel's fp32 evaluation
(emulated here step by step: rounding trick, fused Horner steps, exponent
add) must stay within 3e-6 relative error of 2^x over the arguments the
softmax produces, down to the clamp at -125.
"""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "score_keys_pooled_b200", "csrc")
sys.path.insert(0, CSRC)
import exp2_poly  # noqa: E402


def _kernel_coefficients():
    text = open(os.path.join(CSRC, "sparse_attn2.cuh")).read()
    found = dict(re.findall(r"constexpr float kExp2C(\d) = ([0-9.eE+-]+)f;", text))
    return np.array([float(found[str(j)]) for j in range(exp2_poly.DEGREE + 1)], dtype=np.float32)


def test_kernel_coefficients_are_the_remez_fit():
    c, err = exp2_poly.remez()
    assert 1e-7 < err < 3e-6
    assert np.array_equal(_kernel_coefficients(), c.astype(np.float32))
    # sanity of the fit: 2^f = 1 + f ln2 + ... near 0
    assert abs(c[0] - 1) < 1e-5 and abs(c[1] - np.log(2)) < 1e-4


def test_fp32_evaluation_error_bound():
    c32 = _kernel_coefficients()
    x = np.concatenate([np.linspace(-125.0, 8.0, 3_000_001), np.linspace(-1.0, 1.0, 1_000_001),
                        np.arange(-125, 9, dtype=np.float64)]).astype(np.float32)
    got = exp2_poly.emulate(x, c32).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 3e-6, (rel.max(), x[np.argmax(rel)])


def test_clamp_keeps_very_small_arguments_tiny_and_positive():
    c32 = _kernel_coefficients()
    got = exp2_poly.emulate(np.array([-126.0, -300.0, -1e30], dtype=np.float32), c32)
    assert np.all(got > 0) and np.all(got < 2.0 ** -124)
