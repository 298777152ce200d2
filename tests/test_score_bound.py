"""The score tolerance of the GPU parity tests, checked on the CPU.

The library scores keys in fixed point (its header and the scorer's source
describe the scheme): each key row as a 22-bit integer against the row's
largest binary exponent, split into three signed 8-bit digits; each pooled
query as a 29-bit integer against its own exponent, in four digits; the digit
products of weight 2^8 and up summed exactly, one of weight 1 left out; the
result rounded once in fp64 and once to fp32.  `parity.score_error_bound`
states how far that can be from the exact score beyond half an fp32 ulp.
Here a numpy model of the scheme (written from that description, not from
the kernels) is run on inputs spanning many binades, and every score is
checked against the exact fp64 dot product within half an ulp plus the
bound.  The inputs make two of the bound's terms bind: keys spanning 80
binades (the key-rounding term) and keys nearly orthogonal to the query,
whose scores cancel (the query-rounding term); without either term these
checks fail (thousands of scores).  The third term, the omitted digit
product, lies below both here.
"""
import math

import numpy as np
import pytest

from oracle import s2o_oracle as O
from score_keys_pooled_b200 import synth
from tests import parity


def _signed_digits(x, n):
    """x = sum_k d_k 256^(n-1-k), d_k in [-128, 127] (top digit unbounded)."""
    out = []
    for _ in range(n - 1):
        lo = ((x & 0xFF) ^ 0x80) - 0x80
        out.append(lo)
        x = (x - lo) >> 8
    out.append(x)
    return out[::-1]


def _model_scores(qbar, kbits):
    """fp32 scores of one pooled query against key rows [n, 128] (bf16 bits)."""
    kb = kbits.astype(np.int64)
    ex = (kb >> 7) & 0xFF
    mant = np.where(ex == 0, kb & 0x7F, (kb & 0x7F) | 0x80)
    exf = np.maximum(ex, 1)
    E = np.maximum(1, (kb & 0x7FFF).max(axis=1) >> 7)
    sh = exf - E[:, None] + 14
    r = np.minimum(-sh, 9)
    F = np.where(sh >= 0, mant << np.maximum(sh, 0),
                 (mant + (1 << np.maximum(r - 1, 0))) >> np.maximum(r, 1))
    F = np.where(kb & 0x8000, -F, F)
    mx = np.abs(qbar).max()
    f = (np.frexp(mx)[1] - 1) if mx > 0 else 0
    G = np.rint(qbar * 2.0 ** (28 - f)).astype(np.int64)
    qd = _signed_digits(G, 4)
    kd = _signed_digits(F, 3)
    assert np.abs(kd[0]).max() <= 64 and np.abs(qd[0]).max() <= 33
    assert all(np.abs(x).max() <= 128 for x in kd[1:] + qd[1:])
    S = [sum(kd[b] @ qd[t - b] for b in range(3) if 0 <= t - b <= 3) for t in range(5)]
    Y = (S[0] * 256 + S[1]) * 2 ** 24 + (S[2] * 256 + S[3]) * 256 + S[4]
    assert np.abs(Y).max() < 2 ** 51
    s64 = Y.astype(np.float64) * np.ldexp(math.sqrt(2.0), (f + E - 172).astype(np.int64))
    return s64.astype(np.float32).astype(np.float64)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_half_ulp_plus_bound_covers_the_fixed_point_scores(seed):
    rng = np.random.default_rng(seed)
    n = 512
    K = rng.standard_normal((n, 128)) * np.exp2(rng.integers(-40, 41, size=(n, 128)))
    K[:4] = 0.0
    K[4, :] = 0.0
    K[4, 7] = 3.0
    K[5] = rng.standard_normal(128) * 2.0 ** -130  # subnormal bf16
    kbits = synth.to_bf16_bits(K.astype(np.float32))
    Kf = O.widen_bf16(kbits)
    for scale in (2.0 ** -100, 1.0, 2.0 ** 40):
        qbar = rng.standard_normal(128) * scale
        qbar[rng.random(128) < 0.1] *= 2.0 ** -30
        exact = Kf @ qbar / math.sqrt(128)
        got = _model_scores(qbar, kbits)
        half_ulp = 0.5 * np.spacing(np.abs(exact).astype(np.float32)).astype(np.float64)
        bound = parity.score_error_bound(qbar, Kf)
        assert np.all(np.abs(got - exact) <= half_ulp + bound), np.max(np.abs(got - exact) - half_ulp - bound)


@pytest.mark.parametrize("seed", [3, 4])
def test_bound_covers_cancelling_scores(seed):
    rng = np.random.default_rng(seed)
    for _ in range(6):
        qbar = rng.standard_normal(128)
        qbar[rng.random(128) < 0.2] *= 2.0 ** -20  # bits below the query's 29-bit fixed point
        V = rng.standard_normal((256, 128))
        V -= np.outer(V @ qbar / (qbar @ qbar), qbar)  # nearly orthogonal once rounded to bf16
        kbits = synth.to_bf16_bits(V.astype(np.float32))
        Kf = O.widen_bf16(kbits)
        exact = Kf @ qbar / math.sqrt(128)
        got = _model_scores(qbar, kbits)
        half_ulp = 0.5 * np.spacing(np.abs(exact).astype(np.float32)).astype(np.float64)
        assert np.all(np.abs(got - exact) <= half_ulp + parity.score_error_bound(qbar, Kf))


def test_the_bound_is_needed():
    """Without the bound, half an ulp alone fails on ordinary inputs: the
    fixed point is not exact, so the tolerance is not vacuous slack."""
    rng = np.random.default_rng(7)
    K = rng.standard_normal((256, 128)).astype(np.float32)
    kbits = synth.to_bf16_bits(K)
    Kf = O.widen_bf16(kbits)
    qbar = rng.standard_normal(128) * 0.3
    exact = Kf @ qbar / math.sqrt(128)
    got = _model_scores(qbar, kbits)
    half_ulp = 0.5 * np.spacing(np.abs(exact).astype(np.float32)).astype(np.float64)
    assert np.any(np.abs(got - exact) > half_ulp + 1e-13 * np.abs(exact))


def test_digit_ranges_keep_accumulators_exact():
    """The scheme's integer ranges: key digits |d0| <= 64, |d1|, |d2| <= 128;
    query digits |c0| <= 33, |c1..c3| <= 128; so every S_t (a sum of at most
    three 128-term digit products) fits int32, hi = 256 S0 + S1 and
    mid = 256 S2 + S3 fit int32, and |Y| < 2^51 (Y converts to fp64
    exactly).  Checked from the ranges and on extreme inputs."""
    dmax = [64, 128, 128]
    cmax = [33, 128, 128, 128]
    S = [sum(128 * cmax[t - b] * dmax[b] for b in range(3) if 0 <= t - b <= 3) for t in range(5)]
    hi, mid = 256 * S[0] + S[1], 256 * S[2] + S[3]
    Y = hi * 2 ** 24 + mid * 256 + S[4]
    assert max(S) < 2 ** 31 and hi < 2 ** 31 and mid < 2 ** 31
    assert Y < 2 ** 51
    # extreme rows: every element at the row maximum (largest top digits) or
    # alternating signs, with the query at the top of its range
    rng = np.random.default_rng(5)
    for sign in (1.0, -1.0):
        K = np.full((8, 128), 3.0e38 * sign, dtype=np.float32)
        K[1::2, ::2] *= -1
        K[4:] = rng.choice([-1.0, 1.0], size=(4, 128)) * np.float32(1.9921875)  # mantissa all ones
        kbits = synth.to_bf16_bits(K)
        qbar = np.full(128, 1.999999) * sign
        qbar[::3] *= -1
        with np.errstate(over="ignore"):  # rows of 3e38 overflow fp32 (the kernel flags those)
            got = _model_scores(qbar, kbits)  # asserts inside check the digit ranges
            exact = O.widen_bf16(kbits) @ qbar / math.sqrt(128)
            fin = np.isfinite(exact.astype(np.float32))
            half_ulp = 0.5 * np.spacing(np.abs(exact).astype(np.float32)).astype(np.float64)
        bound = parity.score_error_bound(qbar, O.widen_bf16(kbits))
        assert np.all(np.abs(got[fin] - exact[fin]) <= half_ulp[fin] + bound[fin])
