"""Comparison helpers: GPU plan / output against the fp64 oracle.

Index lists and block counts must match the oracle exactly, except where the
inputs do not decide the answer at the precision the GPU computes in:

  * a position p of the order may hold a different key than the oracle's
    only if the two keys' oracle (fp64) scores differ by at most
    1e-6 x max|s| over the segment's admissible keys (a score near-tie);
  * C(s) may differ from the oracle's only if every block between the two
    stop points has a mass within 1e-6 x tau of tau (a mass near-tie).

Every allowance used is counted.  The totals are printed in pytest's
terminal summary (see tests/conftest.py) and, when S2O_NEAR_TIE_LOG names a
file, appended to it per case.  Outputs must be within max-abs 1.5e-2 and
relative RMS 4e-3 of the oracle evaluated on the same bf16 inputs and the
same kept set.
"""
from __future__ import annotations

import json
import os

import numpy as np

from oracle import s2o_oracle as O

MAX_ABS = 1.5e-2
REL_RMS = 4e-3


def score_error_bound(qbar: np.ndarray, Kf: np.ndarray) -> np.ndarray:
    """Bound on |GPU score - exact score| beyond fp32 rounding, per key row.

    The GPU scores in fixed point (the integer tensor-core scorer): qbar is
    rounded to a multiple of 2^(f-28), f = floor(log2 max|qbar|); each key
    element to a multiple of 2^(E-148), E = max(1, biased bf16 exponent of
    the row's largest magnitude), which changes only elements below
    2^(E-141); one digit product of weight 2^(f+E-176) is left out.  The
    three terms are
        [2^(f-29) ||k||_1 + 2^(E-149) sum_{d: |k_d| < 2^(E-141)} |qbar_d|
         + 2^(f+E-156)] / sqrt(d).
    Kf: [n, d] fp64 key rows (bf16 values).  The 1e-6 x max|s| near-tie band
    of the order is three orders above this for bf16 data of any scale.
    """
    Kf = np.asarray(Kf, dtype=np.float64)
    mq = float(np.max(np.abs(qbar))) if qbar.size else 0.0
    f = (np.frexp(mq)[1] - 1) if mq > 0 else 0
    mk = np.max(np.abs(Kf), axis=1)
    E = np.where(mk >= 2.0 ** -126, np.frexp(np.maximum(mk, 2.0 ** -126))[1] + 126, 1)
    d = Kf.shape[1]
    small = np.abs(Kf) < np.ldexp(1.0, E - 141)[:, None]
    b = (np.ldexp(1.0, f - 29) * np.abs(Kf).sum(axis=1) + np.ldexp(1.0, E - 149) * (small @ np.abs(qbar))
         + np.ldexp(1.0, f + E - 156))
    return b / np.sqrt(d)

# allowances used in this process: segments compared, positions holding a
# different (near-tied) key, and blocks between differing stop points
TOTALS = {"segments": 0, "swapped_positions": 0, "C_flips": 0, "online_C_flips": 0, "cases": 0}


def log_near_ties(record: dict):
    TOTALS["cases"] += 1
    TOTALS["online_C_flips"] += int(record.get("C_flips", 0)) if record.get("online") else 0
    path = os.environ.get("S2O_NEAR_TIE_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(record) + "\n")


def compare_segment_plan(gpu_perm: np.ndarray, gpu_C: int, sp: O.SegmentPlan, p: O.Params, full_list=True,
                         prefix_only=False):
    """Returns (swapped_positions, C_flip); raises AssertionError on a real mismatch.

    prefix_only: only the first Bk * gpu_C entries are defined (the filtered
    plan); they must be distinct members of Cand(s) and match the oracle's.
    """
    n = len(sp.order)
    gpu_perm = np.asarray(gpu_perm, dtype=np.int64)
    assert len(gpu_perm) == n
    if n:
        lo = int(sp.order.min())
        if prefix_only:
            head = gpu_perm[:min(n, p.Bk * gpu_C)]
            assert np.all((head >= lo) & (head < lo + n)), "perm prefix leaves Cand(s)"
            assert len(np.unique(head)) == len(head), "perm prefix repeats a key"
        else:
            assert np.array_equal(np.sort(gpu_perm), np.arange(lo, lo + n)), "perm is not a permutation of Cand(s)"
    if prefix_only:
        span = min(n, p.Bk * gpu_C)
    else:
        span = n if full_list else min(n, p.Bk * max(gpu_C, sp.C) + p.Bk)
    swapped = 0
    if span:
        mism = np.nonzero(gpu_perm[:span] != sp.order[:span])[0]
        if mism.size:
            # the scores of the two keys at each differing position, both fp64 oracle values
            s_gpu = sp.scores[gpu_perm[mism]]
            s_ora = sp.scores[sp.order[mism]]
            gap = np.abs(s_gpu - s_ora)
            bad = mism[gap > sp.tie_tol]
            assert bad.size == 0, (f"positions {bad[:5]}: keys {gpu_perm[bad[:5]]} for {sp.order[bad[:5]]}, "
                                   f"score gaps {gap[gap > sp.tie_tol][:5]} > {sp.tie_tol:.3g}")
        swapped = int(mism.size)
    flip = 0
    if gpu_C != sp.C:
        lo_b, hi_b = min(gpu_C, sp.C), max(gpu_C, sp.C)
        ties = set(int(x) for x in sp.mass_ties)
        assert all(b in ties for b in range(lo_b, hi_b)), \
            f"C(s) {gpu_C} != oracle {sp.C} and the blocks between are not mass near-ties"
        flip = hi_b - lo_b
    TOTALS["segments"] += 1
    TOTALS["swapped_positions"] += swapped
    TOTALS["C_flips"] += flip
    return swapped, flip


def output_errors(gpu: np.ndarray, ref: np.ndarray):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = gpu - ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    denom = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 1.0
    rel_rms = float(np.sqrt(np.mean(diff ** 2)) / denom) if diff.size else 0.0
    return max_abs, rel_rms


def assert_output_close(gpu, ref, what=""):
    max_abs, rel_rms = output_errors(gpu, ref)
    assert max_abs <= MAX_ABS and rel_rms <= REL_RMS, f"{what}: max_abs {max_abs:.3g}, rel_rms {rel_rms:.3g}"
    return max_abs, rel_rms
