"""Comparison helpers: GPU plan / output against the fp64 oracle.

Index lists and block counts must match the oracle exactly, except inside
near-tie sets the oracle reports: runs of the oracle order whose adjacent
scores differ by at most 1e-6 x max|s| (their relative order is not decided
by the inputs at the precision the GPU computes in), and blocks whose mass
lies within 1e-6 x tau of tau.  Every such allowance is counted and logged.
Outputs must be within max-abs 1.5e-2 and relative RMS 4e-3 of the oracle
evaluated on the same bf16 inputs and the same kept set.
"""
from __future__ import annotations

import json
import os

import numpy as np

from oracle import s2o_oracle as O

MAX_ABS = 1.5e-2
REL_RMS = 4e-3


def log_near_ties(record: dict):
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
    # near-tie runs of the oracle order
    run = np.zeros(n, dtype=np.int64)
    if n > 1:
        brk = np.ones(n - 1, dtype=bool)
        brk[sp.score_ties] = False
        run[1:] = np.cumsum(brk)
    if prefix_only:
        span = min(n, p.Bk * gpu_C)
    else:
        span = n if full_list else min(n, p.Bk * max(gpu_C, sp.C) + p.Bk)
    swapped = 0
    if n:
        pos = np.empty(n, dtype=np.int64)
        pos[sp.order - lo] = np.arange(n)
        gpos = pos[gpu_perm[:span] - lo]
        mism = gpu_perm[:span] != sp.order[:span]
        bad = np.nonzero(mism & (run[gpos] != run[:span]))[0]
        assert bad.size == 0, f"position {bad[:5]}: keys outside the oracle's near-tie runs"
        swapped = int(mism.sum())
    flip = 0
    if gpu_C != sp.C:
        lo_b, hi_b = min(gpu_C, sp.C), max(gpu_C, sp.C)
        ties = set(int(x) for x in sp.mass_ties)
        assert all(b in ties for b in range(lo_b, hi_b)), \
            f"C(s) {gpu_C} != oracle {sp.C} and the blocks between are not mass near-ties"
        flip = hi_b - lo_b
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
