"""Plain fp64 CPU oracle for S2O's prefill hot path.

TEST INFRASTRUCTURE ONLY. This module is the checker: only the test suite, the
smoke check and the CPU-baseline leg of the benchmark import it. The product
library never calls it and shares no code with it.

Source: "S2O: Early Stopping for Sparse Attention via Online Permutation"
(arXiv 2602.22575), as described on

  * the pith.science page, "read the original abstract": keys are loaded in
    a non-contiguous, importance-guided order given by an index list, blocks
    are processed from high to low importance and processing stops once the
    current block's score falls below a threshold;
  * the gist.science technical summary (in French), section 1 "Permutation en
    ligne via Chargement Guide par Index" (segment ranking: historical keys
    are scored against a representative query of the segment, under a causal
    mask; the physical K/V layout is kept and an index array drives the
    loads), section 2 "Regle d'Arret Anticipe" (blocks in decreasing estimated
    importance, stop once the block's marginal attention mass falls below
    tau) and section 3 "Implementation du Noyau" (pass 1: dense causal window
    of the segment; pass 2: historical keys in permuted order with the early
    stop).

The pages give no formulas.  Where they leave a step open, this oracle takes
the following readings (the GPU library takes the same ones):

  * representative query: the unweighted mean of the segment's query rows over
    all query heads of the GQA group (query head h uses KV head h // G);
  * score of key j: s_j = qbar . k_j / sqrt(d), natural exponent;
  * admissible keys of segment s: A(s) = [0, e(s)), e(s) = min(N, Lq*(s+1));
  * always kept: sinks [0, n_sink) and the window [max(0, Lq*s - W), e(s));
  * candidates: the rest of A(s), i.e. [n_sink, Lq*s - W) when non-empty;
  * order: candidates by s_j descending, ties to the lower index;
  * blocks: Bk consecutive entries of that order (the last may be partial);
  * block mass: m_b = sum_{j in b} exp(s_j - M) / Z, with M and Z the max and
    the sum of exp(s_j - M) over all of A(s);
  * stop: C = index of the first block with m_b < tau (that block is not
    kept), or the number of blocks if none is below tau;
  * attention: every row i of the segment, for every head of the group, gets
    exact softmax attention over Keep(s) intersected with [0, i];
  * run-time stop (the pages' own rule, an alternative to the planned stop):
    a tile (the segment's rows of a pair of query heads, or of one head when
    the group size is odd) processes the always-kept keys, then candidate
    blocks in the plan's order; after each block every row's gain is the
    block's share of the exp-sum the row has processed so far (the block
    included); the tile stops after the first block whose mean gain over its
    rows is below tau, keeping that block;
  * Q_perm (optional): the segment's rows are ordered by the mean over the
    group's heads of q_i . qbar (the shared guide vector), ties to the lower
    row; the first Lq/2 rows and the rest form two sub-segments, each planned
    with its own pooled query; a row attends over its sub-segment's kept set;
  * MSE against dense attention: the mean over every output element of the
    squared difference between the sparse and the dense causal output;
  * contiguous comparator: original-order blocks of Bk candidates ranked by
    the sum of their pooled-softmax masses, ties to the lower block.

All arithmetic is IEEE fp64 on inputs widened exactly from bf16.  Loops are
plain; numpy's matmul, sort and sum are used as library steps only.  The
oracle is single-threaded when its caller limits BLAS to one thread.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

NEAR_TIE_REL = 1e-6  # relative width of the near-tie bands for scores and masses


@dataclass(frozen=True)
class Params:
    """Method constants.  Defaults are the library's compiled specialisation."""

    Lq: int = 128          # query-segment length
    Bk: int = 64           # stopping granularity (keys per block)
    n_sink: int = 64       # sink tokens [0, n_sink) are always kept
    window_prev: int = 128  # keys before the segment that are always kept
    tau: float = 1e-3      # stopping threshold on block mass


# ---------------------------------------------------------------------------
# bf16 handling (the oracle's own; inputs arrive as raw bf16 bit patterns)
# ---------------------------------------------------------------------------

def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """Exact bf16 -> fp64: a bf16 value is the top half of an fp32 word."""
    if bits.dtype != np.uint16:
        raise TypeError("expected raw bf16 bits as uint16")
    f32 = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return f32.astype(np.float64)


def _f64(x: np.ndarray) -> np.ndarray:
    if x.dtype == np.uint16:
        return widen_bf16(x)
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Segment geometry
# ---------------------------------------------------------------------------

def num_segments(N: int, p: Params) -> int:
    return (N + p.Lq - 1) // p.Lq


def segment_rows(N: int, s: int, p: Params) -> tuple[int, int]:
    return p.Lq * s, min(N, p.Lq * (s + 1))


def admissible_end(N: int, s: int, p: Params) -> int:
    """e(s): keys [0, e(s)) are causally admissible for segment s."""
    return min(N, p.Lq * (s + 1))


def window_start(s: int, p: Params) -> int:
    return max(0, p.Lq * s - p.window_prev)


def candidate_range(N: int, s: int, p: Params) -> tuple[int, int]:
    """[lo, hi) of the candidate keys: A(s) minus sinks and window."""
    lo, hi = p.n_sink, window_start(s, p)
    if hi <= lo:
        return lo, lo
    return lo, hi


def num_candidates(N: int, s: int, p: Params) -> int:
    lo, hi = candidate_range(N, s, p)
    return hi - lo


def candidate_offsets(N: int, p: Params) -> np.ndarray:
    """off[s] = sum of |Cand(t)| for t < s; off[S] = total per (b, kvh)."""
    S = num_segments(N, p)
    off = np.zeros(S + 1, dtype=np.int64)
    for s in range(S):
        off[s + 1] = off[s] + num_candidates(N, s, p)
    return off


def num_blocks(n_cand: int, p: Params) -> int:
    return (n_cand + p.Bk - 1) // p.Bk


def always_kept(N: int, s: int, p: Params) -> np.ndarray:
    """Sinks union window, ascending."""
    e = admissible_end(N, s, p)
    sinks = set(range(0, min(p.n_sink, e)))
    window = set(range(window_start(s, p), e))
    return np.array(sorted(sinks | window), dtype=np.int64)


# ---------------------------------------------------------------------------
# Plan: pooled query, scores, (M, Z), order, block masses, stop
# ---------------------------------------------------------------------------

@dataclass
class SegmentPlan:
    s: int
    qbar: np.ndarray            # [d]
    scores: np.ndarray          # [e(s)] s_j for every admissible key
    M: float
    Z: float
    order: np.ndarray           # candidate indices, importance order
    masses: np.ndarray          # [n_blocks]
    C: int                      # kept candidate blocks
    score_ties: np.ndarray      # positions p with |sigma_p - sigma_{p+1}| <= tol
    mass_ties: np.ndarray       # blocks b with |m_b - tau| <= 1e-6 tau
    tie_tol: float = 0.0
    keep: np.ndarray = field(default=None)  # Keep(s), ascending


def pooled_query(Qf: np.ndarray, b: int, kvh: int, s: int, G: int, p: Params) -> np.ndarray:
    """qbar = mean over the group's G query heads and the segment's rows."""
    N = Qf.shape[2]
    r0, r1 = segment_rows(N, s, p)
    acc = np.zeros(Qf.shape[3], dtype=np.float64)
    count = 0
    for g in range(G):
        h = kvh * G + g
        for i in range(r0, r1):
            acc += _f64(Qf[b, h, i])
            count += 1
    return acc / count


def key_scores(qbar: np.ndarray, Kf: np.ndarray, b: int, kvh: int, e: int) -> np.ndarray:
    """s_j = qbar . k_j / sqrt(d) for j in [0, e)."""
    d = Kf.shape[3]
    K = _f64(Kf[b, kvh, :e])
    return (K @ qbar) / math.sqrt(d)


def plan_segment(Qf, Kf, b: int, kvh: int, s: int, G: int, p: Params) -> SegmentPlan:
    return plan_segment_with_query(pooled_query(Qf, b, kvh, s, G, p), Kf, b, kvh, s, p)


def plan(Qf, Kf, p: Params, segments=None):
    """Plan of every (b, kvh, s), in the library's packed layout.

    Returns dict with
      scores   [B, Hkv, T]  candidate scores, candidate-position order
      perm     [B, Hkv, T]  candidate indices in importance order (absolute)
      nblocks  [B, Hkv, S]  kept candidate blocks C(s)
      seg_stats[B, Hkv, S, 2]  (M, Z)
      plans    {(b, kvh, s): SegmentPlan}
    where T = sum_s |Cand(s)| and segment s occupies [off[s], off[s+1]).
    With `segments` given, only those segments are planned (other entries of
    the packed arrays are left at -1 / nan).
    """
    B, Hq, N, d = Qf.shape
    Hkv = Kf.shape[1]
    G = Hq // Hkv
    S = num_segments(N, p)
    off = candidate_offsets(N, p)
    T = int(off[-1])
    scores = np.full((B, Hkv, T), np.nan)
    perm = np.full((B, Hkv, T), -1, dtype=np.int64)
    nblocks = np.full((B, Hkv, S), -1, dtype=np.int64)
    stats = np.full((B, Hkv, S, 2), np.nan)
    plans = {}
    segs = range(S) if segments is None else segments
    for b in range(B):
        for kvh in range(Hkv):
            for s in segs:
                sp = plan_segment(Qf, Kf, b, kvh, s, G, p)
                lo, hi = candidate_range(N, s, p)
                scores[b, kvh, off[s]:off[s + 1]] = sp.scores[lo:hi]
                perm[b, kvh, off[s]:off[s + 1]] = sp.order
                nblocks[b, kvh, s] = sp.C
                stats[b, kvh, s] = (sp.M, sp.Z)
                plans[(b, kvh, s)] = sp
    return dict(scores=scores, perm=perm, nblocks=nblocks, seg_stats=stats, plans=plans, offsets=off)


def keep_set(N: int, s: int, perm_seg: np.ndarray, C: int, p: Params) -> np.ndarray:
    """Keep(s) = sinks U window U first C*Bk entries of the segment's order."""
    n = len(perm_seg)
    return np.union1d(always_kept(N, s, p), np.asarray(perm_seg[:min(C * p.Bk, n)], dtype=np.int64))


# ---------------------------------------------------------------------------
# Attention over a kept set
# ---------------------------------------------------------------------------

def attention_segment(Qf, Kf, Vf, b: int, kvh: int, s: int, G: int, keep: np.ndarray,
                      p: Params, phys_of_logical: np.ndarray | None = None) -> np.ndarray:
    """Exact softmax attention of the segment's rows over keep intersected with [0, i].

    Returns [G, rows, d].  Keys are addressed through an index list: logical key
    j is read from physical row phys_of_logical[j] (identity when None).  This is
    the "virtual to physical" loading of the pages; the causal mask and the kept
    set use logical positions.
    Softmax is two-pass per row: the maximum first, then the normalised sum.
    """
    N, d = Qf.shape[2], Qf.shape[3]
    r0, r1 = segment_rows(N, s, p)
    keep = np.asarray(keep, dtype=np.int64)
    phys = keep if phys_of_logical is None else np.asarray(phys_of_logical)[keep]
    Kk = _f64(Kf[b, kvh][phys])
    Vk = _f64(Vf[b, kvh][phys])
    out = np.zeros((G, r1 - r0, d))
    rows = np.arange(r0, r1)
    visible = keep[None, :] <= rows[:, None]
    for g in range(G):
        Qs = _f64(Qf[b, kvh * G + g, r0:r1])
        S = (Qs @ Kk.T) / math.sqrt(d)
        S = np.where(visible, S, -np.inf)
        m = S.max(axis=1, keepdims=True)
        P = np.exp(S - m)
        ell = P.sum(axis=1, keepdims=True)
        out[g] = (P @ Vk) / ell
    return out


def dense_segment(Qf, Kf, Vf, b: int, kvh: int, s: int, G: int, p: Params) -> np.ndarray:
    """Causal attention of the segment's rows over every admissible key."""
    N = Qf.shape[2]
    keep = np.arange(0, admissible_end(N, s, p), dtype=np.int64)
    return attention_segment(Qf, Kf, Vf, b, kvh, s, G, keep, p)


def attention(Qf, Kf, Vf, perm, nblocks, p: Params, segments=None, offsets=None):
    """Sparse prefill output O[B, Hq, N, d] (fp64) for the given plan.

    perm / nblocks in the packed layout of `plan`.  Rows of segments not listed
    in `segments` are left at nan.
    """
    B, Hq, N, d = Qf.shape
    Hkv = Kf.shape[1]
    G = Hq // Hkv
    S = num_segments(N, p)
    off = candidate_offsets(N, p) if offsets is None else offsets
    O = np.full((B, Hq, N, d), np.nan)
    segs = range(S) if segments is None else segments
    for b in range(B):
        for kvh in range(Hkv):
            for s in segs:
                keep = keep_set(N, s, perm[b, kvh, off[s]:off[s + 1]], int(nblocks[b, kvh, s]), p)
                r0, r1 = segment_rows(N, s, p)
                O[b, kvh * G:(kvh + 1) * G, r0:r1] = attention_segment(Qf, Kf, Vf, b, kvh, s, G, keep, p)
    return O


def dense_attention(Qf, Kf, Vf, p: Params, segments=None):
    B, Hq, N, d = Qf.shape
    Hkv = Kf.shape[1]
    G = Hq // Hkv
    S = num_segments(N, p)
    O = np.full((B, Hq, N, d), np.nan)
    segs = range(S) if segments is None else segments
    for b in range(B):
        for kvh in range(Hkv):
            for s in segs:
                r0, r1 = segment_rows(N, s, p)
                O[b, kvh * G:(kvh + 1) * G, r0:r1] = dense_segment(Qf, Kf, Vf, b, kvh, s, G, p)
    return O


# ---------------------------------------------------------------------------
# Run-time (online) stop rule
# ---------------------------------------------------------------------------

NEAR_TIE_ONLINE_REL = 1e-4  # relative band around tau for the online block gains


@dataclass
class OnlineStop:
    C: int                  # candidate blocks processed, the stopping block included
    gains: np.ndarray       # mean relative gain of each processed candidate block
    near_ties: np.ndarray   # processed blocks whose gain lies within the band of tau


def online_stop_segment(Qf, Kf, b: int, kvh: int, s: int, heads, perm_seg: np.ndarray, p: Params,
                        phys_of_logical: np.ndarray | None = None) -> OnlineStop:
    """The pages' run-time stop (gist.science technical summary, section 2;
    arxivlens "Methodology": stop on the marginal softmax gain).

    The tile is the segment's rows of the query heads in `heads`.  Pass 1
    takes the always-kept keys (sinks and window; each row sees those <= i).
    Candidate blocks then follow in the order perm_seg, Bk keys each.  After
    block b every row i has the gain g_i(b) = W_i(b) / L_i(b): W_i(b) is the
    sum of exp(q_i . k_j / sqrt(d)) over the block, L_i(b) the same sum over
    everything the row has processed, block b included.  The tile's gain is
    the mean of g_i(b) over its rows (rows past N do not exist).  Processing
    stops after the first block whose tile gain is below tau; that block has
    been computed and stays in the output.  With no such block every
    candidate block is processed.
    """
    N, d = Qf.shape[2], Qf.shape[3]
    r0, r1 = segment_rows(N, s, p)
    rows = np.arange(r0, r1)
    always = always_kept(N, s, p)
    perm_seg = np.asarray(perm_seg, dtype=np.int64)
    nb = num_blocks(len(perm_seg), p)
    phys = (lambda j: j) if phys_of_logical is None else (lambda j: np.asarray(phys_of_logical)[j])
    Ka = _f64(Kf[b, kvh][phys(always)])
    Kc = _f64(Kf[b, kvh][phys(perm_seg)]) if len(perm_seg) else np.zeros((0, d))
    vis = always[None, :] <= rows[:, None]
    # per (head, row): a fixed reference (the row's max over everything it
    # could see) keeps the exponentials in range; the gains do not depend on it
    Sa, Sc = [], []
    for h in heads:
        Qs = _f64(Qf[b, h, r0:r1])
        Sa.append(np.where(vis, (Qs @ Ka.T) / math.sqrt(d), -np.inf))
        Sc.append((Qs @ Kc.T) / math.sqrt(d))
    Sa = np.concatenate(Sa, axis=0)
    Sc = np.concatenate(Sc, axis=0) if len(perm_seg) else np.zeros((Sa.shape[0], 0))
    ref = np.maximum(Sa.max(axis=1), Sc.max(axis=1) if Sc.shape[1] else -np.inf)[:, None]
    L = np.exp(Sa - ref).sum(axis=1)
    gains = []
    C = nb
    for blk in range(nb):
        W = np.exp(Sc[:, blk * p.Bk:(blk + 1) * p.Bk] - ref).sum(axis=1)
        L = L + W
        g = float(np.mean(W / L))
        gains.append(g)
        if g < p.tau:
            C = blk + 1
            break
    gains = np.array(gains, dtype=np.float64)
    ties = np.nonzero(np.abs(gains - p.tau) <= NEAR_TIE_ONLINE_REL * p.tau)[0]
    return OnlineStop(C=C, gains=gains, near_ties=ties)


def tile_heads(kvh: int, G: int, pair: int) -> list:
    """Query heads of one tile of the online rule: the pair 2*pair, 2*pair+1
    of the group when G is even (the heads the library's kernel computes
    together), else the single head `pair`."""
    if G % 2 == 0:
        return [kvh * G + 2 * pair, kvh * G + 2 * pair + 1]
    return [kvh * G + pair]


# ---------------------------------------------------------------------------
# Query permutation with finer sub-segments (Q_perm)
# ---------------------------------------------------------------------------

@dataclass
class SubPlan:
    rows: np.ndarray        # [rows] segment rows in Q_perm order (absolute indices)
    sub_of_row: np.ndarray  # [rows] sub-segment (0 or 1) of each row, in row order
    plans: list             # [SegmentPlan, SegmentPlan] of the two sub-segments
    imp: np.ndarray = field(default=None)  # [rows] importance of each row, in row order


def qperm_segment(Qf, Kf, b: int, kvh: int, s: int, G: int, p: Params) -> SubPlan:
    """Q_perm (gist.science technical summary, section 1, "Classement par
    Segment": queries reordered inside the segment by a coarse importance score
    against a shared guide vector), with finer sub-segments whose kept sets
    differ.  Guide vector: the segment's pooled query qbar.  Row importance:
    the mean over the group's heads of q_{h,i} . qbar.  Rows are ordered by
    importance descending, ties to the lower row; the first Lq/2 rows form
    sub-segment 0, the others sub-segment 1.  Each sub-segment is planned like
    a segment (same admissible keys, candidates and rule) with its own pooled
    query: the mean over its rows and the group's heads.  An empty
    sub-segment 1 (a segment of at most Lq/2 rows) reuses qbar."""
    N = Qf.shape[2]
    r0, r1 = segment_rows(N, s, p)
    rows = np.arange(r0, r1)
    qbar = pooled_query(Qf, b, kvh, s, G, p)
    imp = np.zeros(r1 - r0)
    for g in range(G):
        imp += _f64(Qf[b, kvh * G + g, r0:r1]) @ qbar
    imp /= G
    order = rows[np.lexsort((rows, -imp))]
    n0 = min(p.Lq // 2, r1 - r0)
    groups = [np.sort(order[:n0]), np.sort(order[n0:])]
    sub_of_row = np.zeros(r1 - r0, dtype=np.int64)
    sub_of_row[groups[1] - r0] = 1
    plans = []
    for grp in groups:
        if len(grp) == 0:
            q = qbar
        else:
            acc = np.zeros(Qf.shape[3])
            for g in range(G):
                acc += _f64(Qf[b, kvh * G + g][grp]).sum(axis=0)
            q = acc / (G * len(grp))
        plans.append(plan_segment_with_query(q, Kf, b, kvh, s, p))
    return SubPlan(rows=order, sub_of_row=sub_of_row, plans=plans, imp=imp)


def plan_segment_with_query(qbar: np.ndarray, Kf, b: int, kvh: int, s: int, p: Params) -> SegmentPlan:
    """plan_segment with a given pooled query (scores, order, masses, stop)."""
    N = Kf.shape[2]
    e = admissible_end(N, s, p)
    sc = key_scores(qbar, Kf, b, kvh, e)
    if not np.all(np.isfinite(sc)):
        raise ValueError("non-finite score")
    M = float(np.max(sc))
    Z = float(np.sum(np.exp(sc - M)))
    lo, hi = candidate_range(N, s, p)
    cand = np.arange(lo, hi, dtype=np.int64)
    cs = sc[lo:hi]
    order = cand[np.lexsort((cand, -cs))] if hi > lo else cand
    w = np.exp(sc[order] - M) / Z
    nb = num_blocks(hi - lo, p)
    masses = np.array([w[k * p.Bk:(k + 1) * p.Bk].sum() for k in range(nb)], dtype=np.float64)
    C = nb
    for k in range(nb):
        if masses[k] < p.tau:
            C = k
            break
    tol = NEAR_TIE_REL * float(np.max(np.abs(sc)))
    srt = sc[order]
    score_ties = np.nonzero(np.abs(srt[:-1] - srt[1:]) <= tol)[0] if len(srt) > 1 else np.zeros(0, np.int64)
    mass_ties = np.nonzero(np.abs(masses - p.tau) <= NEAR_TIE_REL * p.tau)[0]
    keep = keep_set(N, s, order, C, p)
    return SegmentPlan(s=s, qbar=qbar, scores=sc, M=M, Z=Z, order=order, masses=masses, C=C,
                       score_ties=score_ties, mass_ties=mass_ties, tie_tol=tol, keep=keep)


def attention_qperm_segment(Qf, Kf, Vf, b: int, kvh: int, s: int, G: int, keeps, sub_of_row: np.ndarray,
                            p: Params) -> np.ndarray:
    """Each row attends over its own sub-segment's kept set (and [0, i])."""
    r0, r1 = segment_rows(Qf.shape[2], s, p)
    out = np.zeros((G, r1 - r0, Qf.shape[3]))
    for sub in (0, 1):
        if not np.any(sub_of_row == sub):
            continue
        full = attention_segment(Qf, Kf, Vf, b, kvh, s, G, keeps[sub], p)
        out[:, sub_of_row == sub] = full[:, sub_of_row == sub]
    return out


# ---------------------------------------------------------------------------
# Ranking accuracy: the pooled order against the true attention mass
# ---------------------------------------------------------------------------

@dataclass
class BlockTruth:
    mass: np.ndarray     # [n_blocks] true mean mass of each block of the order
    always: float        # true mean mass of the always-kept keys
    kept: int            # blocks the plan keeps (C)
    true: int            # blocks whose true mass is >= tau
    both: int            # blocks in both sets
    captured: float      # true mass of the kept blocks
    total: float         # true mass of all candidate blocks


def true_block_masses(Qf, Kf, b: int, kvh: int, s: int, G: int, perm_seg: np.ndarray, C: int,
                      p: Params) -> BlockTruth:
    """Checks the pooled estimate against exact attention (the referee
    reports on the pith.science page note that ranking accuracy is not
    measured).  For every row i of the segment and head of the group, the
    exact causal softmax over all of [0, i] gives each candidate key its
    probability; a block's true mass is the mean over those rows of the
    probabilities of its keys.  The kept set is the plan's first C blocks,
    the true set the blocks whose true mass is at least tau."""
    N, d = Qf.shape[2], Qf.shape[3]
    r0, r1 = segment_rows(N, s, p)
    e = admissible_end(N, s, p)
    rows = np.arange(r0, r1)
    Ka = _f64(Kf[b, kvh, :e])
    perm_seg = np.asarray(perm_seg, dtype=np.int64)
    col = np.zeros(e)
    for g in range(G):
        Qs = _f64(Qf[b, kvh * G + g, r0:r1])
        S = (Qs @ Ka.T) / math.sqrt(d)
        S = np.where(np.arange(e)[None, :] <= rows[:, None], S, -np.inf)
        P = np.exp(S - S.max(axis=1, keepdims=True))
        P = P / P.sum(axis=1, keepdims=True)
        col += P.sum(axis=0)
    col /= G * (r1 - r0)
    nb = num_blocks(len(perm_seg), p)
    mass = np.array([col[perm_seg[k * p.Bk:(k + 1) * p.Bk]].sum() for k in range(nb)], dtype=np.float64)
    always = float(col[always_kept(N, s, p)].sum())
    kept = min(C, nb)
    tset = mass >= p.tau
    return BlockTruth(mass=mass, always=always, kept=kept, true=int(tset.sum()), both=int(tset[:kept].sum()),
                      captured=float(mass[:kept].sum()), total=float(mass.sum()))


# ---------------------------------------------------------------------------
# Contiguous top-k comparator (block-sparse baseline at matched block count)
# ---------------------------------------------------------------------------

def contiguous_plan_segment(sp: SegmentPlan, N: int, C_match: int, p: Params) -> np.ndarray:
    """Kept tokens of the block-granular comparator for one segment.

    The candidates are cut into blocks of Bk keys in their original order; each
    block is ranked by its pooled-softmax mass sum exp(s_j - M) / Z (ties to
    the lower block); the top C_match blocks are kept.  Returns the kept blocks'
    token indices, block by block in rank order, each block ascending, followed
    by the remaining candidate blocks in rank order.
    """
    lo, hi = candidate_range(N, sp.s, p)
    nb = num_blocks(hi - lo, p)
    w = np.exp(sp.scores[lo:hi] - sp.M) / sp.Z
    bm = np.array([w[k * p.Bk:(k + 1) * p.Bk].sum() for k in range(nb)])
    rank = np.lexsort((np.arange(nb), -bm))
    out = [np.arange(lo + k * p.Bk, min(hi, lo + (k + 1) * p.Bk)) for k in rank]
    return np.concatenate(out).astype(np.int64) if out else np.zeros(0, np.int64)


# ---------------------------------------------------------------------------
# Measurement definitions
# ---------------------------------------------------------------------------

def kept_pairs_segment(N: int, s: int, keep: np.ndarray, p: Params) -> int:
    """Number of (row, key) pairs computed for one head: sum_i |Keep(s) cap [0, i]|."""
    r0, r1 = segment_rows(N, s, p)
    keep = np.sort(np.asarray(keep))
    total = 0
    for i in range(r0, r1):
        total += int(np.searchsorted(keep, i, side="right"))
    return total


def mse_segment(Qf, Kf, Vf, b: int, kvh: int, s: int, G: int, keep: np.ndarray, p: Params) -> tuple[float, int]:
    """Squared error of the sparse output against dense causal attention for
    one segment (all heads of the group, all rows, all channels).

    The pages quote a "single-operator MSE" of S2O against full attention
    (pith.science page, "read the original abstract") without defining it;
    the reading taken here is the mean over every output element (b, h, i, c)
    of (O_sparse - O_dense)^2, both exact fp64 evaluations on the same bf16
    inputs.  Returns (sum of squared differences, number of elements) so that
    sums over segments give the mean over any set of segments.
    """
    sparse = attention_segment(Qf, Kf, Vf, b, kvh, s, G, keep, p)
    dense = dense_segment(Qf, Kf, Vf, b, kvh, s, G, p)
    diff = sparse - dense
    return float(np.sum(diff * diff)), int(diff.size)


def mse(Qf, Kf, Vf, perm, nblocks, p: Params, segments=None, offsets=None) -> float:
    """Mean over the listed segments' output elements (every (b, kvh) and
    head) of the squared difference between the plan's sparse output and
    dense causal attention; all segments when `segments` is None."""
    B, Hq, N, d = Qf.shape
    Hkv = Kf.shape[1]
    G = Hq // Hkv
    off = candidate_offsets(N, p) if offsets is None else offsets
    segs = range(num_segments(N, p)) if segments is None else segments
    sse, n = 0.0, 0
    for b in range(B):
        for kvh in range(Hkv):
            for s in segs:
                keep = keep_set(N, s, perm[b, kvh, off[s]:off[s + 1]], int(nblocks[b, kvh, s]), p)
                e, m = mse_segment(Qf, Kf, Vf, b, kvh, s, G, keep, p)
                sse += e
                n += m
    return sse / n if n else 0.0
