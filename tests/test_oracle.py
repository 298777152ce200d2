"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test checks one part of the method (pooling, scores, order, masses, stop,
attention) against a closed form, an invariant, a library routine or a
brute-force evaluation on a tiny input.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import s2o_oracle as O
from score_keys_pooled_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
E = math.e


def _ev(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"e": E}))


def _bits(x):
    return synth.to_bf16_bits(np.asarray(x, dtype=np.float32))


# ---------------------------------------------------------------------------
# bf16 widening
# ---------------------------------------------------------------------------

def test_widen_bf16_known_patterns():
    bits = np.array([0x3F80, 0xC000, 0x0001, 0x7F7F, 0x0000, 0x8000, 0x3EAB], dtype=np.uint16)
    got = O.widen_bf16(bits)
    want = [1.0, -2.0, 2.0 ** -133, (2 - 2 ** -7) * 2.0 ** 127, 0.0, -0.0, 0.333984375]
    assert list(got) == want


# ---------------------------------------------------------------------------
# geometry
# ---------------------------------------------------------------------------

def test_candidate_offsets_closed_form_default_params():
    # with Lq=128, W=128, n_sink=64 and N a multiple of 128:
    # |Cand(s)| = max(0, 128 s - 192) and off(s) = 64 (s-2)^2 for s >= 2
    p = O.Params()
    N = 128 * 40
    off = O.candidate_offsets(N, p)
    for s in range(41):
        want = 64 * (s - 2) ** 2 if s >= 2 else 0
        assert off[s] == want
    for s in range(40):
        assert O.num_candidates(N, s, p) == max(0, 128 * s - 192)


def test_sets_partition_admissible_keys():
    p = O.Params(Lq=4, Bk=2, n_sink=1, window_prev=4)
    for N in (1, 3, 8, 13, 16):
        for s in range(O.num_segments(N, p)):
            e = O.admissible_end(N, s, p)
            lo, hi = O.candidate_range(N, s, p)
            kept = set(O.always_kept(N, s, p).tolist())
            cand = set(range(lo, hi))
            assert kept.isdisjoint(cand)
            assert kept | cand == set(range(e))


# ---------------------------------------------------------------------------
# pooling and scores
# ---------------------------------------------------------------------------

def test_pooled_query_closed_form_and_group_mapping():
    # head g of group 1 has row i = (g+1) * ((i - r0) mod 16) in dim 0 (bf16-exact);
    # the mean over G=4 heads and 128 rows is (1+2+3+4) * 8 * (0+...+15) / 512
    p = O.Params()
    B, Hkv, G, N, d = 1, 2, 4, 256, 8
    Q = np.zeros((B, Hkv * G, N, d), dtype=np.float32)
    Q[:, 0:4] = 1000.0  # group 0 must not leak into group 1
    for g in range(G):
        for i in range(128, 256):
            Q[0, 4 + g, i, 0] = (g + 1) * ((i - 128) % 16)
            Q[0, 4 + g, i, 3] = -1.0
    qb = O.pooled_query(_bits(Q), 0, 1, 1, G, p)
    want0 = (1 + 2 + 3 + 4) * 8 * 120 / 512
    assert qb[0] == want0
    assert qb[3] == -1.0
    assert np.all(qb[[1, 2, 4, 5, 6, 7]] == 0.0)


def test_scores_one_hot_keys_are_exact():
    p = O.Params(Lq=4, Bk=2, n_sink=1, window_prev=0)
    d = 16
    N = 8
    a = np.array([0, 1, -3, 2, 0.5, 7, -1, 4], dtype=np.float32)
    K = np.zeros((1, 1, N, d), dtype=np.float32)
    K[0, 0, :, 5] = a
    Q = np.zeros((1, 1, N, d), dtype=np.float32)
    Q[0, 0, 4:8, 5] = 3.0
    sp = O.plan_segment(_bits(Q), _bits(K), 0, 0, 1, 1, p)
    assert np.array_equal(sp.scores, 3.0 * a.astype(np.float64) / 4.0)


# ---------------------------------------------------------------------------
# hand-worked two-segment examples (tests/golden/hand_two_segment.json)
# ---------------------------------------------------------------------------

def _golden_case(case):
    sh = case["shape"]
    Q = np.zeros((sh["B"], sh["Hq"], sh["N"], sh["d"]), dtype=np.float32)
    if "Q_rows_dim0" in case:
        for i, v in case["Q_rows_dim0"].items():
            Q[0, :, int(i), 0] = v
    for h, rows in case.get("Q_rows_dim0_by_head", {}).items():
        for i, v in rows.items():
            Q[0, int(h), int(i), 0] = v
    K = np.zeros((sh["B"], sh["Hkv"], sh["N"], sh["d"]), dtype=np.float32)
    K[0, 0, :, 0] = case["K_dim0"]
    V = np.zeros_like(K)
    V[0, 0, :, 0] = case["V_dim0"]
    V[0, 0, :, 1] = case["V_dim1_all"]
    return _bits(Q), _bits(K), _bits(V)


def _load_golden():
    with open(os.path.join(GOLDEN, "hand_two_segment.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("ci", [0, 1])
def test_hand_worked_plans(ci):
    g = _load_golden()
    case = g["cases"][ci]
    Q, K, V = _golden_case(case)
    for stop in case["stops"]:
        p = O.Params(tau=stop["tau"], **case["params"])
        res = O.plan(Q, K, p)
        for seg in case["segments"]:
            sp = res["plans"][(0, 0, seg["s"])]
            assert sp.order.tolist() == seg["order"]
            assert sp.M == pytest.approx(_ev(seg["M"]), rel=0, abs=1e-14)
            assert sp.Z == pytest.approx(_ev(seg["Z"]), rel=1e-14)
            want_m = [_ev(x) for x in seg["masses"]]
            assert np.allclose(sp.masses, want_m, rtol=1e-13, atol=0)
        assert res["nblocks"][0, 0].tolist() == stop["C"]


def test_hand_worked_outputs():
    g = _load_golden()
    case = g["cases"][0]
    Q, K, V = _golden_case(case)
    p = O.Params(tau=0.2, **case["params"])
    res = O.plan(Q, K, p)
    out = O.attention(Q, K, V, res["perm"], res["nblocks"], p)
    for i, (x0, x1) in case["outputs_tau_0.2"]["rows"].items():
        row = out[0, 0, int(i)]
        assert row[0] == pytest.approx(_ev(x0), rel=1e-14, abs=1e-15)
        assert row[1] == pytest.approx(_ev(x1), rel=1e-14)
        assert np.all(row[2:] == 0)


def test_hand_worked_contiguous_comparator():
    g = _load_golden()
    spec = g["contiguous"]
    case = [c for c in g["cases"] if c["name"] == spec["case"]][0]
    Q, K, V = _golden_case(case)
    p = O.Params(tau=0.2, **case["params"])
    sp = O.plan_segment(Q, K, 0, 0, spec["s"], 1, p)
    full = O.contiguous_plan_segment(sp, case["shape"]["N"], spec["C_match"], p)
    assert full.tolist() == spec["expected_full"]
    assert full[:spec["C_match"] * p.Bk].tolist() == spec["expected_prefix"]


def _contig_case(spec, a):
    sh = spec["shape"]
    N, d = sh["N"], sh["d"]
    Q = np.zeros((1, 1, N, d), dtype=np.float32)
    Q[0, 0, 8:12, 0] = 2.0
    K = np.zeros((1, 1, N, d), dtype=np.float32)
    K[0, 0, 1:8, 0] = a
    return _bits(Q), _bits(K)


@pytest.mark.parametrize("ci", [0, 1])
def test_contiguous_comparator_hand_cases(ci):
    # tests/golden/hand_contiguous.json: the highest-mass block is not the one
    # with the highest score, nor the one with the highest sum of raw scores
    # or of mean mass per key; and an exact mass tie goes to the lower block
    with open(os.path.join(GOLDEN, "hand_contiguous.json")) as f:
        spec = json.load(f)
    case = spec["cases"][ci]
    Q, K = _contig_case(spec, case["a_candidates"])
    p = O.Params(tau=0.0, **spec["params"])
    sp = O.plan_segment(Q, K, 0, 0, 2, 1, p)
    assert np.array_equal(sp.scores[1:8], np.asarray(case["a_candidates"], dtype=np.float64))
    full = O.contiguous_plan_segment(sp, spec["shape"]["N"], case["C_match"], p)
    assert full.tolist() == case["expected_full"]
    assert full[:case["C_match"] * p.Bk].tolist() == case["expected_prefix"]


# ---------------------------------------------------------------------------
# MSE against dense attention
# ---------------------------------------------------------------------------

def test_mse_hand_worked_closed_form():
    with open(os.path.join(GOLDEN, "hand_mse.json")) as f:
        spec = json.load(f)
    g = _load_golden()
    case = [c for c in g["cases"] if c["name"] == spec["case"]][0]
    Q, K, V = _golden_case(case)
    p = O.Params(tau=spec["tau"], **case["params"])
    res = O.plan(Q, K, p)
    got = O.mse(Q, K, V, res["perm"], res["nblocks"], p)
    want = sum((_ev(sx) - _ev(dx)) ** 2 for sx, dx in spec["rows"].values()) / spec["elements"]
    assert want > 1e-4
    assert got == pytest.approx(want, rel=1e-12, abs=0)
    # segment 0 has nothing to drop
    sse0, n0 = O.mse_segment(Q, K, V, 0, 0, 0, 1, res["plans"][(0, 0, 0)].keep, p)
    assert sse0 == 0.0 and n0 == 16


def test_mse_is_zero_at_tau_zero():
    # tau = 0 keeps every admissible key, so the sparse output is the dense one
    Q, K, V = _random_case(7, Hq=2, Hkv=1, N=640, d=32)
    for tau, zero in ((0.0, True), (5e-2, False)):
        p = O.Params(tau=tau)
        res = O.plan(Q, K, p)
        m = O.mse(Q, K, V, res["perm"], res["nblocks"], p)
        assert (m == 0.0) == zero


# ---------------------------------------------------------------------------
# all-ties closed form: Q = 0 makes every score exactly 0
# ---------------------------------------------------------------------------

# tau = 0.0625 = 64/1024 hits the mass of the e(s)=1024 segment exactly (a power
# of two, so the fp64 sum is exact): a block whose mass equals tau is kept.
@pytest.mark.parametrize("tau", [0.0, 1e-3, 0.05, 0.0625, 0.07, 2.0])
def test_all_ties_closed_form(tau):
    p = O.Params(tau=tau)
    B, Hq, Hkv, N, d = 1, 2, 1, 1024, 128
    rng = np.random.default_rng(5)
    Q = np.zeros((B, Hq, N, d), dtype=np.uint16)
    K = _bits(rng.standard_normal((B, Hkv, N, d)))
    res = O.plan(Q, K, p)
    for s in range(O.num_segments(N, p)):
        sp = res["plans"][(0, 0, s)]
        e = O.admissible_end(N, s, p)
        lo, hi = O.candidate_range(N, s, p)
        assert sp.M == 0.0 and sp.Z == float(e)
        assert sp.order.tolist() == list(range(lo, hi))
        nb = O.num_blocks(hi - lo, p)
        assert np.allclose(sp.masses, 64.0 / e, rtol=1e-14, atol=0)
        want_C = nb if 64.0 / e >= tau else 0
        assert sp.C == want_C
        if e == 1024 and tau == 0.0625:
            assert nb > 0 and sp.C == nb and np.all(sp.masses == tau)
        # every adjacent pair is an exact tie
        assert len(sp.score_ties) == max(0, hi - lo - 1)


# ---------------------------------------------------------------------------
# invariants on random inputs
# ---------------------------------------------------------------------------

def _random_case(seed, B=1, Hq=4, Hkv=1, N=768, d=64, planted=True):
    Q, K, V = synth.generate(B, Hq, Hkv, N, d, planted=planted, band=d >= 32, n_stripe=6, seed=seed)
    return Q, K, V


def test_masses_sum_to_one_and_are_nonincreasing():
    p = O.Params(tau=1e-3)
    Q, K, V = _random_case(1)
    N = Q.shape[2]
    res = O.plan(Q, K, p)
    for s in range(O.num_segments(N, p)):
        sp = res["plans"][(0, 0, s)]
        always = O.always_kept(N, s, p)
        rest = np.exp(sp.scores[always] - sp.M).sum() / sp.Z
        assert sp.masses.sum() + rest == pytest.approx(1.0, abs=1e-12)
        assert np.all(np.diff(sp.masses) <= 0)
        # the stop rule: every kept block is >= tau, the first dropped one < tau
        assert np.all(sp.masses[:sp.C] >= p.tau)
        if sp.C < len(sp.masses):
            assert sp.masses[sp.C] < p.tau


def test_order_is_sorted_with_index_tiebreak():
    p = O.Params()
    Q, K, V = _random_case(2)
    res = O.plan(Q, K, p)
    N = Q.shape[2]
    for s in range(O.num_segments(N, p)):
        sp = res["plans"][(0, 0, s)]
        sc = sp.scores[sp.order]
        for a in range(len(sc) - 1):
            assert sc[a] > sc[a + 1] or (sc[a] == sc[a + 1] and sp.order[a] < sp.order[a + 1])


def test_tau_zero_equals_library_causal_attention():
    # tau = 0 keeps every block, so the output must be plain causal attention;
    # torch's scaled_dot_product_attention in fp64 is the independent reference.
    p = O.Params(tau=0.0)
    Q, K, V = _random_case(3, Hq=4, Hkv=2, N=640, d=64)
    res = O.plan(Q, K, p)
    N = Q.shape[2]
    for s in range(O.num_segments(N, p)):
        lo, hi = O.candidate_range(N, s, p)
        assert res["nblocks"][0, 0, s] == O.num_blocks(hi - lo, p)
    out = O.attention(Q, K, V, res["perm"], res["nblocks"], p)
    G = 2
    q = torch.from_numpy(O.widen_bf16(Q))
    k = torch.from_numpy(O.widen_bf16(K)).repeat_interleave(G, dim=1)
    v = torch.from_numpy(O.widen_bf16(V)).repeat_interleave(G, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True).numpy()
    assert np.max(np.abs(out - ref)) < 1e-12


def test_output_invariant_under_physical_permutation():
    # Keys are addressed through an index list; storing K/V rows in another
    # physical order and remapping the indices must not change the output.
    p = O.Params(tau=3e-3)
    Q, K, V = _random_case(4, Hq=2, Hkv=1, N=896, d=64)
    N = Q.shape[2]
    res = O.plan(Q, K, p)
    rng = np.random.default_rng(11)
    pi = rng.permutation(N)            # logical j lives at physical row pi[j]
    Kp = np.empty_like(K)
    Vp = np.empty_like(V)
    Kp[:, :, pi] = K
    Vp[:, :, pi] = V
    off = res["offsets"]
    for s in (0, 1, 3, 6):
        keep = O.keep_set(N, s, res["perm"][0, 0, off[s]:off[s + 1]], int(res["nblocks"][0, 0, s]), p)
        a = O.attention_segment(Q, K, V, 0, 0, s, 2, keep, p)
        b = O.attention_segment(Q, Kp, Vp, 0, 0, s, 2, keep, p, phys_of_logical=pi)
        assert np.max(np.abs(a - b)) <= 1e-12


def test_near_tie_reporting():
    p = O.Params(Lq=4, Bk=2, n_sink=1, window_prev=0, tau=0.3)
    N, d = 8, 4
    K = np.zeros((1, 1, N, d), dtype=np.float32)
    K[0, 0, :, 0] = [0, 1, 1, 2, 0, 0, 0, 0]  # keys 1 and 2 tie exactly
    Q = np.zeros((1, 1, N, d), dtype=np.float32)
    Q[0, 0, 4:, 0] = 2.0
    sp = O.plan_segment(_bits(Q), _bits(K), 0, 0, 1, 1, p)
    assert sp.order.tolist() == [3, 1, 2]
    assert sp.score_ties.tolist() == [1]


# ---------------------------------------------------------------------------
# brute force on N = 16
# ---------------------------------------------------------------------------

def _brute_force(Qv, Kv, Vv, G, Lq, Bk, n_sink, W, tau):
    """Plain-Python evaluation of the method on a tiny input (lists and math)."""
    B, Hq, N, d = len(Qv), len(Qv[0]), len(Qv[0][0]), len(Qv[0][0][0])
    Hkv = Hq // G
    out = [[[[0.0] * d for _ in range(N)] for _ in range(Hq)] for _ in range(B)]
    Cs = {}
    S = -(-N // Lq)
    for b in range(B):
        for kv in range(Hkv):
            for s in range(S):
                rows = list(range(Lq * s, min(N, Lq * s + Lq)))
                e = rows[-1] + 1
                qbar = [sum(Qv[b][kv * G + g][i][c] for g in range(G) for i in rows) / (G * len(rows))
                        for c in range(d)]
                sc = [sum(qbar[c] * Kv[b][kv][j][c] for c in range(d)) / math.sqrt(d) for j in range(e)]
                Mx = max(sc)
                Zs = sum(math.exp(x - Mx) for x in sc)
                w0 = max(0, Lq * s - W)
                always = set(range(min(n_sink, e))) | set(range(w0, e))
                cand = [j for j in range(e) if j not in always]
                order = sorted(cand, key=lambda j: (-sc[j], j))
                blocks = [order[k:k + Bk] for k in range(0, len(order), Bk)]
                mass = [sum(math.exp(sc[j] - Mx) for j in blk) / Zs for blk in blocks]
                # C = the largest c such that each of the first c blocks has mass >= tau
                C = 0
                while C < len(blocks) and all(mass[t] >= tau for t in range(C + 1)):
                    C += 1
                Cs[(b, kv, s)] = C
                keep = always | {j for blk in blocks[:C] for j in blk}
                for g in range(G):
                    h = kv * G + g
                    for i in rows:
                        vis = [j for j in range(i + 1) if j in keep]
                        logits = [sum(Qv[b][h][i][c] * Kv[b][kv][j][c] for c in range(d)) / math.sqrt(d)
                                  for j in vis]
                        mx = max(logits)
                        ws = [math.exp(x - mx) for x in logits]
                        tot = sum(ws)
                        for c in range(d):
                            out[b][h][i][c] = sum(wj * Vv[b][kv][j][c] for wj, j in zip(ws, vis)) / tot
    return out, Cs


@pytest.mark.parametrize("tau", [0.0, 0.05, 0.2])
def test_brute_force_n16(tau):
    p = O.Params(Lq=4, Bk=2, n_sink=1, window_prev=4, tau=tau)
    rng = np.random.default_rng(7)
    B, Hq, Hkv, N, d = 1, 2, 1, 16, 8
    Q = _bits(rng.standard_normal((B, Hq, N, d)) * 1.5)
    K = _bits(rng.standard_normal((B, Hkv, N, d)) * 1.5)
    V = _bits(rng.standard_normal((B, Hkv, N, d)))
    res = O.plan(Q, K, p)
    out = O.attention(Q, K, V, res["perm"], res["nblocks"], p)
    bf, Cs = _brute_force(O.widen_bf16(Q).tolist(), O.widen_bf16(K).tolist(), O.widen_bf16(V).tolist(),
                          2, 4, 2, 1, 4, tau)
    for (b, kv, s), C in Cs.items():
        assert res["nblocks"][b, kv, s] == C
    assert np.max(np.abs(out - np.array(bf))) < 1e-12
    if tau > 0:
        # the threshold must actually bind somewhere for the test to mean something
        full = [O.num_blocks(O.num_candidates(N, s, p), p) for s in range(4)]
        assert any(res["nblocks"][0, 0, s] < full[s] for s in range(4))


def test_kept_pairs_dense_closed_form():
    p = O.Params(tau=0.0)
    N = 512
    total = 0
    for s in range(O.num_segments(N, p)):
        keep = np.arange(O.admissible_end(N, s, p))
        total += O.kept_pairs_segment(N, s, keep, p)
    assert total == N * (N + 1) // 2


# ---------------------------------------------------------------------------
# the bound behind the filtered plan
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("tau", [1e-4, 1e-3, 3e-3, 1e-2, 5e-2])
def test_stop_point_within_threshold_prefix(tau):
    # A block is a sum of Bk masses; if all of them are below tau/Bk it is
    # below tau.  So the stop point can be no later than the first block that
    # starts at or after n_hi = #{candidates with mass >= tau/Bk}, and the
    # first Bk*ceil(n_hi/Bk) entries of the order decide C.  The masses here
    # are recomputed from the scores, not taken from the oracle's blocks.
    p = O.Params(tau=tau)
    seen_bound = False
    for seed in (1, 2):
        Q, K, V = _random_case(seed, N=4096)
        N = Q.shape[2]
        res = O.plan(Q, K, p)
        for s in range(O.num_segments(N, p)):
            sp = res["plans"][(0, 0, s)]
            lo, hi = O.candidate_range(N, s, p)
            if hi <= lo:
                continue
            w = np.exp(sp.scores[lo:hi] - sp.M) / sp.Z
            n_hi = int(np.count_nonzero(w >= tau / p.Bk))
            bound = -(-n_hi // p.Bk)
            assert sp.C <= bound
            # the same C from the prefix alone
            L = min(hi - lo, p.Bk * bound)
            head = np.exp(sp.scores[sp.order[:L]] - sp.M) / sp.Z
            C2 = bound
            for k in range(L // p.Bk):
                if head[k * p.Bk:(k + 1) * p.Bk].sum() < tau:
                    C2 = k
                    break
            assert C2 == sp.C
            seen_bound |= bound < O.num_blocks(hi - lo, p)
    # at these sizes the bound cuts the order for the larger thresholds
    assert seen_bound or tau < 3e-3


# ---------------------------------------------------------------------------
# run-time (online) stop rule
# ---------------------------------------------------------------------------

def test_online_tau_zero_processes_every_block_and_is_dense():
    p = O.Params(tau=0.0)
    Q, K, V = _random_case(5, Hq=4, Hkv=1, N=896, d=64)
    N = Q.shape[2]
    res = O.plan(Q, K, p)
    off = res["offsets"]
    for s in range(O.num_segments(N, p)):
        perm_seg = res["perm"][0, 0, off[s]:off[s + 1]]
        for pair in range(2):
            st = O.online_stop_segment(Q, K, 0, 0, s, O.tile_heads(0, 4, pair), perm_seg, p)
            assert st.C == O.num_blocks(len(perm_seg), p)
            assert np.all(st.gains > 0)
        keep = O.keep_set(N, s, perm_seg, st.C, p)
        got = O.attention_segment(Q, K, V, 0, 0, s, 4, keep, p)
        want = O.dense_segment(Q, K, V, 0, 0, s, 4, p)
        assert np.max(np.abs(got - want)) <= 1e-12


def test_online_all_ties_closed_form():
    # Q = 0 makes every score 0, so every key weighs 1: after candidate block b
    # row i has processed n_i always-kept keys plus Bk (b + 1) candidates and
    # its gain is Bk / (n_i + Bk (b + 1)).  n_i counts sinks and window keys
    # <= i directly from the geometry below.
    N, Lq, Bk, W, ns = 4096, 128, 64, 128, 64
    tau = 0.03
    p = O.Params(tau=tau)
    rng = np.random.default_rng(3)
    Q = np.zeros((1, 2, N, 64), dtype=np.uint16)
    K = _bits(rng.standard_normal((1, 1, N, 64)))
    hit = 0
    for s in (2, 9, 20, 31):
        r0 = Lq * s
        rows = np.arange(r0, min(N, r0 + Lq))
        n_i = ns + (rows - (r0 - W) + 1)          # sinks, then the window up to row i
        ncand = max(0, Lq * s - W - ns)
        nb = ncand // Bk
        want_C, want_g = nb, []
        for blk in range(nb):
            g = float(np.mean(Bk / (n_i + Bk * (blk + 1))))
            want_g.append(g)
            if g < tau:
                want_C = blk + 1
                break
        perm_seg = np.arange(ns, ns + ncand)
        st = O.online_stop_segment(Q, K, 0, 0, s, [0, 1], perm_seg, p)
        assert st.C == want_C
        assert np.allclose(st.gains, want_g, rtol=1e-12, atol=0)
        hit += want_C < nb
    assert hit >= 2  # the threshold binds in some of these segments


def _brute_online(Qv, Kv, heads, s, perm_seg, Lq, Bk, n_sink, W, tau):
    """Plain-Python gains and stop point of one tile (lists and math.exp)."""
    N, d = len(Kv), len(Kv[0])
    r0, r1 = Lq * s, min(N, Lq * s + Lq)
    e = r1
    always = sorted(set(range(min(n_sink, e))) | set(range(max(0, Lq * s - W), e)))
    nb = -(-len(perm_seg) // Bk)  # the last block may be partial
    L, gains, C = {}, [], nb
    for h in heads:
        for i in range(r0, r1):
            L[(h, i)] = sum(math.exp(sum(Qv[h][i][c] * Kv[j][c] for c in range(d)) / math.sqrt(d))
                            for j in always if j <= i)
    for blk in range(nb):
        tot, cnt = 0.0, 0
        for h in heads:
            for i in range(r0, r1):
                w = sum(math.exp(sum(Qv[h][i][c] * Kv[j][c] for c in range(d)) / math.sqrt(d))
                        for j in perm_seg[blk * Bk:(blk + 1) * Bk])
                L[(h, i)] += w
                tot += w / L[(h, i)]
                cnt += 1
        gains.append(tot / cnt)
        if tot / cnt < tau:
            C = blk + 1
            break
    return C, gains


@pytest.mark.parametrize("tau", [0.2, 0.3])
def test_online_brute_force_n16(tau):
    p = O.Params(Lq=4, Bk=2, n_sink=1, window_prev=4, tau=tau)
    rng = np.random.default_rng(9)
    N, d = 16, 8
    Q = _bits(rng.standard_normal((1, 2, N, d)) * 1.5)
    K = _bits(rng.standard_normal((1, 1, N, d)) * 1.5)
    Qv, Kv = O.widen_bf16(Q)[0].tolist(), O.widen_bf16(K)[0, 0].tolist()
    res = O.plan(Q, K, p)
    off = res["offsets"]
    stopped = 0
    for s in range(O.num_segments(N, p)):
        perm_seg = res["perm"][0, 0, off[s]:off[s + 1]]
        st = O.online_stop_segment(Q, K, 0, 0, s, [0, 1], perm_seg, p)
        C, g = _brute_online(Qv, Kv, [0, 1], s, [int(x) for x in perm_seg], 4, 2, 1, 4, tau)
        assert st.C == C
        assert np.allclose(st.gains, g, rtol=1e-12, atol=0)
        stopped += C < -(-len(perm_seg) // 2)
    assert stopped >= 1


def test_online_invariant_under_physical_permutation():
    p = O.Params(tau=0.01)
    Q, K, V = _random_case(6, Hq=2, Hkv=1, N=1024, d=64)
    N = Q.shape[2]
    res = O.plan(Q, K, p)
    rng = np.random.default_rng(12)
    pi = rng.permutation(N)
    Kp = np.empty_like(K)
    Kp[:, :, pi] = K
    off = res["offsets"]
    for s in (2, 4, 7):
        perm_seg = res["perm"][0, 0, off[s]:off[s + 1]]
        a = O.online_stop_segment(Q, K, 0, 0, s, [0, 1], perm_seg, p)
        b = O.online_stop_segment(Q, Kp, 0, 0, s, [0, 1], perm_seg, p, phys_of_logical=pi)
        assert a.C == b.C
        assert np.allclose(a.gains, b.gains, rtol=1e-12, atol=0)


# ---------------------------------------------------------------------------
# ranking accuracy: true block masses
# ---------------------------------------------------------------------------

def test_true_masses_sum_to_one_with_the_always_kept_keys():
    # each row's softmax sums to 1, so the mean over rows does too
    p = O.Params(tau=1e-3)
    Q, K, V = _random_case(8, Hq=4, Hkv=1, N=1024, d=64)
    N = Q.shape[2]
    res = O.plan(Q, K, p)
    off = res["offsets"]
    for s in range(O.num_segments(N, p)):
        bt = O.true_block_masses(Q, K, 0, 0, s, 4, res["perm"][0, 0, off[s]:off[s + 1]], int(res["nblocks"][0, 0, s]), p)
        assert bt.total + bt.always == pytest.approx(1.0, abs=1e-12)
        assert 0 <= bt.both <= min(bt.kept, bt.true)
        assert bt.captured <= bt.total + 1e-15


def test_true_masses_uniform_closed_form():
    # Q = 0: row i attends uniformly to its i + 1 keys, so a candidate key
    # (j < every row) gets mean_i 1/(i + 1) and a block 64 times that
    N = 1024
    p = O.Params(tau=1e-3)
    rng = np.random.default_rng(2)
    Q = np.zeros((1, 2, N, 64), dtype=np.uint16)
    K = _bits(rng.standard_normal((1, 1, N, 64)))
    for s in (2, 5, 7):
        rows = np.arange(128 * s, 128 * s + 128)
        per_key = float(np.mean(1.0 / (rows + 1)))
        ncand = 128 * s - 192
        perm_seg = np.arange(64, 64 + ncand)[::-1].copy()
        bt = O.true_block_masses(Q, K, 0, 0, s, 2, perm_seg, 2, p)
        assert np.allclose(bt.mass, 64 * per_key, rtol=1e-12, atol=0)
        assert bt.true == (len(bt.mass) if 64 * per_key >= p.tau else 0)
        kept = min(2, len(bt.mass))
        assert bt.kept == kept and bt.both == (kept if 64 * per_key >= p.tau else 0)
        assert bt.captured == pytest.approx(kept * 64 * per_key, rel=1e-12)


def test_true_masses_brute_force_n16():
    p = O.Params(Lq=4, Bk=2, n_sink=1, window_prev=4, tau=0.1)
    rng = np.random.default_rng(4)
    N, d, G = 16, 8, 2
    Q = _bits(rng.standard_normal((1, G, N, d)) * 1.5)
    K = _bits(rng.standard_normal((1, 1, N, d)) * 1.5)
    Qv, Kv = O.widen_bf16(Q)[0].tolist(), O.widen_bf16(K)[0, 0].tolist()
    res = O.plan(Q, K, p)
    off = res["offsets"]
    for s in range(2, O.num_segments(N, p)):
        perm_seg = [int(x) for x in res["perm"][0, 0, off[s]:off[s + 1]]]
        rows = range(4 * s, 4 * s + 4)
        col = {j: 0.0 for j in range(N)}
        for g in range(G):
            for i in rows:
                w = [math.exp(sum(Qv[g][i][c] * Kv[j][c] for c in range(d)) / math.sqrt(d)) for j in range(i + 1)]
                for j in range(i + 1):
                    col[j] += w[j] / sum(w) / (G * 4)
        want = [sum(col[j] for j in perm_seg[k:k + 2]) for k in range(0, len(perm_seg), 2)]
        bt = O.true_block_masses(Q, K, 0, 0, s, G, perm_seg, int(res["nblocks"][0, 0, s]), p)
        assert np.allclose(bt.mass, want, rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------------------
# Q_perm with finer sub-segments
# ---------------------------------------------------------------------------

def test_qperm_partition_follows_a_known_importance():
    # rows q_i = c_i u with a shared unit u: qbar = mean(c) u and the importance
    # of row i is c_i mean(c), so with mean(c) > 0 the rows order by c_i
    # (ties to the lower row); some c repeat to exercise the tie-break
    N, d = 512, 64
    p = O.Params(tau=1e-3)
    rng = np.random.default_rng(13)
    u = np.zeros(d); u[3] = 1.0
    c = rng.integers(1, 40, size=N).astype(np.float32) / 8.0
    Q = _bits((c[None, None, :, None] * u[None, None, None, :]).repeat(2, axis=1))
    K = _bits(rng.standard_normal((1, 1, N, d)))
    for s in (2, 3):
        r0 = 128 * s
        rows = np.arange(r0, r0 + 128)
        want_order = rows[np.lexsort((rows, -c[r0:r0 + 128]))]
        sp = O.qperm_segment(Q, K, 0, 0, s, 2, p)
        assert np.array_equal(sp.rows, want_order)
        assert np.array_equal(np.nonzero(sp.sub_of_row == 0)[0] + r0, np.sort(want_order[:64]))
        # each sub-segment's pooled query is the mean of its rows (both heads)
        for sub in (0, 1):
            grp = np.sort(want_order[64 * sub:64 * (sub + 1)])
            want_q = float(np.mean(c[grp])) * u
            assert np.allclose(sp.plans[sub].qbar, want_q, rtol=0, atol=1e-12)


def test_qperm_identical_rows_reduce_to_the_segment_plan():
    # every row of a segment equal: both sub-segments pool to qbar, so their
    # plans and the outputs equal the unpermuted method
    N, d = 768, 64
    p = O.Params(tau=3e-3)
    rng = np.random.default_rng(14)
    base = rng.standard_normal((1, 2, N // 128, 1, d))
    Q = _bits(np.repeat(base, 128, axis=3).reshape(1, 2, N, d))
    K = _bits(rng.standard_normal((1, 1, N, d)))
    V = _bits(rng.standard_normal((1, 1, N, d)))
    for s in range(O.num_segments(N, p)):
        sp = O.qperm_segment(Q, K, 0, 0, s, 2, p)
        ref = O.plan_segment(Q, K, 0, 0, s, 2, p)
        for sub in (0, 1):
            assert np.array_equal(sp.plans[sub].order, ref.order)
            assert sp.plans[sub].C == ref.C
        keeps = [sp.plans[0].keep, sp.plans[1].keep]
        got = O.attention_qperm_segment(Q, K, V, 0, 0, s, 2, keeps, sp.sub_of_row, p)
        want = O.attention_segment(Q, K, V, 0, 0, s, 2, ref.keep, p)
        assert np.max(np.abs(got - want)) <= 1e-12


def test_qperm_each_row_uses_its_own_kept_set():
    # brute force on N = 16 (Lq = 4: sub-segments of 2 rows): each row's
    # output is plain softmax attention over its own sub-segment's kept keys
    p = O.Params(Lq=4, Bk=2, n_sink=1, window_prev=4, tau=0.15)
    rng = np.random.default_rng(15)
    N, d = 16, 8
    Q = _bits(rng.standard_normal((1, 1, N, d)) * 1.5)
    K = _bits(rng.standard_normal((1, 1, N, d)) * 1.5)
    V = _bits(rng.standard_normal((1, 1, N, d)))
    Qv, Kv, Vv = O.widen_bf16(Q)[0, 0], O.widen_bf16(K)[0, 0], O.widen_bf16(V)[0, 0]
    differ = 0
    for s in range(O.num_segments(N, p)):
        sp = O.qperm_segment(Q, K, 0, 0, s, 1, p)
        keeps = [sp.plans[0].keep, sp.plans[1].keep]
        differ += not np.array_equal(keeps[0], keeps[1])
        got = O.attention_qperm_segment(Q, K, V, 0, 0, s, 1, keeps, sp.sub_of_row, p)
        for r, i in enumerate(range(4 * s, 4 * s + 4)):
            keys = [int(j) for j in keeps[int(sp.sub_of_row[r])] if j <= i]
            w = [math.exp(float(Qv[i] @ Kv[j]) / math.sqrt(d)) for j in keys]
            want = sum(wj * Vv[j] for wj, j in zip(w, keys)) / sum(w)
            assert np.allclose(got[0, r], want, rtol=0, atol=1e-12)
    assert differ >= 1  # some segment's two sub-segments keep different keys
