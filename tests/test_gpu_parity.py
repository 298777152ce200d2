"""GPU parity: the CUDA plan and attention, called through the C ABI, against
the fp64 oracle on the same seeded bf16 inputs."""
import numpy as np
import pytest
import torch

import score_keys_pooled_b200 as s2o
from score_keys_pooled_b200 import synth
from oracle import s2o_oracle as O
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    s2o.lib()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def run_path(Q, K, V, tau, out_dtype=s2o.OUT_BF16):
    B, Hq, N, d = Q.shape
    cfg = s2o.make_config(B, Hq, K.shape[1], N, tau=tau)
    q, k, v = dev(Q), dev(K), dev(V)
    bufs = s2o.plan(cfg, q, k)
    assert s2o.last_launch_count() >= 6
    out = s2o.attention(cfg, q, k, v, bufs["perm"], bufs["nblocks"], out_dtype=out_dtype)
    assert s2o.last_launch_count() == 1
    assert s2o.last_device_error() == 0
    return cfg, bufs, out


def host_plan(cfg, bufs):
    BH = cfg.B * cfg.Hkv
    S, T = s2o.num_segments(cfg), s2o.num_candidates(cfg)
    perm = bufs["perm"][:BH * T].cpu().numpy().reshape(cfg.B, cfg.Hkv, T)
    nb = bufs["nblocks"].cpu().numpy().reshape(cfg.B, cfg.Hkv, S)
    scores = bufs["scores"][:BH * T].cpu().numpy().reshape(cfg.B, cfg.Hkv, T)
    stats = bufs["seg_stats"].cpu().numpy().reshape(cfg.B, cfg.Hkv, S, 2)
    return perm, nb, scores, stats


def check_plan(Q, K, cfg, bufs, p, segments=None, kvheads=None, what="", prefix_only=False):
    perm, nb, scores, stats = host_plan(cfg, bufs)
    G = cfg.Hq // cfg.Hkv
    off = O.candidate_offsets(cfg.N, p)
    S = O.num_segments(cfg.N, p)
    segs = range(S) if segments is None else segments
    heads = [(b, h) for b in range(cfg.B) for h in (range(cfg.Hkv) if kvheads is None else kvheads)]
    swaps = flips = 0
    plans = {}
    for b, kvh in heads:
        for s in segs:
            sp = O.plan_segment(Q, K, b, kvh, s, G, p)
            plans[(b, kvh, s)] = sp
            lo, hi = O.candidate_range(cfg.N, s, p)
            # scores: the exact values rounded to fp32 (half an ulp), plus the
            # fixed-point representation's bound
            e = len(sp.scores)
            bound = parity.score_error_bound(sp.qbar, O.widen_bf16(K[b, kvh, :e]) if K.dtype == np.uint16
                                             else K[b, kvh, :e])
            gs = scores[b, kvh, off[s]:off[s + 1]].astype(np.float64)
            ref = sp.scores[lo:hi]
            half_ulp = 0.5 * np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
            assert np.all(np.abs(gs - ref) <= half_ulp + bound[lo:hi] + 1e-300)
            # (in fp64: numpy keeps float32 - float in float32)
            assert abs(float(stats[b, kvh, s, 0]) - sp.M) <= (0.5 * float(np.spacing(np.float32(abs(sp.M))))
                                                              + float(bound.max(initial=0.0)))
            assert abs(float(stats[b, kvh, s, 1]) / sp.Z - 1.0) <= 1e-5
            sw, fl = parity.compare_segment_plan(perm[b, kvh, off[s]:off[s + 1]], int(nb[b, kvh, s]), sp, p,
                                                 prefix_only=prefix_only)
            swaps += sw
            flips += fl
    parity.log_near_ties({"case": what, "tau": p.tau, "segments": len(segs) * len(heads),
                          "swapped_positions": swaps, "C_flips": flips})
    return perm, nb, plans


def check_output(Q, K, V, cfg, perm, nb, out, p, segments=None, kvheads=None, what=""):
    G = cfg.Hq // cfg.Hkv
    off = O.candidate_offsets(cfg.N, p)
    S = O.num_segments(cfg.N, p)
    segs = range(S) if segments is None else segments
    got = out.float().cpu().numpy()
    worst = (0.0, 0.0)
    for b in range(cfg.B):
        for kvh in (range(cfg.Hkv) if kvheads is None else kvheads):
            for s in segs:
                keep = O.keep_set(cfg.N, s, perm[b, kvh, off[s]:off[s + 1]], int(nb[b, kvh, s]), p)
                ref = O.attention_segment(Q, K, V, b, kvh, s, G, keep, p)
                r0, r1 = O.segment_rows(cfg.N, s, p)
                g = got[b, kvh * G:(kvh + 1) * G, r0:r1]
                e = parity.assert_output_close(g, ref, f"{what} b={b} kvh={kvh} s={s}")
                worst = (max(worst[0], e[0]), max(worst[1], e[1]))
    return worst


SMALL = [
    # (B, Hq, Hkv, N, tau, planted, band)
    (1, 1, 1, 1024, 1e-3, True, False),
    (1, 8, 2, 1280, 3e-3, True, True),
    (1, 8, 2, 1280, 0.0, True, True),
    (1, 8, 2, 1280, 2.0, True, True),
    (2, 4, 2, 768, 1e-2, True, False),
    (1, 4, 1, 1000, 1e-2, True, True),
    (1, 4, 1, 1111, 5e-3, False, False),
    (1, 4, 4, 640, 1e-3, True, True),
    (1, 6, 2, 900, 3e-3, True, True),  # G = 3: the odd-group kernel
]


@pytest.mark.parametrize("B,Hq,Hkv,N,tau,planted,band", SMALL)
@pytest.mark.parametrize("out_dtype", [s2o.OUT_BF16, s2o.OUT_F32])
def test_small_cases_full_parity(B, Hq, Hkv, N, tau, planted, band, out_dtype):
    Q, K, V = synth.generate(B, Hq, Hkv, N, 128, planted=planted, band=band, n_stripe=8, seed=N + Hq)
    p = O.Params(tau=tau)
    cfg, bufs, out = run_path(Q, K, V, tau, out_dtype)
    perm, nb, plans = check_plan(Q, K, cfg, bufs, p, what=f"small N={N}")
    if tau == 0.0:
        for (b, kvh, s), sp in plans.items():
            assert nb[b, kvh, s] == O.num_blocks(O.num_candidates(N, s, p), p)
    check_output(Q, K, V, cfg, perm, nb, out, p, what=f"small N={N}")


@pytest.mark.parametrize("N", [1, 63, 64, 127, 128, 129, 255, 256, 300, 385])
def test_ragged_and_tiny_lengths(N):
    Q, K, V = synth.generate(1, 2, 1, N, 128, planted=N > 4, band=True, n_stripe=2, seed=N)
    p = O.Params(tau=1e-3)
    cfg, bufs, out = run_path(Q, K, V, 1e-3)
    perm, nb, _ = check_plan(Q, K, cfg, bufs, p, what=f"ragged N={N}")
    check_output(Q, K, V, cfg, perm, nb, out, p, what=f"ragged N={N}")


@pytest.mark.parametrize("tau", [1e-3, 0.0625, 0.07])
def test_all_ties_bit_exact(tau):
    # Q = 0: every score is exactly 0, so the order is ascending and
    # m_b = 64 / e(s) exactly; no tolerance applies.
    N = 1024
    Q = np.zeros((1, 4, N, 128), dtype=np.uint16)
    _, K, V = synth.generate(1, 4, 1, N, 128, planted=True, band=False, n_stripe=8, seed=3)
    cfg, bufs, out = run_path(Q, K, V, tau)
    perm, nb, scores, stats = host_plan(cfg, bufs)
    p = O.Params(tau=tau)
    off = O.candidate_offsets(N, p)
    assert np.all(scores == 0.0)
    for s in range(O.num_segments(N, p)):
        lo, hi = O.candidate_range(N, s, p)
        assert np.array_equal(perm[0, 0, off[s]:off[s + 1]], np.arange(lo, hi))
        e = O.admissible_end(N, s, p)
        nbk = O.num_blocks(hi - lo, p)
        assert nb[0, 0, s] == (nbk if 64.0 / e >= tau else 0)
        assert stats[0, 0, s, 0] == 0.0 and stats[0, 0, s, 1] == float(e)


@pytest.mark.parametrize("seed", [41, 42])
def test_scores_across_wide_exponent_ranges(seed):
    """Inputs that strain the scorer's fixed point: key rows whose elements
    span up to 80 binades (most of a row's small elements are rounded), rows
    with a single nonzero element, rows of bf16 subnormals and zeros, and
    pooled queries from 2^-100 to 2^40 in scale.  Scores must stay within half
    an ulp plus the representation bound of the exact values, and the order,
    M, Z and C(s) must match the oracle as everywhere else."""
    B, Hq, Hkv, N, tau = 1, 4, 2, 1280, 1e-3
    Q, K, V = synth.generate(B, Hq, Hkv, N, 128, planted=True, band=True, n_stripe=8, seed=seed)
    rng = np.random.default_rng(seed)
    Kf = O.widen_bf16(K).astype(np.float32)
    # per-element scales 2^e, e uniform in [-40, 40], on a third of the rows
    rows = rng.random(N) < 1 / 3
    Kf[:, :, rows] *= np.exp2(rng.integers(-40, 41, size=(B, Hkv, int(rows.sum()), 128))).astype(np.float32)
    # single-element rows and subnormal rows
    for j in rng.choice(np.arange(64, N), size=24, replace=False):
        Kf[:, :, j] = 0.0
        Kf[:, :, j, rng.integers(0, 128)] = rng.choice([-1.0, 1.0]) * np.float32(2.0 ** rng.integers(-30, 30))
    for j in rng.choice(np.arange(64, N), size=8, replace=False):
        Kf[:, :, j] = rng.standard_normal(128).astype(np.float32) * np.float32(2.0 ** -130)
    K = synth.to_bf16_bits(Kf)
    # pooled queries of very different scales, one segment each
    Qf = O.widen_bf16(Q).astype(np.float32)
    for s, e in ((2, -100), (3, -20), (5, 20), (7, 40)):
        Qf[:, :, 128 * s:128 * s + 128] *= np.float32(2.0 ** e)
    Q = synth.to_bf16_bits(Qf)
    cfg = s2o.make_config(B, Hq, Hkv, N, tau=tau)
    bufs = s2o.plan(cfg, dev(Q), dev(K))
    assert s2o.last_device_error() == 0
    check_plan(Q, K, cfg, bufs, O.Params(tau=tau), what=f"wide exponents seed={seed}")


@pytest.mark.parametrize("world", [2, 3, 8])
def test_kv_head_shards_reassemble_the_whole_problem(world):
    """One problem sharded by KV head (bench.py --shard heads): every rank's
    library call on its share, run here one after another on one GPU, gives
    exactly the whole call's C(s) and output rows."""
    import bench
    B, Hq, Hkv, N, tau = 1, 32, 8, 2048, 3e-3
    Q, K, V = synth.generate(B, Hq, Hkv, N, 128, planted=True, band=True, n_stripe=16, seed=23)
    cfg, bufs, out = run_path(Q, K, V, tau)
    G = Hq // Hkv
    S = s2o.num_segments(cfg)
    nb_all = bufs["nblocks"].view(B, Hkv, S)
    for rank in range(world):
        k0, k1 = bench.kv_head_slice(Hkv, world, rank)
        q, k, v = bench.shard_inputs(Q, K, V, world, rank)
        c_loc, b_loc, o_loc = run_path(q, k, v, tau)
        assert torch.equal(b_loc["nblocks"].view(B, k1 - k0, S), nb_all[:, k0:k1])
        assert torch.equal(o_loc, out[:, k0 * G:k1 * G])


def test_nonfinite_input_is_reported():
    Q, K, V = synth.generate(1, 4, 1, 512, 128, planted=True, band=False, n_stripe=4, seed=9)
    K = K.copy()
    K[0, 0, 300, 5] = 0x7FC0  # bf16 NaN
    cfg = s2o.make_config(1, 4, 1, 512, tau=1e-3)
    s2o.plan(cfg, dev(Q), dev(K))
    assert s2o.last_device_error() == 6
    assert s2o.last_device_error() == 0  # the word is cleared by the read


def test_out_of_range_plan_is_clamped_and_reported():
    Q, K, V = synth.generate(1, 4, 1, 768, 128, planted=True, band=False, n_stripe=4, seed=10)
    cfg = s2o.make_config(1, 4, 1, 768, tau=0.0)
    q, k, v = dev(Q), dev(K), dev(V)
    bufs = s2o.plan(cfg, q, k)
    perm = bufs["perm"].clone()
    perm[3] = 10 ** 6
    s2o.attention(cfg, q, k, v, perm, bufs["nblocks"])
    assert s2o.last_device_error() == 7
    nbad = bufs["nblocks"].clone()
    nbad[4] = 999
    s2o.attention(cfg, q, k, v, bufs["perm"], nbad)
    assert s2o.last_device_error() == 7
    assert s2o.last_device_error() == 0


@pytest.mark.parametrize("B,Hq,Hkv,N,out_dtype", [(1, 8, 2, 1536, s2o.OUT_BF16), (2, 4, 2, 1000, s2o.OUT_F32),
                                                  (2, 4, 4, 640, s2o.OUT_BF16), (1, 6, 2, 900, s2o.OUT_BF16)])
def test_host_buffer_entry_matches_device_path(B, Hq, Hkv, N, out_dtype):
    # the host entry pipelines its work by (b, kvh) over three streams; the
    # result must equal the device path bit for bit
    Q, K, V = synth.generate(B, Hq, Hkv, N, 128, planted=True, band=True, n_stripe=8, seed=12)
    cfg, bufs, out = run_path(Q, K, V, 1e-3, out_dtype)
    arena = torch.empty(s2o.prefill_arena_size(cfg, out_dtype), dtype=torch.uint8, device="cuda")
    pin = lambda a: torch.from_numpy(a.view(np.int16)).pin_memory()
    odt = torch.int16 if out_dtype == s2o.OUT_BF16 else torch.float32
    O_host = torch.empty(Q.shape, dtype=odt).pin_memory()
    nb_host = torch.empty(cfg.B * cfg.Hkv * s2o.num_segments(cfg), dtype=torch.int32)
    s2o.prefill_host(cfg, pin(Q), pin(K), pin(V), O_host, arena, nblocks_host=nb_host, out_dtype=out_dtype)
    got = O_host.view(torch.bfloat16) if out_dtype == s2o.OUT_BF16 else O_host
    assert torch.equal(got, out.cpu())
    assert torch.equal(nb_host, bufs["nblocks"].cpu())


def sampled_segments(S):
    base = {0, 1, 2, 3, S // 4, S // 2, 3 * S // 4, S - 1}
    rng = np.random.default_rng(1)
    extra = [int(x) for x in rng.choice(np.arange(4, S - 1), 8, replace=False)]
    return sorted(base | set(extra))


@pytest.mark.parametrize("name", ["tiny_1k", "llama_16k"])
def test_workload_full_plan_sampled_output(name):
    w = synth.WORKLOADS[name]
    Q, K, V = synth.generate_workload(w)
    p = O.Params(tau=w.tau)
    cfg, bufs, out = run_path(Q, K, V, w.tau)
    perm, nb, _ = check_plan(Q, K, cfg, bufs, p, what=name)
    S = O.num_segments(w.N, p)
    segs = None if S <= 8 else sampled_segments(S)
    check_output(Q, K, V, cfg, perm, nb, out, p, segments=segs, what=name)


@pytest.mark.parametrize("name", ["llama_128k", "flat_128k"])
def test_workload_128k_sampled(name):
    # full-size launch (the benchmark's configuration); the oracle checks
    # sampled segments of every KV head for the plan and of two KV heads for
    # the output
    w = synth.WORKLOADS[name]
    Q, K, V = synth.generate_workload(w)
    p = O.Params(tau=w.tau)
    cfg, bufs, out = run_path(Q, K, V, w.tau)
    S = O.num_segments(w.N, p)
    segs = sampled_segments(S)
    perm, nb, _ = check_plan(Q, K, cfg, bufs, p, segments=segs, what=name)
    check_output(Q, K, V, cfg, perm, nb, out, p, segments=segs[::2], kvheads=[0, w.Hkv - 1], what=name)


def test_sweep_64k_tau_and_contiguous():
    w = synth.WORKLOADS["sweep_64k"]
    Q, K, V = synth.generate_workload(w)
    S = O.num_segments(w.N, O.Params())
    segs = [2, 5, S // 3, S - 1]
    q, k, v = dev(Q), dev(K), dev(V)
    for tau in synth.TAU_SWEEP:
        p = O.Params(tau=tau)
        cfg = s2o.make_config(w.B, w.Hq, w.Hkv, w.N, tau=tau)
        bufs = s2o.plan(cfg, q, k)
        assert s2o.last_device_error() == 0
        perm, nb, plans = check_plan(Q, K, cfg, bufs, p, segments=segs, kvheads=[0, 5], what=f"sweep tau={tau}")
        if tau in (1e-3, 1e-2):
            out = s2o.attention(cfg, q, k, v, bufs["perm"], bufs["nblocks"])
            check_output(Q, K, V, cfg, perm, nb, out, p, segments=segs, kvheads=[5], what=f"sweep tau={tau}")
            # contiguous comparator at the same per-segment block count
            pc = torch.empty_like(bufs["perm"])
            s2o.plan_contiguous(cfg, bufs["scores"], bufs["seg_stats"], bufs["nblocks"], pc)
            assert s2o.last_device_error() == 0
            T = s2o.num_candidates(cfg)
            pch = pc[:cfg.B * cfg.Hkv * T].cpu().numpy().reshape(cfg.B, cfg.Hkv, T)
            off = O.candidate_offsets(w.N, p)
            for s in segs:
                sp = plans[(0, 5, s)]
                want = O.contiguous_plan_segment(sp, w.N, int(nb[0, 5, s]), p)
                got = pch[0, 5, off[s]:off[s + 1]]
                # block ranks may only differ between blocks of near-equal mass
                gb = got.reshape(-1, p.Bk)[:, 0]
                wb = want.reshape(-1, p.Bk)[:, 0]
                if not np.array_equal(gb, wb):
                    lo, hi = O.candidate_range(w.N, s, p)
                    wts = np.exp(sp.scores[lo:hi] - sp.M) / sp.Z
                    bm = wts.reshape(-1, p.Bk).sum(1)
                    diff = np.nonzero(gb != wb)[0]
                    tolm = 1e-6 * bm.max()
                    assert np.all(np.abs(bm[(gb[diff] - lo) // p.Bk] - bm[(wb[diff] - lo) // p.Bk]) <= tolm)
                assert np.array_equal(np.sort(got), np.arange(O.candidate_range(w.N, s, p)[0],
                                                               O.candidate_range(w.N, s, p)[1]))
            outc = s2o.attention(cfg, q, k, v, pc, bufs["nblocks"])
            check_output(Q, K, V, cfg, pch, nb, outc, p, segments=segs, kvheads=[5], what=f"contig tau={tau}")


def test_contiguous_comparator_hand_case():
    """Keys one-hot along dim 0 (s_j = 0.99989 a_j for the pooled query
    (11.3125, 0, ...)); original-order candidate blocks B0..B4 of 64 keys:
    B0 = 32 keys at 2 and 32 at -10, B1 = B3 = 64 keys at 1.1875, B2 = one key
    at 2.5 and 63 at -10, B4 = 64 keys at -10.  Block masses go B0 > B1 = B3 >
    B2 > B4, while the largest score is in B2 and the largest raw-score sum in
    B1; B1 and B3 hold the same values in the same places, so their masses tie
    exactly and the lower block ranks first."""
    N = 640
    a = np.zeros(N, dtype=np.float32)
    a[64:96], a[96:128] = 2.0, -10.0
    a[128:192] = 1.1875
    a[192], a[193:256] = 2.5, -10.0
    a[256:320] = 1.1875
    a[320:384] = -10.0
    Kf = np.zeros((1, 1, N, 128), dtype=np.float32)
    Kf[0, 0, :, 0] = a
    Qf = np.zeros((1, 2, N, 128), dtype=np.float32)
    Qf[..., 0] = 11.3125
    Q, K = synth.to_bf16_bits(Qf), synth.to_bf16_bits(Kf)
    p = O.Params(tau=1e-3)
    cfg = s2o.make_config(1, 2, 1, N, tau=1e-3)
    bufs = s2o.plan(cfg, dev(Q), dev(K))
    pc = torch.full_like(bufs["perm"], -1)
    s2o.plan_contiguous(cfg, bufs["scores"], bufs["seg_stats"], bufs["nblocks"], pc)
    assert s2o.last_device_error() == 0
    off = O.candidate_offsets(N, p)
    got = pc.cpu().numpy()
    blk = lambda *bs: [j for b in bs for j in range(64 + 64 * b, 128 + 64 * b)]
    want = {3: blk(0, 1, 2), 4: blk(0, 1, 3, 2, 4)}
    for s, w in want.items():
        sp = O.plan_segment(Q, K, 0, 0, s, 2, p)
        assert O.contiguous_plan_segment(sp, N, 1, p).tolist() == w
        assert got[off[s]:off[s + 1]].tolist() == w


def test_mse_measurement_matches_oracle():
    """The benchmark's MSE against dense attention (the plan's fp32 output
    against the tau = 0 output, averaged on the device) against the oracle's
    fp64 MSE on the same kept sets, on sampled segments of llama_16k.  Each
    GPU output is within relative RMS 4e-3 of its oracle value, so by the
    triangle inequality in L2 the two root-mean-square differences agree to
    within 2 x 4e-3 x RMS(dense output).  tau = 3e-3, where these segments
    drop a measurable share of their mass (at 1e-3 llama_16k keeps ~99 %)."""
    import bench
    w = synth.WORKLOADS["llama_16k"]
    Q, K, V = synth.generate_workload(w)
    tau = 3e-3
    p = O.Params(tau=tau)
    q, k, v = dev(Q), dev(K), dev(V)
    cfg = s2o.make_config(w.B, w.Hq, w.Hkv, w.N, tau=tau)
    bufs = s2o.plan(cfg, q, k)
    Os = s2o.attention(cfg, q, k, v, bufs["perm"], bufs["nblocks"], out_dtype=s2o.OUT_F32)
    perm, nb, _, _ = host_plan(cfg, bufs)
    cfg0 = s2o.make_config(w.B, w.Hq, w.Hkv, w.N, tau=0.0)
    b0 = s2o.plan(cfg0, q, k)
    Od = s2o.attention(cfg0, q, k, v, b0["perm"], b0["nblocks"], out_dtype=s2o.OUT_F32)
    assert s2o.last_device_error() == 0
    G = w.Hq // w.Hkv
    S = O.num_segments(w.N, p)
    off = O.candidate_offsets(w.N, p)
    kvh = 3
    sse_o = n_o = sq_o = 0.0
    rows = []
    for s in (5, S // 2, S - 1):
        keep = O.keep_set(w.N, s, perm[0, kvh, off[s]:off[s + 1]], int(nb[0, kvh, s]), p)
        e, m = O.mse_segment(Q, K, V, 0, kvh, s, G, keep, p)
        sse_o += e
        n_o += m
        sq_o += float(np.sum(O.dense_segment(Q, K, V, 0, kvh, s, G, p) ** 2))
        rows.append(O.segment_rows(w.N, s, p))
    sl = lambda t: torch.cat([t[0, kvh * G:(kvh + 1) * G, r0:r1] for r0, r1 in rows], dim=1).unsqueeze(0)
    mse_gpu, _ = bench.mse_on_device(torch, sl(Os), sl(Od))
    mse_ora = sse_o / n_o
    assert mse_ora > 1e-6  # the sampled segments drop real mass
    bound = 2 * parity.REL_RMS * np.sqrt(sq_o / n_o)
    assert abs(np.sqrt(mse_gpu) - np.sqrt(mse_ora)) <= bound, (mse_gpu, mse_ora, bound)


# ---------------------------------------------------------------------------
# s2o_plan_filtered: only the prefix of each order the stop rule can reach
# ---------------------------------------------------------------------------

def filtered_matches_full(cfg, q, k, v):
    """Runs both plans and both attentions; the filtered plan's perm buffer
    starts filled with -1, so an attention that read past a segment's kept
    prefix would raise the bad-plan error."""
    full = s2o.plan(cfg, q, k)
    filt = s2o.alloc_plan(cfg, q.device)
    filt["perm"].fill_(-1)
    s2o.plan(cfg, q, k, bufs=filt, filtered=True)
    assert s2o.last_launch_count() >= 6
    assert s2o.last_device_error() == 0
    BH = cfg.B * cfg.Hkv
    S, T = s2o.num_segments(cfg), s2o.num_candidates(cfg)
    assert torch.equal(filt["nblocks"], full["nblocks"])
    assert torch.equal(filt["scores"][:BH * T], full["scores"][:BH * T])
    assert torch.equal(filt["seg_stats"], full["seg_stats"])
    # positions inside each segment's kept prefix, compared on the device
    nb = full["nblocks"].view(BH, S).long()
    off = torch.tensor([s2o.candidate_offset(cfg, s) for s in range(S + 1)], dtype=torch.int64, device=q.device)
    pos = torch.arange(T, dtype=torch.int64, device=q.device)
    seg = torch.searchsorted(off, pos, right=True) - 1
    inside = (pos - off[seg]).unsqueeze(0) < 64 * nb[:, seg]
    pf = filt["perm"][:BH * T].view(BH, T)
    pa = full["perm"][:BH * T].view(BH, T)
    assert torch.equal(pf[inside], pa[inside])
    kept = float(inside.float().mean()) if T else 0.0
    del inside, pos, seg
    out_a = s2o.attention(cfg, q, k, v, full["perm"], full["nblocks"])
    out_f = s2o.attention(cfg, q, k, v, filt["perm"], filt["nblocks"])
    assert s2o.last_device_error() == 0
    assert torch.equal(out_a, out_f)
    return filt, kept


@pytest.mark.parametrize("B,Hq,Hkv,N,tau,planted,band", SMALL)
def test_filtered_plan_small_cases(B, Hq, Hkv, N, tau, planted, band):
    Q, K, V = synth.generate(B, Hq, Hkv, N, 128, planted=planted, band=band, n_stripe=8, seed=3)
    cfg = s2o.make_config(B, Hq, Hkv, N, tau=tau)
    filt, _ = filtered_matches_full(cfg, dev(Q), dev(K), dev(V))
    check_plan(Q, K, cfg, filt, O.Params(tau=tau), what="filtered small", prefix_only=True)


@pytest.mark.parametrize("name", ["tiny_1k", "llama_16k", "llama_128k", "flat_128k"])
def test_filtered_plan_workloads(name):
    w = synth.WORKLOADS[name]
    Q, K, V = synth.generate_workload(w)
    cfg = s2o.make_config(w.B, w.Hq, w.Hkv, w.N, tau=w.tau)
    filt, kept = filtered_matches_full(cfg, dev(Q), dev(K), dev(V))
    p = O.Params(tau=w.tau)
    S = O.num_segments(w.N, p)
    segs = None if S <= 8 else sampled_segments(S)
    check_plan(Q, K, cfg, filt, p, segments=segs, kvheads=[0, w.Hkv - 1], what=f"filtered {name}",
               prefix_only=True)


def test_clustered_scores_take_every_sort_path():
    """Keys drawn from three distinct vectors: each segment's candidate scores
    take three values, each shared by about a third of the candidates.  The
    order is then fixed by the tie rule alone (equal scores, lower index
    first) and both plans must reproduce the oracle's exactly.  The shapes
    reach the sorter's less common paths: where the first tie group holds
    fewer candidates than a bucket's window of 2816 ranks, two distinct values
    share a bucket and crowd its fine bins (the bucket's radix sort); where a
    tie group exceeds a bucket's room of 2816, the segment goes to the
    global-memory sort."""
    N, tau = 16384, 5e-3
    Q, _, V = synth.generate(1, 2, 1, N, 128, planted=False, band=False, n_stripe=8, seed=5)
    rng = np.random.default_rng(11)
    # spread wide enough that the stop rule cuts most segments inside a group
    vecs = synth.to_bf16_bits((32.0 * rng.standard_normal((3, 128))).astype(np.float32))
    K = vecs[rng.integers(0, 3, N)][None, None].copy()
    cfg = s2o.make_config(1, 2, 1, N, tau=tau)
    filt, _ = filtered_matches_full(cfg, dev(Q), dev(K), dev(V))
    full = s2o.plan(cfg, dev(Q), dev(K))
    assert s2o.last_device_error() == 0
    p = O.Params(tau=tau)
    off = O.candidate_offsets(N, p)
    perm_f, nb_f, _, _ = host_plan(cfg, full)
    perm_p, nb_p, _, _ = host_plan(cfg, filt)
    radix = fallback = cut = 0
    for s in range(O.num_segments(N, p)):
        sp = O.plan_segment(Q, K, 0, 0, s, 2, p)
        n = len(sp.order)
        cut += sp.C < len(sp.masses)
        assert np.array_equal(perm_f[0, 0, off[s]:off[s + 1]], sp.order)
        if sp.mass_ties.size == 0:
            assert nb_f[0, 0, s] == sp.C
        head = p.Bk * int(nb_p[0, 0, s])
        assert np.array_equal(perm_p[0, 0, off[s]:off[s] + min(n, head)], sp.order[:head])
        if n:
            lo, hi = O.candidate_range(N, s, p)
            vals, counts = np.unique(-sp.scores[lo:hi], return_counts=True)  # descending score
            assert len(vals) <= 3
            if counts.max() > 2816:
                fallback += 1
            elif len(counts) > 1 and counts[0] < 2816 and min(counts[0], counts[1]) > 64:
                radix += 1
    assert radix >= 20 and fallback >= 20 and cut >= 20, (radix, fallback, cut)


def test_filtered_plan_tau_sweep():
    w = synth.WORKLOADS["sweep_64k"]
    Q, K, V = synth.generate_workload(w)
    q, k, v = dev(Q), dev(K), dev(V)
    for tau in synth.TAU_SWEEP:
        cfg = s2o.make_config(w.B, w.Hq, w.Hkv, w.N, tau=tau)
        filtered_matches_full(cfg, q, k, v)


# ---------------------------------------------------------------------------
# s2o_attention_online: the pages' run-time stop
# ---------------------------------------------------------------------------

def check_online(Q, K, V, cfg, perm_dev, out, cout, p, segments=None, kvheads=None, what=""):
    """Per tile: the oracle's rule on the GPU's own order must stop where the
    GPU stopped, except inside the band of tau; the output must match the
    oracle over the GPU's kept set."""
    G = cfg.Hq // cfg.Hkv
    S = O.num_segments(cfg.N, p)
    off = O.candidate_offsets(cfg.N, p)
    T = int(off[-1])
    perm = perm_dev[:cfg.B * cfg.Hkv * T].cpu().numpy().reshape(cfg.B, cfg.Hkv, T)
    cg = cout.cpu().numpy().reshape(cfg.B, cfg.Hq, S)
    got = out.float().cpu().numpy()
    flips = 0
    for b in range(cfg.B):
        for kvh in (range(cfg.Hkv) if kvheads is None else kvheads):
            for s in (range(S) if segments is None else segments):
                perm_seg = perm[b, kvh, off[s]:off[s + 1]]
                for pair in range(G // 2):
                    heads = O.tile_heads(kvh, G, pair)
                    c_gpu = int(cg[b, heads[0], s])
                    assert c_gpu == int(cg[b, heads[1], s])
                    st = O.online_stop_segment(Q, K, b, kvh, s, heads, perm_seg, p)
                    if c_gpu != st.C:
                        # the blocks where the two stopped must be near-ties of tau
                        lo_c = min(c_gpu, st.C)
                        assert lo_c - 1 in set(int(x) for x in st.near_ties), \
                            f"{what} b={b} kvh={kvh} s={s} pair={pair}: C {c_gpu} != oracle {st.C}"
                        flips += 1
                    keep = O.keep_set(cfg.N, s, perm_seg, c_gpu, p)
                    ref = O.attention_segment(Q, K, V, b, kvh, s, G, keep, p)
                    r0, r1 = O.segment_rows(cfg.N, s, p)
                    g = got[b, heads[0]:heads[-1] + 1, r0:r1]
                    parity.assert_output_close(g, ref[heads[0] - kvh * G:heads[-1] - kvh * G + 1],
                                               f"{what} online b={b} kvh={kvh} s={s} pair={pair}")
    parity.log_near_ties({"case": what, "online": True, "tau": p.tau, "C_flips": flips})
    return cg


ONLINE_SMALL = [c for c in SMALL if (c[1] // c[2]) % 2 == 0]


@pytest.mark.parametrize("B,Hq,Hkv,N,tau,planted,band", ONLINE_SMALL)
def test_online_small_cases(B, Hq, Hkv, N, tau, planted, band):
    Q, K, V = synth.generate(B, Hq, Hkv, N, 128, planted=planted, band=band, n_stripe=8, seed=N + 7)
    cfg = s2o.make_config(B, Hq, Hkv, N, tau=tau)
    q, k, v = dev(Q), dev(K), dev(V)
    bufs = s2o.plan(cfg, q, k)
    out, cout = s2o.attention_online(cfg, q, k, v, bufs["perm"])
    assert s2o.last_launch_count() == 1
    assert s2o.last_device_error() == 0
    check_online(Q, K, V, cfg, bufs["perm"], out, cout, O.Params(tau=tau), what=f"online small N={N}")


def test_online_tau_zero_equals_planned_kernel_with_every_block():
    Q, K, V = synth.generate(1, 8, 2, 1280, 128, planted=True, band=True, n_stripe=8, seed=21)
    cfg = s2o.make_config(1, 8, 2, 1280, tau=0.0)
    q, k, v = dev(Q), dev(K), dev(V)
    bufs = s2o.plan(cfg, q, k)
    out, cout = s2o.attention_online(cfg, q, k, v, bufs["perm"])
    S = s2o.num_segments(cfg)
    cmax = torch.tensor([max(0, 128 * s - 192) // 64 for s in range(S)], dtype=torch.int32)
    assert torch.equal(cout.cpu().view(8, S), cmax.repeat(8, 1))
    ref = s2o.attention(cfg, q, k, v, bufs["perm"], bufs["nblocks"])  # tau = 0 plans every block too
    assert torch.equal(bufs["nblocks"].cpu().view(2, S), cmax.repeat(2, 1))
    assert torch.equal(out, ref)
    assert s2o.last_device_error() == 0


@pytest.mark.parametrize("name", ["llama_16k", "llama_128k"])
def test_online_workloads(name):
    w = synth.WORKLOADS[name]
    Q, K, V = synth.generate_workload(w)
    cfg = s2o.make_config(w.B, w.Hq, w.Hkv, w.N, tau=w.tau)
    q, k, v = dev(Q), dev(K), dev(V)
    bufs = s2o.plan(cfg, q, k)
    out, cout = s2o.attention_online(cfg, q, k, v, bufs["perm"])
    assert s2o.last_device_error() == 0
    p = O.Params(tau=w.tau)
    S = O.num_segments(w.N, p)
    segs = sampled_segments(S)[::2] if w.N > 20000 else sampled_segments(S)
    check_online(Q, K, V, cfg, bufs["perm"], out, cout, p, segments=segs, kvheads=[0, w.Hkv - 1],
                 what=f"online {name}")


# ---------------------------------------------------------------------------
# s2o_block_truth: ranking accuracy of the pooled order
# ---------------------------------------------------------------------------

def check_truth(Q, K, q, k, cfg, bufs, segs, p, kvheads=None, what=""):
    stats, mass = s2o.block_truth(cfg, q, k, bufs["perm"], bufs["nblocks"], segs)
    assert s2o.last_launch_count() == 2
    assert s2o.last_device_error() == 0
    perm, nb, _, _ = host_plan(cfg, bufs)
    G = cfg.Hq // cfg.Hkv
    off = O.candidate_offsets(cfg.N, p)
    st = stats.cpu().numpy()
    ms = mass.cpu().numpy()
    for k, s in enumerate(segs):
        for b in range(cfg.B):
            for kvh in (range(cfg.Hkv) if kvheads is None else kvheads):
                bk = b * cfg.Hkv + kvh
                bt = O.true_block_masses(Q, K, b, kvh, s, G, perm[b, kvh, off[s]:off[s + 1]], int(nb[b, kvh, s]), p)
                n = len(bt.mass)
                assert np.allclose(ms[k, bk, :n], bt.mass, rtol=2e-4, atol=1e-9), f"{what} s={s} bk={bk}"
                assert int(st[k, bk, 0]) == bt.kept
                # counts may differ only by blocks whose true mass is within 1e-3 of tau
                close = int(np.sum(np.abs(bt.mass - p.tau) <= 1e-3 * p.tau))
                assert abs(int(st[k, bk, 1]) - bt.true) <= close
                assert abs(int(st[k, bk, 2]) - bt.both) <= close
                assert st[k, bk, 3] == pytest.approx(bt.captured, rel=2e-4, abs=1e-9)
                assert st[k, bk, 4] == pytest.approx(bt.total, rel=2e-4, abs=1e-9)


@pytest.mark.parametrize("B,Hq,Hkv,N,tau,planted,band", [c for c in SMALL if c[3] >= 640][:4])
def test_block_truth_small_cases(B, Hq, Hkv, N, tau, planted, band):
    Q, K, V = synth.generate(B, Hq, Hkv, N, 128, planted=planted, band=band, n_stripe=8, seed=N + 3)
    cfg = s2o.make_config(B, Hq, Hkv, N, tau=tau)
    q, k = dev(Q), dev(K)
    bufs = s2o.plan(cfg, q, k)
    S = O.num_segments(N, O.Params(tau=tau))
    check_truth(Q, K, q, k, cfg, bufs, list(range(S)), O.Params(tau=tau), what=f"truth N={N}")


@pytest.mark.parametrize("name", ["llama_16k", "llama_128k"])
def test_block_truth_workloads(name):
    w = synth.WORKLOADS[name]
    Q, K, V = synth.generate_workload(w)
    cfg = s2o.make_config(w.B, w.Hq, w.Hkv, w.N, tau=w.tau)
    q, k = dev(Q), dev(K)
    bufs = s2o.plan(cfg, q, k)
    S = s2o.num_segments(cfg)
    segs = [2, S // 3, S - 1] if w.N > 20000 else [2, 5, S // 2, S - 1]
    check_truth(Q, K, q, k, cfg, bufs, segs, O.Params(tau=w.tau), kvheads=[0, w.Hkv - 1], what=name)


# ---------------------------------------------------------------------------
# Q_perm: two query sub-segments per segment
# ---------------------------------------------------------------------------

def check_qperm(Q, K, V, cfg, qp, out, segments=None, kvheads=None, what=""):
    p = O.Params(tau=cfg.tau)
    G = cfg.Hq // cfg.Hkv
    BH = cfg.B * cfg.Hkv
    S, T = s2o.num_segments(cfg), s2o.num_candidates(cfg)
    off = O.candidate_offsets(cfg.N, p)
    perm = qp["perm"][:2 * BH * T].cpu().numpy().reshape(2, cfg.B, cfg.Hkv, T)
    nb = qp["nblocks"].cpu().numpy().reshape(2, cfg.B, cfg.Hkv, S)
    rs = qp["rowsub"].cpu().numpy().reshape(cfg.B, cfg.Hkv, S, 128)
    got = out.float().cpu().numpy()
    swaps = flips = moved = 0
    for b in range(cfg.B):
        for kvh in (range(cfg.Hkv) if kvheads is None else kvheads):
            for s in (range(S) if segments is None else segments):
                sp = O.qperm_segment(Q, K, b, kvh, s, G, p)
                r0, r1 = O.segment_rows(cfg.N, s, p)
                gsub = rs[b, kvh, s, :r1 - r0].astype(np.int64)
                if not np.array_equal(gsub, sp.sub_of_row):
                    # only rows tied in importance with the boundary may move
                    order = np.sort(sp.imp)[::-1]
                    cut = order[min(64, r1 - r0) - 1]
                    diff = np.nonzero(gsub != sp.sub_of_row)[0]
                    assert np.all(np.abs(sp.imp[diff] - cut) <= 1e-12 * np.max(np.abs(sp.imp))), f"{what} s={s}"
                    moved += len(diff)
                    continue  # the sub-segment plans then differ legitimately
                for sub in (0, 1):
                    sw, fl = parity.compare_segment_plan(perm[sub, b, kvh, off[s]:off[s + 1]], int(nb[sub, b, kvh, s]),
                                                         sp.plans[sub], p, prefix_only=True)
                    swaps += sw
                    flips += fl
                keeps = [O.keep_set(cfg.N, s, perm[sub, b, kvh, off[s]:off[s + 1]], int(nb[sub, b, kvh, s]), p)
                         for sub in (0, 1)]
                ref = O.attention_qperm_segment(Q, K, V, b, kvh, s, G, keeps, gsub, p)
                parity.assert_output_close(got[b, kvh * G:(kvh + 1) * G, r0:r1], ref, f"{what} b={b} kvh={kvh} s={s}")
    parity.log_near_ties({"case": what, "qperm": True, "swapped_positions": swaps, "C_flips": flips,
                          "rows_moved": moved})


@pytest.mark.parametrize("B,Hq,Hkv,N,tau,planted,band", ONLINE_SMALL)
def test_qperm_small_cases(B, Hq, Hkv, N, tau, planted, band):
    Q, K, V = synth.generate(B, Hq, Hkv, N, 128, planted=planted, band=band, n_stripe=8, seed=N + 11)
    cfg = s2o.make_config(B, Hq, Hkv, N, tau=tau)
    q, k, v = dev(Q), dev(K), dev(V)
    qp = s2o.plan_qperm(cfg, q, k)
    assert s2o.last_launch_count() >= 12
    out = s2o.attention_qperm(cfg, q, k, v, qp)
    assert s2o.last_launch_count() == 1
    assert s2o.last_device_error() == 0
    check_qperm(Q, K, V, cfg, qp, out, what=f"qperm small N={N}")


@pytest.mark.parametrize("B,Hq,Hkv,N,tau", [(1, 16, 2, 1280, 3e-3), (2, 8, 1, 1000, 1e-2)])
def test_qperm_two_head_quads_per_segment(B, Hq, Hkv, N, tau):
    # group size 8: each segment's rows go to two CTAs per sub-segment (heads
    # 0-3 and 4-7); the second case also has a ragged last segment whose
    # second sub-segment is short
    Q, K, V = synth.generate(B, Hq, Hkv, N, 128, planted=True, band=True, n_stripe=8, seed=N + 13)
    cfg = s2o.make_config(B, Hq, Hkv, N, tau=tau)
    q, k, v = dev(Q), dev(K), dev(V)
    qp = s2o.plan_qperm(cfg, q, k)
    out = s2o.attention_qperm(cfg, q, k, v, qp)
    assert s2o.last_device_error() == 0
    check_qperm(Q, K, V, cfg, qp, out, what=f"qperm G={Hq // Hkv} N={N}")


def test_qperm_identical_rows_equal_the_plain_path():
    # every row of a segment equal in every head: both sub-segments pool to
    # the segment's query, so plans and output equal the plain method's
    rng = np.random.default_rng(31)
    B, Hq, Hkv, N = 1, 4, 2, 1024
    base = rng.standard_normal((B, Hq, N // 128, 1, 128)).astype(np.float32)
    Q = synth.to_bf16_bits(np.repeat(base, 128, axis=3).reshape(B, Hq, N, 128))
    _, K, V = synth.generate(B, Hq, Hkv, N, 128, planted=True, band=True, n_stripe=8, seed=31)
    cfg = s2o.make_config(B, Hq, Hkv, N, tau=3e-3)
    q, k, v = dev(Q), dev(K), dev(V)
    qp = s2o.plan_qperm(cfg, q, k)
    out = s2o.attention_qperm(cfg, q, k, v, qp)
    bufs = s2o.plan(cfg, q, k)
    ref = s2o.attention(cfg, q, k, v, bufs["perm"], bufs["nblocks"])
    assert s2o.last_device_error() == 0
    S = s2o.num_segments(cfg)
    nb = qp["nblocks"].view(2, -1)
    assert torch.equal(nb[0], bufs["nblocks"]) and torch.equal(nb[1], bufs["nblocks"])
    assert torch.equal(out, ref)


@pytest.mark.parametrize("name", ["llama_16k", "llama_128k"])
def test_qperm_workloads(name):
    w = synth.WORKLOADS[name]
    Q, K, V = synth.generate_workload(w)
    cfg = s2o.make_config(w.B, w.Hq, w.Hkv, w.N, tau=w.tau)
    q, k, v = dev(Q), dev(K), dev(V)
    qp = s2o.plan_qperm(cfg, q, k)
    out = s2o.attention_qperm(cfg, q, k, v, qp)
    assert s2o.last_device_error() == 0
    S = s2o.num_segments(cfg)
    segs = sampled_segments(S)[::2] if w.N > 20000 else sampled_segments(S)
    check_qperm(Q, K, V, cfg, qp, out, segments=segs, kvheads=[0, w.Hkv - 1], what=f"qperm {name}")
