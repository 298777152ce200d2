"""Benchmark of the S2O sparse-prefill hot path on B200.

One step = s2o_plan (pool, score, sort, stop) + s2o_attention over one
synthetic 128K-token Llama-3.1-8B-shaped layer (GQA 32/8, d = 128, bf16,
sinks + 0.5% stripes + local band, tau = 1e-3), inputs resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Prints one JSON line (rank 0).  `value` is dense-equivalent causal attention
TFLOP/s (4 * B * Hq * N^2 * d / 2 FLOP per step, the dense work the sparse
path stands in for) over the whole step (plan + attention), summed over
ranks; each rank runs an independent problem (weak scaling, no collective
on the data path).  `--impl reference` times the fp64 CPU oracle instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "dense-equiv attention TFLOP/s at 128K (GQA 32/8, d128); tensor-pipe % of peak"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def dense_flops(B, Hq, N, d):
    # QK^T and PV over the causal half: 2 matmuls x 2 flop x B Hq N^2 d / 2
    return 2.0 * B * Hq * float(N) * float(N) * d


def kept_pairs(nblocks: np.ndarray, N: int, G: int) -> int:
    """Sum over heads and rows of |Keep(s) cap [0, i]| for the compiled constants.

    Per segment s with rows [128 s, 128 s + L):
      s = 0: causal only            -> sum_i (i + 1)
      s = 1: keys [0, 128) + causal -> L * 128 + L (L + 1) / 2
      s >= 2: sinks 64 + previous window 128 + 64 C(s) kept candidates + causal
    """
    B, Hkv, S = nblocks.shape
    total = 0
    for s in range(S):
        r0 = 128 * s
        L = min(N, r0 + 128) - r0
        diag = L * (L + 1) // 2
        if s == 0:
            per = np.full((B, Hkv), diag, dtype=np.int64)
        elif s == 1:
            per = np.full((B, Hkv), L * 128 + diag, dtype=np.int64)
        else:
            per = L * (64 + 128 + 64 * nblocks[:, :, s].astype(np.int64)) + diag
        total += int(per.sum()) * G
    return total


def kept_pairs_qperm(nblocks2: np.ndarray, rowsub: np.ndarray, N: int, G: int) -> int:
    """kept_pairs for Q_perm: nblocks2 [2, B, Hkv, S]; rowsub [B, Hkv, S, 128]
    gives each row's sub-segment, whose C(s) counts for that row."""
    _, B, Hkv, S = nblocks2.shape
    total = 0
    for s in range(S):
        r0 = 128 * s
        L = min(N, r0 + 128) - r0
        diag = L * (L + 1) // 2
        if s == 0:
            per = np.full((B, Hkv), diag, dtype=np.int64)
        elif s == 1:
            per = np.full((B, Hkv), L * 128 + diag, dtype=np.int64)
        else:
            n1 = rowsub[:, :, s, :L].astype(np.int64).sum(axis=-1)
            n0 = L - n1
            per = L * (64 + 128) + diag + 64 * (n0 * nblocks2[0, :, :, s] + n1 * nblocks2[1, :, :, s])
        total += int(per.sum()) * G
    return total


# DRAM bytes (read + write) per k_sparse_attn2 launch from an ncu capture of
# the current kernel, by workload.  llama_128k: the capture of llama_32k at
# the same kept fraction (tau = 4e-3, 26.7 % of pairs; 436.8 + 232.7 MB)
# scaled by the rows processed (x 4: Q, O, K and V all grow with N).  None
# where no capture exists.
ATTN_TRAFFIC = {"llama_128k": 2.678e9, "llama_32k@0.004": 6.695e8}

# int8 tensor-core rate relative to the measured bf16 rate: the nominal dense
# ratio of B200 (4.5 POPS int8 / 2.25 PFLOP/s bf16)
I8_OVER_BF16 = 2.0
# digit products per (segment, admissible key) pair of the integer scorer:
# 11 products of 128 int8 multiply-adds
I8_MACS_PER_PAIR = 11 * 128


def prefix_lengths(torch, cfg, bufs, filtered: bool, w):
    """Entries of each segment's order the plan sorts: all candidates for the
    full plan; for the filtered plan whole blocks up to the number of
    candidates with s >= M + ln(tau Z / Bk) - 1e-3 (the bound the planner
    uses).  Returns the total over every (b, kvh, s)."""
    B, Hkv = w.B, w.Hkv
    S = (w.N + 127) // 128
    T = (64 * (S - 2) ** 2) if S >= 2 else 0
    if not filtered or w.tau <= 0.0:
        return B * Hkv * T
    cnt = torch.tensor([max(0, 128 * s - 192) for s in range(S)], dtype=torch.int64, device=bufs["scores"].device)
    seg = torch.repeat_interleave(torch.arange(S, device=cnt.device), cnt)
    stats = bufs["seg_stats"].view(B * Hkv, S, 2).double()
    total = 0
    for u in range(B * Hkv):
        thr = stats[u, :, 0] + torch.log(w.tau * stats[u, :, 1] / 64.0) - 1e-3
        sc = bufs["scores"][u * T:(u + 1) * T].double()
        nhi = torch.zeros(S, dtype=torch.int64, device=cnt.device).index_add_(0, seg, (sc >= thr[seg]).long())
        total += int(torch.minimum(cnt, 64 * ((nhi + 63) // 64)).sum())
    return total


def plan_kernel_roofline(s2o, torch, cfg, Q, K, bufs, filtered, w, peaks, peak_src, reps=3):
    """Median device time of each plan kernel over `reps` plans (events on the
    caller's stream between the kernels), and its compulsory HBM bytes:
      k_pool       read Q, write the fp64 pooled queries
      k_kdig       read K, write its three 8-bit digit planes and row exponents
      k_qdig       read the pooled queries, write their four digit planes
      k_score8     read the key and query digits once, write the candidate
                   scores and the causal half of the (max, sumexp) partials;
                   also its int8 multiply-adds (11 x 128 per admissible key
                   per segment) against the int8 tensor peak
      k_seg_stats  read the partials, write (M, Z)
      k_bucket_plan read every candidate score, write the staged (key, index)
                   pairs of the sorted prefix
      k_bucket_sort read the staged pairs, write perm and the sorted scores
      k_mass_stop  read the sorted scores of the prefix, write C(s)
    (the prefix is every candidate for the full plan)."""
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    S = (N + 127) // 128
    T = B * Hkv * ((64 * (S - 2) ** 2) if S >= 2 else 0)
    L = prefix_lengths(torch, cfg, bufs, filtered, w)
    # (max, sum exp) partials: one per (segment, 96-key tile holding admissible keys)
    parts = B * Hkv * sum((min(N, 128 * (s + 1)) + 95) // 96 for s in range(S)) * 8
    ntiles = (N + 95) // 96
    kdig = B * Hkv * ntiles * (3 * 96 * 128 + 100 * 4)
    qdig = B * Hkv * (((S + 127) // 128) * 128 * 4 * 128 + S * 4)
    bytes_of = {
        "k_pool": B * Hq * N * d * 2 + B * Hkv * S * d * 8,
        "k_kdig": B * Hkv * N * d * 2 + kdig,
        "k_qdig": B * Hkv * S * d * 8 + qdig,
        "k_score8": kdig + qdig + T * 4 + parts,
        "k_seg_stats": parts + B * Hkv * S * 16,
        "k_bucket_plan": T * 4 + L * 8,
        "k_bucket_sort": L * 8 + L * 8,
        "k_mass_stop": L * 4 + B * Hkv * S * 4,
    }
    # admissible keys of every segment: e(s) = min(N, 128 (s + 1))
    i8_macs = B * Hkv * I8_MACS_PER_PAIR * sum(min(N, 128 * (s + 1)) for s in range(S))
    i8_peak = float(peaks["bf16_tflops"]) * 1e12 * I8_OVER_BF16 / 2  # multiply-adds per second
    s2o.stage_timing(True)
    try:
        runs = []
        for _ in range(reps):
            s2o.plan(cfg, Q, K, bufs, filtered=filtered)
            runs.append(s2o.last_stage_times())
    finally:
        s2o.stage_timing(False)
    hbm = float(peaks["hbm_gbs"])
    out = {"plan": "filtered" if filtered else "full", "sorted_prefix_entries": L, "candidates": T,
           "peak_hbm_gbs": hbm, "peak_source": f"{peak_src} HBM copy", "kernels": {}}
    names = [n for n, _ in runs[0]]
    total_ms, total_bytes = 0.0, 0.0
    for i, name in enumerate(names):
        ms = float(np.median([r[i][1] for r in runs]))
        total_ms += ms
        ent = {"ms": ms}
        if name in bytes_of:
            b = float(bytes_of[name])
            total_bytes += b
            ent.update(bytes=b, gbs=b / (ms * 1e-3) / 1e9, frac_hbm=b / (ms * 1e-3) / 1e9 / hbm)
        if name == "k_score8":
            ent.update(i8_macs=float(i8_macs), i8_tops=2 * i8_macs / (ms * 1e-3) / 1e12,
                       frac_i8=i8_macs / (ms * 1e-3) / i8_peak,
                       note="int8 peak = measured bf16 burst x 2 (nominal dense ratio)")
        out["kernels"][name] = ent
    out["total_ms"] = total_ms
    out["total_bytes"] = total_bytes
    out["total_gbs"] = total_bytes / (total_ms * 1e-3) / 1e9
    out["total_frac_hbm"] = out["total_gbs"] / hbm
    return out


def reduce_max_ms(ms: float, dist=None, device="cpu") -> float:
    """Max over ranks of a per-rank time (the slowest rank bounds the job)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(ms)
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def kv_head_slice(Hkv: int, world: int, rank: int) -> tuple[int, int]:
    """KV heads [k0, k1) of one rank when a single problem is sharded by KV
    head: each rank plans and attends its KV heads and their groups' query
    heads alone (a KV group's plan and attention depend on nothing else, so
    no data crosses ranks).  Contiguous shares; the first Hkv % world ranks
    take one head more."""
    if not 1 <= world <= Hkv or not 0 <= rank < world:
        raise ValueError("KV-head sharding needs 1 <= world <= Hkv")
    base, extra = divmod(Hkv, world)
    k0 = rank * base + min(rank, extra)
    return k0, k0 + base + (1 if rank < extra else 0)


def shard_inputs(Q, K, V, world: int, rank: int):
    """This rank's Q, K, V (numpy bf16 bits) under kv_head_slice."""
    G = Q.shape[1] // K.shape[1]
    k0, k1 = kv_head_slice(K.shape[1], world, rank)
    c = np.ascontiguousarray
    return c(Q[:, k0 * G:k1 * G]), c(K[:, k0:k1]), c(V[:, k0:k1])


def whole_job_tflops(world: int, flops_per_rank: float, ms: float) -> float:
    """Every rank solves its own problem: the job's throughput is all ranks'
    work over the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return PEAKS_FALLBACK, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None

    def __enter__(self):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.file.flush()

    def summary(self):
        try:
            rows = [l.split(",") for l in open(self.file.name).read().strip().splitlines()]
            os.unlink(self.file.name)
        except OSError:
            return None
        rows = [[x.strip() for x in r] for r in rows if len(r) >= 7]
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[3 + k].lower() == "active"})
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def cpu_oracle_sample(Q, K, V, tau, seconds=15.0):
    """Oracle (fp64, one thread) on sampled segments, KV head by KV head: plan +
    attention of every query head of the group, until `seconds` have passed.
    Returns (dense-equivalent TFLOP/s of the rows done, sample text, seconds)."""
    from threadpoolctl import threadpool_limits
    from oracle import s2o_oracle as O

    p = O.Params(tau=tau)
    N, d = Q.shape[2], Q.shape[3]
    G = Q.shape[1] // K.shape[1]
    S = O.num_segments(N, p)
    order = sorted({S - 1, S // 2, S // 4, 3 * S // 4, 3, 2, 1, 0} | set(range(S - 2, 3, -97)))
    done, flops, t0 = [], 0.0, time.perf_counter()
    with threadpool_limits(1):
        for kvh in range(K.shape[1]):
            for s in order:
                sp = O.plan_segment(Q, K, 0, kvh, s, G, p)
                O.attention_segment(Q, K, V, 0, kvh, s, G, sp.keep, p)
                r0, r1 = O.segment_rows(N, s, p)
                rows = np.arange(r0, r1, dtype=np.float64)
                flops += G * 4.0 * d * float(np.sum(rows + 1))  # dense-equivalent work of these rows
                done.append((kvh, s))
                if time.perf_counter() - t0 > seconds:
                    break
            if time.perf_counter() - t0 > seconds:
                break
    dt = time.perf_counter() - t0
    heads = sorted({h for h, _ in done})
    sample = (f"oracle plan+attention of {len(done)} (KV head, segment) items, KV heads {heads}, segments "
              f"{order} (all {G} query heads of each group) of the {N}-token workload; fp64, 1 thread; "
              f"{dt:.1f} s")
    return flops / dt / 1e12, sample, dt


_FORK = {}  # arrays the all-cores oracle workers inherit (fork, before any CUDA call)


def _oracle_item(item):
    """One (KV head, segment) of the oracle: plan + attention of every query
    head of the group; returns its dense-equivalent FLOPs."""
    from oracle import s2o_oracle as O
    kvh, s = item
    Q, K, V, p = _FORK["Q"], _FORK["K"], _FORK["V"], _FORK["p"]
    N, d = Q.shape[2], Q.shape[3]
    G = Q.shape[1] // K.shape[1]
    sp = O.plan_segment(Q, K, 0, kvh, s, G, p)
    O.attention_segment(Q, K, V, 0, kvh, s, G, sp.keep, p)
    r0, r1 = O.segment_rows(N, s, p)
    return G * 4.0 * d * float(np.sum(np.arange(r0, r1, dtype=np.float64) + 1))


def _one_blas_thread():
    from threadpoolctl import threadpool_limits
    _FORK["limit"] = threadpool_limits(1)


def host_cores():
    """(logical CPUs of the host, CPUs this process may run on)."""
    try:
        aff = len(os.sched_getaffinity(0))
    except AttributeError:
        aff = os.cpu_count() or 1
    return os.cpu_count() or 1, aff


def cpu_oracle_all_cores(Q, K, V, tau, seconds=15.0, max_procs=64):
    """The same oracle items as cpu_oracle_sample, spread over one process per
    available core (at most max_procs, to bound host memory: each item widens
    up to 3 x 134 MB of K/V rows to fp64), one BLAS thread each.  Uses a fork
    pool, so it must run before the process touches CUDA.  Returns
    (dense-equivalent TFLOP/s, processes, sample text)."""
    import multiprocessing as mp
    from oracle import s2o_oracle as O

    p = O.Params(tau=tau)
    N = Q.shape[2]
    S = O.num_segments(N, p)
    order = sorted({S - 1, S // 2, S // 4, 3 * S // 4, 3, 2, 1, 0} | set(range(S - 2, 3, -97)))
    items = [(kvh, s) for s in order for kvh in range(K.shape[1])]
    procs = max(1, min(max_procs, host_cores()[1]))
    _FORK.update(Q=Q, K=K, V=V, p=p)
    flops, done = 0.0, 0
    ctx = mp.get_context("fork")
    pool = ctx.Pool(procs, initializer=_one_blas_thread)
    try:
        t0 = time.perf_counter()
        for f in pool.imap_unordered(_oracle_item, items * 64, chunksize=1):
            flops += f
            done += 1
            if time.perf_counter() - t0 > seconds:
                break
        dt = time.perf_counter() - t0
    finally:
        pool.terminate()
        pool.join()
        _FORK.clear()
    sample = (f"{done} (KV head, segment) items of the same segment list over all KV heads, {procs} processes "
              f"x 1 BLAS thread, {dt:.1f} s wall; items still running at the cut are not counted")
    return flops / dt / 1e12, procs, sample


def cpu_baseline_entry(Qn, Kn, Vn, tau):
    v1, sample, _ = cpu_oracle_sample(Qn, Kn, Vn, tau, seconds=15.0)
    vall, procs, sample_all = cpu_oracle_all_cores(Qn, Kn, Vn, tau, seconds=15.0)
    ncpu, naff = host_cores()
    return {"value": v1, "unit": "TFLOP/s", "cores": 1, "threads": 1, "kind": "oracle", "sample": sample,
            "host_cores": ncpu, "affinity_cores": naff,
            "value_all_cores": vall, "all_cores_processes": procs, "all_cores_sample": sample_all}


def bench_config(w, world: int, plan: str, shard: bool = False) -> dict:
    """The workload description both arms print (Hq, Hkv: one rank's share
    when the problem is sharded by KV head)."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "tau": w.tau,
            "global_batch": w.B if shard else w.B * world, "seq_len": w.N,
            "parallelism": f"kv-head shards x{world}" if shard else f"independent x{world}",
            "l2": "inputs larger than L2 (Q alone is 1 GiB)" if w.N >= 131072 else "inputs per step exceed L2",
            "plan": plan}


def reference_arm(args, w, world, rank):
    """The CPU oracle as the reference implementation, rank 0 only."""
    if rank != 0:
        return
    from score_keys_pooled_b200 import synth
    Q, K, V = synth.generate_workload(w, seed=0)
    budget = max(2.0, 150.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_oracle_sample(Q, K, V, w.tau, seconds=min(2.0, budget))
    vals, total = [], 0.0
    for _ in range(args.steps):
        v, sample, dt = cpu_oracle_sample(Q, K, V, w.tau, seconds=budget)
        vals.append(v)
        total += dt
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * total / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w, world, args.plan),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "threads": 1, "kind": "oracle",
                         "sample": sample, "host_cores": host_cores()[0], "affinity_cores": host_cores()[1]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _median_ms(torch, fn, reps=3, warm=2):
    for _ in range(warm):
        fn()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for e0, e1 in ev:
        e0.record()
        fn()
        e1.record()
    torch.cuda.synchronize()
    return float(np.median([e0.elapsed_time(e1) for e0, e1 in ev]))


def mse_on_device(torch, Os, Od):
    """Mean over every output element of (Os - Od)^2, in fp64, head by head;
    also the mean of Od^2 (to give the relative figure)."""
    sse = sq = 0.0
    for b in range(Os.shape[0]):
        for h in range(Os.shape[1]):
            dd = Od[b, h].double()
            diff = Os[b, h].double() - dd
            sse += float((diff * diff).sum())
            sq += float((dd * dd).sum())
    n = Os.numel()
    return sse / n, sq / n


def c_histogram(nb: np.ndarray, N: int):
    """Per-segment kept fraction C(s) / n_blk(s) over the segments that have
    candidates, binned; and where, per KV head, the first segment that does
    not keep every block lies."""
    S = nb.shape[-1]
    nblk = np.array([max(0, 128 * s - 192) // 64 for s in range(S)])
    segs = np.nonzero(nblk > 0)[0]
    frac = nb[..., segs] / nblk[segs]
    edges = [0.0, 1e-9, 0.1, 0.2, 0.3, 0.4, 0.5, 0.6, 0.7, 0.8, 0.9, 1.0 - 1e-9, 1.0 + 1e-9]
    labels = ["0", "(0,0.1]", "(0.1,0.2]", "(0.2,0.3]", "(0.3,0.4]", "(0.4,0.5]", "(0.5,0.6]", "(0.6,0.7]",
              "(0.7,0.8]", "(0.8,0.9]", "(0.9,1)", "1"]
    counts, _ = np.histogram(frac.ravel(), bins=edges)
    first_cut = []
    for row in frac.reshape(-1, len(segs)):
        cut = np.nonzero(row < 1.0)[0]
        first_cut.append(int(segs[cut[0]]) if cut.size else S)
    ranges = []
    step = max(1, S // 16)
    for a in range(0, S, step):
        sel = (segs >= a) & (segs < a + step)
        if sel.any():
            ranges.append({"segments": [a, min(S, a + step) - 1], "mean_kept_fraction": float(frac[..., sel].mean()),
                           "key_positions": [128 * a, 128 * min(S, a + step)]})
    return {"bins": dict(zip(labels, [int(c) for c in counts])), "segments_with_candidates": int(frac.size),
            "first_segment_not_keeping_all_blocks": {"median": float(np.median(first_cut)),
                                                     "min": int(min(first_cut)), "max": int(max(first_cut))},
            "by_position": ranges}


def report_main(args):
    """Accuracy and per-configuration report (not the headline benchmark):
    one JSON line per configuration with sparsity, MSE against dense causal
    attention, plan and attention time; the tau sweep with the contiguous
    block comparator at the same per-segment block count; the C(s) histogram
    of the flat workload.  MSE is measured on the library's fp32 outputs: the
    plan's sparse output against its tau = 0 output (which keeps every
    admissible key, i.e. dense causal attention)."""
    import torch
    import score_keys_pooled_b200 as s2o
    from score_keys_pooled_b200 import synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    what = args.report
    names = {"configs": ["tiny_1k", "llama_16k", "llama_128k", "sweep_64k", "flat_128k"],
             "sweep": ["sweep_64k"]}[what]
    for name in names:
        w = synth.WORKLOADS[name]
        Qn, Kn, Vn = synth.generate_workload(w, seed=0)
        to_dev = lambda a: torch.from_numpy(a.view(np.int16)).to(dev)
        Q, K, V = to_dev(Qn), to_dev(Kn), to_dev(Vn)
        del Qn, Kn, Vn
        G = w.Hq // w.Hkv
        dense = dense_flops(w.B, w.Hq, w.N, w.d)
        pairs_dense = w.B * w.Hq * w.N * (w.N + 1) / 2.0
        taus = synth.TAU_SWEEP if what == "sweep" else (w.tau,)
        # dense causal attention: tau = 0 keeps every block
        cfg0 = s2o.make_config(w.B, w.Hq, w.Hkv, w.N, tau=0.0)
        bufs = s2o.alloc_plan(cfg0, dev)
        s2o.plan(cfg0, Q, K, bufs)
        Od = s2o.attention(cfg0, Q, K, V, bufs["perm"], bufs["nblocks"], out_dtype=s2o.OUT_F32)
        dense_ms = _median_ms(torch, lambda: s2o.attention(cfg0, Q, K, V, bufs["perm"], bufs["nblocks"], out_dtype=s2o.OUT_F32))
        Os = torch.empty_like(Od)
        for tau in taus:
            cfg = s2o.make_config(w.B, w.Hq, w.Hkv, w.N, tau=tau)
            plan_ms = _median_ms(torch, lambda: s2o.plan(cfg, Q, K, bufs, filtered=True))
            full_ms = _median_ms(torch, lambda: s2o.plan(cfg, Q, K, bufs, filtered=False), reps=2, warm=1)
            s2o.plan(cfg, Q, K, bufs, filtered=False)
            attn_ms = _median_ms(torch, lambda: s2o.attention(cfg, Q, K, V, bufs["perm"], bufs["nblocks"], Os, out_dtype=s2o.OUT_F32))
            if s2o.last_device_error() != 0:
                raise RuntimeError(f"device error in the report ({name}, tau={tau})")
            nb = bufs["nblocks"].cpu().numpy().reshape(w.B, w.Hkv, -1)
            density = kept_pairs(nb, w.N, G) / pairs_dense
            mse, msq = mse_on_device(torch, Os, Od)
            line = {"report": what, "workload": name, "tau": tau, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N,
                    "kept_pair_fraction": density, "sparsity": 1.0 - density,
                    "mse_vs_dense": mse, "relative_mse": mse / msq if msq else None,
                    "plan_filtered_ms": plan_ms, "plan_full_ms": full_ms, "attention_ms": attn_ms,
                    "dense_attention_ms": dense_ms, "step_tflops_dense_equiv": dense / ((plan_ms + attn_ms) * 1e-3) / 1e12,
                    "attention_speedup_vs_dense_kernel": dense_ms / attn_ms}
            if what == "sweep" or name == "sweep_64k":
                # contiguous top-k: original-order blocks by pooled mass, the same C(s) per segment
                pc = torch.empty_like(bufs["perm"])
                s2o.plan_contiguous(cfg, bufs["scores"], bufs["seg_stats"], bufs["nblocks"], pc)
                Oc = s2o.attention(cfg, Q, K, V, pc, bufs["nblocks"], out_dtype=s2o.OUT_F32)
                if s2o.last_device_error() != 0:
                    raise RuntimeError("device error in the contiguous comparator")
                msec, _ = mse_on_device(torch, Oc, Od)
                line.update(contiguous_mse_vs_dense=msec,
                            contiguous_over_s2o_mse=(msec / mse) if mse > 0 else None)
                del Oc, pc
            if name == "flat_128k" or what == "configs":
                line["C_histogram"] = c_histogram(nb, w.N)
            print(json.dumps(line), flush=True)
        del bufs, Od, Os, Q, K, V
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama_128k")
    ap.add_argument("--impl", default="s2o", choices=["s2o", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--online-steps", type=int, default=3,
                    help="steps of the run-time stop variant (full plan + s2o_attention_online), reported beside "
                         "the headline; 0 skips it")
    ap.add_argument("--graph", action=argparse.BooleanOptionalAction, default=False,
                    help="replay the timed step's plan and attention as CUDA graphs instead of launching them")
    ap.add_argument("--plan", default="filtered", choices=["full", "filtered"],
                    help="s2o_plan (every segment fully ordered) or s2o_plan_filtered (only the prefix the "
                         "stop rule can reach; same kept sets and output)")
    ap.add_argument("--shard", default="none", choices=["none", "heads"],
                    help="none: every rank solves its own problem (weak scaling); heads: the ranks share one "
                         "problem, each taking a contiguous share of its KV heads (strong scaling, no data "
                         "exchange)")
    ap.add_argument("--tau", type=float, default=None,
                    help="override the workload's tau (e.g. to profile a small workload at the headline's density)")
    ap.add_argument("--report", default=None, choices=["configs", "sweep"],
                    help="instead of the benchmark line, print one accuracy/timing line per configuration "
                         "(configs) or per tau of the sweep workload with the contiguous comparator (sweep)")
    args = ap.parse_args()
    if args.report:
        report_main(args)
        return
    if args.warmup < 3 and args.impl == "s2o":
        ap.error("--warmup must be >= 3")

    from score_keys_pooled_b200 import synth
    w = synth.WORKLOADS[args.workload]
    if args.tau is not None:
        import dataclasses
        w = dataclasses.replace(w, tau=args.tau)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        reference_arm(args, w, world, rank)
        return

    # each rank solves an independent problem (its own seed): weak scaling;
    # or (--shard heads) its share of the KV heads of one problem: strong
    shard = args.shard == "heads" and world > 1
    dense_full = dense_flops(w.B, w.Hq, w.N, w.d)
    Qn, Kn, Vn = synth.generate_workload(w, seed=0 if shard else rank)
    if shard:
        import dataclasses
        Qn, Kn, Vn = shard_inputs(Qn, Kn, Vn, world, rank)
        w = dataclasses.replace(w, Hq=Qn.shape[1], Hkv=Kn.shape[1])

    # the CPU baseline forks its worker pool, so it runs before any CUDA call
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_entry(Qn, Kn, Vn, w.tau)

    import torch
    import score_keys_pooled_b200 as s2o

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)

    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).to(dev)
    Q, K, V = to_dev(Qn), to_dev(Kn), to_dev(Vn)
    cfg = s2o.make_config(w.B, w.Hq, w.Hkv, w.N, tau=w.tau)
    bufs = s2o.alloc_plan(cfg, dev)
    O = torch.empty(Q.shape, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    filtered = args.plan == "filtered"

    def step():
        s2o.plan(cfg, Q, K, bufs, filtered=filtered)
        s2o.attention(cfg, Q, K, V, bufs["perm"], bufs["nblocks"], O)

    for _ in range(args.warmup):
        step()
    st = s2o.last_device_error()
    if st != 0:
        raise RuntimeError(f"device error after warm-up: {s2o.status_string(st)}")

    # the step's launches, captured once as two CUDA graphs (plan, attention)
    # and replayed: the same kernels on the same buffers, without the host's
    # per-launch gaps between them
    plan_run = lambda: s2o.plan(cfg, Q, K, bufs, filtered=filtered)
    attn_run = lambda: s2o.attention(cfg, Q, K, V, bufs["perm"], bufs["nblocks"], O)
    n_plan, n_attn = 0, 0
    if args.graph:
        g_plan, g_attn = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_plan):
            plan_run()
            n_plan = s2o.last_launch_count()
        with torch.cuda.graph(g_attn):
            attn_run()
            n_attn = s2o.last_launch_count()
        plan_run, attn_run = g_plan.replay, g_attn.replay
        for _ in range(2):
            plan_run()
            attn_run()
        st = s2o.last_device_error()
        if st != 0:
            raise RuntimeError(f"device error in the graph warm-up: {s2o.status_string(st)}")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    launches = 0
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for k in range(args.steps):
            ev[k][0].record(stream)
            plan_run()
            launches += n_plan if args.graph else s2o.last_launch_count()
            ev[k][1].record(stream)
            attn_run()
            launches += n_attn if args.graph else s2o.last_launch_count()
            ev[k][2].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    plan_ms = [e[0].elapsed_time(e[1]) for e in ev]
    attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
    total_ms = reduce_max_ms(total_ms, dist, dev)
    st = s2o.last_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the timed region: {s2o.status_string(st)}")

    # the other plan entry point, timed alone for the report (same inputs)
    other = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(3)]
    for e0, e1 in other:
        e0.record(stream)
        s2o.plan(cfg, Q, K, bufs, filtered=not filtered)
        e1.record(stream)
    torch.cuda.synchronize()
    other_ms = float(np.median([e0.elapsed_time(e1) for e0, e1 in other]))
    s2o.plan(cfg, Q, K, bufs, filtered=filtered)

    nb = bufs["nblocks"].cpu().numpy().reshape(w.B, w.Hkv, -1)
    G = w.Hq // w.Hkv
    pairs = kept_pairs(nb, w.N, G)
    dense = dense_flops(w.B, w.Hq, w.N, w.d)
    density = pairs / (w.B * w.Hq * w.N * (w.N + 1) / 2.0)
    ms_step = total_ms / args.steps
    job_flops = dense_full if shard else world * dense
    job_tflops = lambda ms: job_flops / (ms * 1e-3) / 1e12
    value = job_tflops(ms_step)

    # roofline of the dominant kernel (sparse attention): algorithmic flops
    # = 4 d x kept (row, key) pairs, per launch, over its CUDA-event time
    peaks, peak_src = load_peaks()
    attn_mean = float(np.mean(attn_ms))
    achieved = 4.0 * w.d * pairs / (attn_mean * 1e-3) / 1e12
    # the burst peak: each attention launch runs for tens of milliseconds,
    # not the seconds-long loop the sustained figure was taken over
    peak = float(peaks["bf16_tflops"])
    peak_sus = float(peaks.get("bf16_tflops_sustained", peak))
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": ATTN_TRAFFIC.get(w.name if args.tau is None else f"{w.name}@{w.tau:g}"),
                "kernel": "k_sparse_attn2",
                "peak_source": f"{peak_src} bf16 burst (cuBLAS)",
                "peak_sustained": peak_sus, "frac_of_sustained": achieved / peak_sus}

    # per-kernel time of the plan (CUDA events between its kernels) against
    # each kernel's compulsory HBM bytes
    plan_roofline = plan_kernel_roofline(s2o, torch, cfg, Q, K, bufs, filtered, w, peaks, peak_src)

    # accuracy: MSE of the sparse output against dense causal attention (the
    # tau = 0 plan keeps every admissible key), both from fp32 outputs
    Os = s2o.attention(cfg, Q, K, V, bufs["perm"], bufs["nblocks"], out_dtype=s2o.OUT_F32)
    cfg0 = s2o.make_config(w.B, w.Hq, w.Hkv, w.N, tau=0.0)
    s2o.plan(cfg0, Q, K, bufs)
    Od = s2o.attention(cfg0, Q, K, V, bufs["perm"], bufs["nblocks"], out_dtype=s2o.OUT_F32)
    mse, msq = mse_on_device(torch, Os, Od)
    accuracy = {"mse_vs_dense": mse, "relative_mse": mse / msq if msq else None,
                "definition": "mean over all output elements of (O_sparse - O_dense)^2, fp32 outputs of the "
                              "library; dense = the tau = 0 plan"}
    del Os, Od
    torch.cuda.empty_cache()
    s2o.plan(cfg, Q, K, bufs, filtered=filtered)

    # the pages' run-time stop: the full order, then the attention kernel
    # deciding the stop itself; timed after the headline, reported beside it
    online = None
    if args.online_steps > 0 and (w.Hq // w.Hkv) % 2 == 0:
        cout = torch.empty(w.B * w.Hq * s2o.num_segments(cfg), dtype=torch.int32, device=dev)
        for _ in range(2):
            s2o.plan(cfg, Q, K, bufs, filtered=False)
            s2o.attention_online(cfg, Q, K, V, bufs["perm"], O, cout)
        evo = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.online_steps)]
        for e in evo:
            e[0].record(stream)
            s2o.plan(cfg, Q, K, bufs, filtered=False)
            e[1].record(stream)
            s2o.attention_online(cfg, Q, K, V, bufs["perm"], O, cout)
            e[2].record(stream)
        torch.cuda.synchronize()
        if s2o.last_device_error() != 0:
            raise RuntimeError("device error in the run-time stop variant")
        op = float(np.mean([e[0].elapsed_time(e[1]) for e in evo]))
        oa = float(np.mean([e[1].elapsed_time(e[2]) for e in evo]))
        co = cout.cpu().numpy().reshape(w.B, w.Hq, -1)
        online = {"plan_ms": op, "attention_ms": oa, "value": job_tflops(op + oa),
                  "kept_pair_fraction": kept_pairs(co, w.N, 1) / (w.B * w.Hq * w.N * (w.N + 1) / 2.0),
                  "rule": "stop after the first candidate block whose mean relative gain over the tile is < tau"}
        s2o.plan(cfg, Q, K, bufs, filtered=filtered)

    # Q_perm: two query sub-segments per segment, each with its own plan
    qperm = None
    if args.online_steps > 0 and (w.Hq // w.Hkv) % 2 == 0:
        for _ in range(2):
            qp = s2o.plan_qperm(cfg, Q, K)
            s2o.attention_qperm(cfg, Q, K, V, qp, O)
        evq = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.online_steps)]
        for e in evq:
            e[0].record(stream)
            qp = s2o.plan_qperm(cfg, Q, K)
            e[1].record(stream)
            s2o.attention_qperm(cfg, Q, K, V, qp, O)
            e[2].record(stream)
        torch.cuda.synchronize()
        if s2o.last_device_error() != 0:
            raise RuntimeError("device error in the Q_perm variant")
        qpl = float(np.mean([e[0].elapsed_time(e[1]) for e in evq]))
        qat = float(np.mean([e[1].elapsed_time(e[2]) for e in evq]))
        nb2 = qp["nblocks"].cpu().numpy().reshape(2, w.B, w.Hkv, -1)
        rsub = qp["rowsub"].cpu().numpy().reshape(w.B, w.Hkv, -1, 128)
        qperm = {"plan_ms": qpl, "attention_ms": qat, "value": job_tflops(qpl + qat),
                 "kept_pair_fraction": kept_pairs_qperm(nb2, rsub, w.N, w.Hq // w.Hkv) /
                 (w.B * w.Hq * w.N * (w.N + 1) / 2.0)}
        del qp

    # ranking accuracy of the pooled order on sampled segments (exact
    # attention mass per candidate block against the plan's kept blocks)
    ranking = None
    if args.online_steps > 0:
        s2o.plan(cfg, Q, K, bufs, filtered=False)
        S = s2o.num_segments(cfg)
        rng = np.random.default_rng(5)
        segs = sorted(set([2, S // 4, S // 2, 3 * S // 4, S - 1] +
                          [int(x) for x in rng.choice(np.arange(3, S - 1), min(27, max(0, S - 4)), replace=False)]))
        segs = [x for x in segs if 2 <= x < S]
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r0.record(stream)
        st, _ = s2o.block_truth(cfg, Q, K, bufs["perm"], bufs["nblocks"], segs, with_mass=False)
        r1.record(stream)
        torch.cuda.synchronize()
        if s2o.last_device_error() != 0:
            raise RuntimeError("device error in the ranking measurement")
        a = st.cpu().numpy().astype(np.float64)
        kept, true, both = a[..., 0].sum(), a[..., 1].sum(), a[..., 2].sum()
        ranking = {"segments": len(segs), "precision": both / kept if kept else 1.0,
                   "recall": both / true if true else 1.0,
                   "captured_mass": float(a[..., 3].sum() / a[..., 4].sum()) if a[..., 4].sum() > 0 else 1.0,
                   "ms": r0.elapsed_time(r1)}
        s2o.plan(cfg, Q, K, bufs, filtered=filtered)

    # end to end through the host-buffer C ABI call (pinned host memory)
    e2e = None
    if args.e2e_steps > 0:
        pin = lambda a: torch.from_numpy(a.view(np.int16)).pin_memory()
        Qh, Kh, Vh = pin(Qn), pin(Kn), pin(Vn)
        Oh = torch.empty(Qn.shape, dtype=torch.int16).pin_memory()
        nbh = torch.empty(nb.size, dtype=torch.int32).pin_memory()
        del bufs
        torch.cuda.empty_cache()
        arena = torch.empty(s2o.prefill_arena_size(cfg), dtype=torch.uint8, device=dev)
        s2o.prefill_host(cfg, Qh, Kh, Vh, Oh, arena, nblocks_host=nbh)
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            s2o.prefill_host(cfg, Qh, Kh, Vh, Oh, arena, nblocks_host=nbh)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
        e2e_ms = reduce_max_ms(e2e_ms, dist, dev)
        h2d = (Qn.nbytes + Kn.nbytes + Vn.nbytes)
        d2h = Qn.nbytes + nb.size * 4
        e2e = {"value": job_tflops(e2e_ms), "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}
        del arena

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong" if shard else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": bench_config(w, world, args.plan, shard),
            "plan_ms": float(np.mean(plan_ms)), "attention_ms": attn_mean,
            "plan_other": {"kind": "full" if filtered else "filtered", "ms": other_ms},
            "online_stop": online,
            "ranking": ranking,
            "qperm": qperm,
            "attention_only_tflops": job_tflops(attn_mean),
            "kept_pair_fraction": density, "accuracy": accuracy,
            "roofline": roofline, "plan_roofline": plan_roofline,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "launch_mode": "cuda graph replay" if args.graph else "eager",
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
