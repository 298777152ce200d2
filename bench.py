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


def reduce_max_ms(ms: float, dist=None, device="cpu") -> float:
    """Max over ranks of a per-rank time (the slowest rank bounds the job)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(ms)
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


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


def bench_config(w, world: int, plan: str) -> dict:
    """The workload description both arms print."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "tau": w.tau,
            "global_batch": w.B * world, "seq_len": w.N, "parallelism": f"independent x{world}",
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
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


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
    ap.add_argument("--plan", default="filtered", choices=["full", "filtered"],
                    help="s2o_plan (every segment fully ordered) or s2o_plan_filtered (only the prefix the "
                         "stop rule can reach; same kept sets and output)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "s2o":
        ap.error("--warmup must be >= 3")

    from score_keys_pooled_b200 import synth
    w = synth.WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        reference_arm(args, w, world, rank)
        return

    import torch
    import score_keys_pooled_b200 as s2o

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)

    # each rank solves an independent problem (its own seed): weak scaling
    Qn, Kn, Vn = synth.generate_workload(w, seed=rank)
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
            s2o.plan(cfg, Q, K, bufs, filtered=filtered)
            launches += s2o.last_launch_count()
            ev[k][1].record(stream)
            s2o.attention(cfg, Q, K, V, bufs["perm"], bufs["nblocks"], O)
            launches += s2o.last_launch_count()
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
    value = whole_job_tflops(world, dense, ms_step)

    # roofline of the dominant kernel (sparse attention): algorithmic flops
    # = 4 d x kept (row, key) pairs, per launch, over its CUDA-event time
    peaks, peak_src = load_peaks()
    attn_mean = float(np.mean(attn_ms))
    achieved = 4.0 * w.d * pairs / (attn_mean * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    # DRAM bytes per launch of k_sparse_attn2 from an ncu capture of the 32K
    # workload (764.7 MB), scaled by the rows processed to the 128K launch;
    # None for other workloads
    traffic = 3.06e9 if w.name == "llama_128k" else None
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic, "kernel": "k_sparse_attn2",
                "peak_source": f"{peak_src} bf16 sustained"}

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
        online = {"plan_ms": op, "attention_ms": oa, "value": whole_job_tflops(world, dense, op + oa),
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
        qperm = {"plan_ms": qpl, "attention_ms": qat, "value": whole_job_tflops(world, dense, qpl + qat),
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
        e2e = {"value": whole_job_tflops(world, dense, e2e_ms), "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}
        del arena

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample, _ = cpu_oracle_sample(Qn, Kn, Vn, w.tau, seconds=15.0)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": 1, "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": bench_config(w, world, args.plan),
            "plan_ms": float(np.mean(plan_ms)), "attention_ms": attn_mean,
            "plan_other": {"kind": "full" if filtered else "filtered", "ms": other_ms},
            "online_stop": online,
            "ranking": ranking,
            "qperm": qperm,
            "attention_only_tflops": whole_job_tflops(world, dense, attn_mean),
            "kept_pair_fraction": density,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
