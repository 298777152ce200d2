"""The multi-rank bookkeeping of bench.py on CPU (gloo, world size 2): every
rank solves its own problem, the job time is the max over ranks and the job
throughput is all ranks' work over that time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [120.0, 150.0][rank]
        ms = bench.reduce_max_ms(local_ms, dist, "cpu")
        val = bench.whole_job_tflops(world, 1.0e14, ms)
        q.put((rank, ms, val))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, val in out:
        assert ms == 150.0
        assert val == pytest.approx(2 * 1.0e14 / 0.150 / 1e12)


def test_single_rank_is_identity():
    assert bench.reduce_max_ms(12.5) == 12.5
    assert bench.whole_job_tflops(1, 1.407e14, 204.6) == pytest.approx(1.407e14 / 0.2046 / 1e12)


def test_kept_pairs_closed_form_matches_dense_at_full_blocks():
    import numpy as np
    N = 1024
    S = N // 128
    full = np.array([[[max(0, 2 * s - 3) for s in range(S)]]])
    assert bench.kept_pairs(full, N, 4) == 4 * N * (N + 1) // 2


def test_kv_head_slices_partition_the_heads():
    for Hkv in (1, 2, 3, 8, 13):
        for world in range(1, Hkv + 1):
            got = [bench.kv_head_slice(Hkv, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == Hkv
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))      # contiguous, disjoint
            sizes = [k1 - k0 for k0, k1 in got]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        bench.kv_head_slice(4, 5, 0)


def _shard_rank(rank, world, port, q):
    """Each rank plans its KV heads of one problem with the oracle and
    gathers the others' C(s); the assembled plan must be the whole problem's."""
    import numpy as np
    from oracle import s2o_oracle as O
    from score_keys_pooled_b200 import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        Q, K, V = synth.generate(1, 6, 3, 512, 32, planted=True, band=True, n_stripe=4, seed=17)
        p = O.Params(tau=2e-3)
        q_loc, k_loc, _ = bench.shard_inputs(Q, K, V, world, rank)
        mine = O.plan(q_loc, k_loc, p)["nblocks"]
        parts = [None] * world
        dist.all_gather_object(parts, (rank, mine))
        whole = np.concatenate([m for _, m in sorted(parts, key=lambda x: x[0])], axis=1)
        ref = O.plan(Q, K, p)["nblocks"]
        q.put((rank, bool(np.array_equal(whole, ref)), whole.shape))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_one_problem_by_kv_head():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=5) for _ in range(2))
    assert [o[0] for o in out] == [0, 1]
    assert all(o[1] for o in out), out
