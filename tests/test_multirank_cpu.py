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
