"""The allocation-free plan entry point (s2o_plan_noalloc).

Some callers may not allocate device memory themselves: plugins inside an
engine that owns all device memory through its own pool, and code on a
latency-critical path where cudaMalloc/cudaFree would synchronise the device.
s2o_plan_noalloc serves them from a fixed 32 MiB scratch buffer compiled into
the library.  These tests call it through the C ABI and check that it returns
exactly what s2o_plan (with a caller-allocated workspace) returns, bit for bit,
on two calls in a row with different inputs, after a call of another shape has
left unrelated values in the shared buffer: the buffer keeps the previous
call's contents, which must not leak into the next result.
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import score_keys_pooled_b200 as s2o
from score_keys_pooled_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    s2o.lib()


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def _stale_fill(shape):
    """A call of another shape and seed, so the shared scratch holds unrelated
    values (sorted keys, partial sums, bucket tables) when the call under test
    starts."""
    B, Hq, Hkv, N = shape
    cfg = s2o.make_config(B, Hq, Hkv, N, tau=5e-3)
    Q, K, _ = synth.generate(B, Hq, Hkv, N, 128, planted=False, band=False, n_stripe=0, seed=99)
    q, k = _dev(Q), _dev(K)
    s2o.plan_noalloc(cfg, q, k, s2o.alloc_plan(cfg, q.device, workspace=False))
    assert s2o.last_device_error() == 0


@pytest.mark.parametrize("shape", [(1, 8, 2, 2048), (1, 4, 1, 1111)])
def test_noalloc_plan_matches_workspace_plan_on_consecutive_calls(shape):
    B, Hq, Hkv, N = shape
    cfg = s2o.make_config(B, Hq, Hkv, N, tau=1e-3)
    _stale_fill((1, 4, 2, 11264))
    for seed in (21, 22):
        Q, K, _ = synth.generate(B, Hq, Hkv, N, 128, planted=True, band=True, n_stripe=8, seed=seed)
        q, k = _dev(Q), _dev(K)
        # the reference plan runs on a workspace poisoned with 0xFF bytes: a
        # word read before it is written would show up as a difference
        ref = s2o.alloc_plan(cfg, q.device)
        ref["workspace"].fill_(255)
        s2o.plan(cfg, q, k, bufs=ref)
        ref_launches = s2o.last_launch_count()
        assert s2o.last_device_error() == 0
        got = s2o.alloc_plan(cfg, q.device, workspace=False)
        before = torch.cuda.memory_allocated()
        s2o.plan_noalloc(cfg, q, k, got)
        assert s2o.last_launch_count() == ref_launches
        assert s2o.last_device_error() == 0
        assert torch.cuda.memory_allocated() == before
        T = cfg.B * cfg.Hkv * s2o.num_candidates(cfg)
        # the same kernels on the same inputs: every output bit for bit
        assert torch.equal(got["perm"][:T], ref["perm"][:T])
        assert torch.equal(got["nblocks"], ref["nblocks"])
        assert torch.equal(got["scores"][:T], ref["scores"][:T])
        assert torch.equal(got["seg_stats"], ref["seg_stats"])


def test_noalloc_rejects_configs_beyond_its_scratch():
    cfg = s2o.make_config(1, 32, 8, 16384, tau=1e-3)
    assert s2o.plan_workspace_size(cfg) > 32 << 20
    P = ctypes.c_void_p
    good = P(1 << 20)
    code = s2o.lib().s2o_plan_noalloc(ctypes.byref(cfg), good, good, good, good, good, None, None)
    assert code == 3  # S2O_ERR_WORKSPACE_TOO_SMALL, nothing launched
    assert s2o.last_launch_count() == 0
