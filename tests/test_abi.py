"""Host-side checks of the C ABI (no GPU needed: no call here reaches CUDA)."""
import ctypes
import subprocess

import numpy as np
import pytest

import score_keys_pooled_b200 as s2o
from score_keys_pooled_b200 import build


@pytest.fixture(scope="module")
def L():
    build.build()
    return s2o.lib()


def test_library_exports_every_header_symbol(L):
    names = s2o.header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", s2o.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(names) <= exported


def test_segment_geometry_matches_closed_form(L):
    for N in (1, 127, 128, 129, 1024, 16384, 131072, 1000):
        cfg = s2o.make_config(1, 32, 8, N)
        S = (N + 127) // 128
        assert s2o.num_segments(cfg) == S
        for s in range(S + 1):
            want = 64 * (s - 2) ** 2 if s >= 2 else 0
            assert s2o.candidate_offset(cfg, s) == want
        assert s2o.num_candidates(cfg) == (64 * (S - 2) ** 2 if S >= 2 else 0)
    cfg = s2o.make_config(1, 32, 8, 131072)
    assert s2o.num_candidates(cfg) == 66_846_976  # 128 * (1023*1024/2 - 1) - 192 * 1022


@pytest.mark.parametrize("field,value,code", [
    ("d", 64, 2), ("Lq", 64, 2), ("Bk", 32, 2), ("n_sink", 0, 2), ("window_prev", 256, 2),
    ("N", 0, 1), ("Hkv", 3, 1), ("tau", -1.0, 1), ("tau", float("nan"), 1), ("N", (1 << 19) + 1, 2),
])
def test_config_validation(L, field, value, code):
    cfg = s2o.make_config(1, 32, 8, 1024)
    setattr(cfg, field, value)
    n = ctypes.c_size_t(0)
    assert L.s2o_plan_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == code
    assert s2o.num_segments(cfg) == -1


def test_null_and_alignment_rejected_before_any_launch(L):
    cfg = s2o.make_config(1, 4, 1, 1024)
    P = ctypes.c_void_p
    good = P(1 << 20)
    assert L.s2o_plan(ctypes.byref(cfg), None, good, good, good, good, None, good, 1 << 30, None) == 1
    assert L.s2o_plan(ctypes.byref(cfg), P((1 << 20) + 2), good, good, good, good, None, good, 1 << 30, None) == 1
    assert L.s2o_attention(ctypes.byref(cfg), good, good, good, good, good, good, 7, None) == 1
    assert L.s2o_attention(ctypes.byref(cfg), good, good, None, good, good, good, 0, None) == 1
    ws = s2o.plan_workspace_size(cfg)
    assert L.s2o_plan(ctypes.byref(cfg), good, good, good, good, good, None, P(1 << 20), ws - 1, None) == 3
    assert L.s2o_plan_contiguous(ctypes.byref(cfg), good, None, good, good, None) == 1
    # the run-time stop: null output count, bad dtype, and an odd group size (its tile is a head pair)
    assert L.s2o_attention_online(ctypes.byref(cfg), good, good, good, good, good, 0, None, None) == 1
    assert L.s2o_attention_online(ctypes.byref(cfg), good, good, good, good, good, 7, good, None) == 1
    odd = s2o.make_config(1, 3, 1, 1024)
    assert L.s2o_attention_online(ctypes.byref(odd), good, good, good, good, good, 0, good, None) == 2
    assert L.s2o_plan_filtered(ctypes.byref(cfg), None, good, good, good, good, None, good, 1 << 30, None) == 1


def test_status_strings(L):
    for code in range(8):
        assert s2o.status_string(code)
    assert s2o.status_string(0) == "ok"


def test_workspace_size_grows_with_candidates(L):
    small = s2o.plan_workspace_size(s2o.make_config(1, 4, 1, 1024))
    big = s2o.plan_workspace_size(s2o.make_config(1, 4, 1, 4096))
    assert big > small > 0
    cfg = s2o.make_config(1, 32, 8, 131072)
    # 4 sort buffers of 4 bytes per candidate dominate
    assert s2o.plan_workspace_size(cfg) >= 16 * 8 * s2o.num_candidates(cfg)


def test_noalloc_rejects_configs_over_its_scratch(L):
    """s2o_plan_noalloc refuses, before any CUDA call, every config whose plan
    workspace exceeds its 32 MiB scratch; the header's example (B = 1, 8 KV
    heads: N above about 5K) holds for the current workspace layout (the key
    digits take 384 bytes per key and KV head)."""
    limit = 32 << 20
    P = ctypes.c_void_p
    good = P(1 << 20)
    assert s2o.plan_workspace_size(s2o.make_config(1, 32, 8, 5120)) <= limit
    for N in (5504, 8192, 131072):
        cfg = s2o.make_config(1, 32, 8, N)
        assert s2o.plan_workspace_size(cfg) > limit
        assert L.s2o_plan_noalloc(ctypes.byref(cfg), good, good, good, good, good, None, None) == 3
