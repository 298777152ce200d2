"""S2O sparse prefill attention for B200: thin Python binding of libs2o.so.

The functions below only marshal arguments (torch tensors -> device pointers,
the current CUDA stream) into the C ABI declared in include/s2o.h; every step
of the method runs in the library's CUDA kernels.  There is no CPU fallback:
if the compiled library is missing, importing the binding's entry points
raises.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB_PATH = os.path.join(PKG, "libs2o.so")
HEADER = os.path.join(ROOT, "include", "s2o.h")

OUT_BF16, OUT_F32 = 0, 1

STATUS = {
    0: "S2O_OK", 1: "S2O_ERR_INVALID_ARG", 2: "S2O_ERR_UNSUPPORTED_SHAPE",
    3: "S2O_ERR_WORKSPACE_TOO_SMALL", 4: "S2O_ERR_CUDA", 5: "S2O_ERR_DEVICE_TIMEOUT",
    6: "S2O_ERR_NONFINITE", 7: "S2O_ERR_BAD_PLAN",
}


class S2OError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)}")
        self.code = code


class Config(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("N", ctypes.c_int32), ("d", ctypes.c_int32), ("Lq", ctypes.c_int32),
                ("Bk", ctypes.c_int32), ("n_sink", ctypes.c_int32), ("window_prev", ctypes.c_int32),
                ("tau", ctypes.c_double)]


def make_config(B, Hq, Hkv, N, d=128, tau=1e-3, Lq=128, Bk=64, n_sink=64, window_prev=128) -> Config:
    return Config(B, Hq, Hkv, N, d, Lq, Bk, n_sink, window_prev, float(tau))


_lib = None
_P = ctypes.c_void_p
_CFG = ctypes.POINTER(Config)


def lib() -> ctypes.CDLL:
    """The loaded CUDA library (built in-tree by score_keys_pooled_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run `python -m score_keys_pooled_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.s2o_num_segments.argtypes = [_CFG]
        L.s2o_num_segments.restype = ctypes.c_int32
        L.s2o_num_candidates.argtypes = [_CFG]
        L.s2o_num_candidates.restype = ctypes.c_int64
        L.s2o_candidate_offset.argtypes = [_CFG, ctypes.c_int32]
        L.s2o_candidate_offset.restype = ctypes.c_int64
        L.s2o_plan_workspace_size.argtypes = [_CFG, ctypes.POINTER(ctypes.c_size_t)]
        L.s2o_plan.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
        L.s2o_plan_filtered.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
        L.s2o_plan_noalloc.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, _P]
        L.s2o_plan_contiguous.argtypes = [_CFG, _P, _P, _P, _P, _P]
        L.s2o_attention.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, ctypes.c_int32, _P]
        L.s2o_attention_bounded.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, ctypes.c_int32, ctypes.c_uint32, _P]
        L.s2o_attention_online.argtypes = [_CFG, _P, _P, _P, _P, _P, ctypes.c_int32, _P, _P]
        L.s2o_block_truth_workspace_size.argtypes = [_CFG, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
        L.s2o_plan_qperm_workspace_size.argtypes = [_CFG, ctypes.POINTER(ctypes.c_size_t)]
        L.s2o_plan_qperm.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
        L.s2o_attention_qperm.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int32, _P]
        L.s2o_block_truth.argtypes = [_CFG, _P, _P, _P, _P, _P, ctypes.c_int32, _P, _P, _P, ctypes.c_size_t, _P]
        L.s2o_prefill_arena_size.argtypes = [_CFG, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
        L.s2o_prefill_host.argtypes = [_CFG, _P, _P, _P, _P, ctypes.c_int32, _P, _P, ctypes.c_size_t, _P]
        L.s2o_status_string.argtypes = [ctypes.c_int]
        L.s2o_status_string.restype = ctypes.c_char_p
        L.s2o_last_device_error.argtypes = [_P]
        L.s2o_last_launch_count.restype = ctypes.c_int32
        L.s2o_stage_timing.argtypes = [ctypes.c_int32]
        L.s2o_stage_timing.restype = ctypes.c_int
        L.s2o_last_stage_times.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_char_p),
                                           ctypes.c_int32]
        L.s2o_last_stage_times.restype = ctypes.c_int32
        for name in ("s2o_plan_workspace_size", "s2o_plan", "s2o_plan_filtered", "s2o_plan_noalloc", "s2o_plan_contiguous", "s2o_attention", "s2o_attention_bounded", "s2o_attention_online",
                     "s2o_block_truth_workspace_size", "s2o_block_truth", "s2o_plan_qperm_workspace_size",
                     "s2o_plan_qperm", "s2o_attention_qperm",
                     "s2o_prefill_arena_size", "s2o_prefill_host", "s2o_last_device_error"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/s2o.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(s2o_[a-z_0-9]+)\s*\(", text)))


def _check(code: int, what: str):
    if code != 0:
        raise S2OError(code, what)


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def num_segments(cfg: Config) -> int:
    return lib().s2o_num_segments(ctypes.byref(cfg))


def num_candidates(cfg: Config) -> int:
    return lib().s2o_num_candidates(ctypes.byref(cfg))


def candidate_offset(cfg: Config, s: int) -> int:
    return lib().s2o_candidate_offset(ctypes.byref(cfg), s)


def plan_workspace_size(cfg: Config) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().s2o_plan_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "s2o_plan_workspace_size")
    return n.value


def prefill_arena_size(cfg: Config, out_dtype: int = OUT_BF16) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().s2o_prefill_arena_size(ctypes.byref(cfg), out_dtype, ctypes.byref(n)), "s2o_prefill_arena_size")
    return n.value


def alloc_plan(cfg: Config, device="cuda", workspace=True):
    """Device buffers for one s2o_plan call (allocated by torch)."""
    import torch
    BH = cfg.B * cfg.Hkv
    S, T = num_segments(cfg), num_candidates(cfg)
    out = dict(
        scores=torch.empty(BH * T + 4, dtype=torch.float32, device=device),
        perm=torch.empty(BH * T + 4, dtype=torch.int32, device=device),
        nblocks=torch.empty(BH * S, dtype=torch.int32, device=device),
        seg_stats=torch.empty(BH * S * 2, dtype=torch.float32, device=device),
    )
    if workspace:
        out["workspace"] = torch.empty(plan_workspace_size(cfg), dtype=torch.uint8, device=device)
    return out


def plan(cfg: Config, Q, K, bufs=None, stream=None, filtered: bool = False):
    """Run s2o_plan (or s2o_plan_filtered); returns the buffer dict (scores,
    perm, nblocks, seg_stats)."""
    bufs = alloc_plan(cfg, Q.device) if bufs is None else bufs
    ws = bufs["workspace"]
    fn, name = (lib().s2o_plan_filtered, "s2o_plan_filtered") if filtered else (lib().s2o_plan, "s2o_plan")
    _check(fn(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(bufs["scores"]), _ptr(bufs["perm"]),
              _ptr(bufs["nblocks"]), _ptr(bufs.get("seg_stats")), _ptr(ws), ws.numel(), _stream(stream)), name)
    return bufs


def plan_noalloc(cfg: Config, Q, K, bufs, stream=None):
    """s2o_plan_noalloc: the plan with the library's static scratch; `bufs`
    holds the output buffers (no workspace is needed or used)."""
    _check(lib().s2o_plan_noalloc(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(bufs["scores"]), _ptr(bufs["perm"]),
                                  _ptr(bufs["nblocks"]), _ptr(bufs.get("seg_stats")), _stream(stream)),
           "s2o_plan_noalloc")
    return bufs


def plan_contiguous(cfg: Config, scores, seg_stats, nblocks_match, perm_out, stream=None):
    _check(lib().s2o_plan_contiguous(ctypes.byref(cfg), _ptr(scores), _ptr(seg_stats), _ptr(nblocks_match),
                                     _ptr(perm_out), _stream(stream)), "s2o_plan_contiguous")
    return perm_out


def attention(cfg: Config, Q, K, V, perm, nblocks, O=None, out_dtype: int = OUT_BF16, stream=None):
    import torch
    if O is None:
        O = torch.empty(Q.shape, dtype=torch.bfloat16 if out_dtype == OUT_BF16 else torch.float32,
                        device=Q.device)
    _check(lib().s2o_attention(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V), _ptr(perm), _ptr(nblocks),
                               _ptr(O), out_dtype, _stream(stream)), "s2o_attention")
    return O


def attention_bounded(cfg: Config, Q, K, V, perm, nblocks, max_polls: int, O=None, out_dtype: int = OUT_BF16,
                      stream=None):
    """s2o_attention with every pipeline wait limited to max_polls polls (tests of the timeout path)."""
    import torch
    if O is None:
        O = torch.empty(Q.shape, dtype=torch.bfloat16 if out_dtype == OUT_BF16 else torch.float32,
                        device=Q.device)
    _check(lib().s2o_attention_bounded(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V), _ptr(perm), _ptr(nblocks),
                                       _ptr(O), out_dtype, max_polls, _stream(stream)), "s2o_attention_bounded")
    return O


def attention_online(cfg: Config, Q, K, V, perm, O=None, nblocks_out=None, out_dtype: int = OUT_BF16, stream=None):
    """s2o_attention_online: the run-time stop; returns (O, nblocks_out [B*Hq*S])."""
    import torch
    if O is None:
        O = torch.empty(Q.shape, dtype=torch.bfloat16 if out_dtype == OUT_BF16 else torch.float32,
                        device=Q.device)
    if nblocks_out is None:
        nblocks_out = torch.empty(cfg.B * cfg.Hq * num_segments(cfg), dtype=torch.int32, device=Q.device)
    _check(lib().s2o_attention_online(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V), _ptr(perm), _ptr(O), out_dtype,
                                      _ptr(nblocks_out), _stream(stream)), "s2o_attention_online")
    return O, nblocks_out


def plan_qperm(cfg: Config, Q, K, stream=None):
    """s2o_plan_qperm; returns dict(scores [2*B*Hkv*T], perm, nblocks [2*B*Hkv*S], rowsub [B*Hkv*S*128])."""
    import torch
    BH = cfg.B * cfg.Hkv
    S, T = num_segments(cfg), num_candidates(cfg)
    dev = Q.device
    out = dict(scores=torch.empty(2 * BH * T + 4, dtype=torch.float32, device=dev),
               perm=torch.empty(2 * BH * T + 4, dtype=torch.int32, device=dev),
               nblocks=torch.empty(2 * BH * S, dtype=torch.int32, device=dev),
               rowsub=torch.empty(BH * S * 128, dtype=torch.uint8, device=dev))
    n = ctypes.c_size_t(0)
    _check(lib().s2o_plan_qperm_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "s2o_plan_qperm_workspace_size")
    ws = torch.empty(n.value, dtype=torch.uint8, device=dev)
    _check(lib().s2o_plan_qperm(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(out["scores"]), _ptr(out["perm"]),
                                _ptr(out["nblocks"]), _ptr(out["rowsub"]), _ptr(ws), ws.numel(), _stream(stream)),
           "s2o_plan_qperm")
    return out


def attention_qperm(cfg: Config, Q, K, V, qp, O=None, out_dtype: int = OUT_BF16, stream=None):
    import torch
    if O is None:
        O = torch.empty(Q.shape, dtype=torch.bfloat16 if out_dtype == OUT_BF16 else torch.float32,
                        device=Q.device)
    _check(lib().s2o_attention_qperm(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(V), _ptr(qp["perm"]),
                                     _ptr(qp["nblocks"]), _ptr(qp["rowsub"]), _ptr(O), out_dtype, _stream(stream)),
           "s2o_attention_qperm")
    return O


def block_truth(cfg: Config, Q, K, perm, nblocks, segments, with_mass: bool = True, stream=None):
    """s2o_block_truth on the listed segments; returns (stats [n, B*Hkv, 5],
    mass [n, B*Hkv, nbmax] or None) as device tensors."""
    import numpy as np
    import torch
    segs = np.ascontiguousarray(np.asarray(segments, dtype=np.int32))
    n = len(segs)
    BH = cfg.B * cfg.Hkv
    nbmax = max(0, 128 * (num_segments(cfg) - 1) - 192) // 64
    stats = torch.empty(n * BH * 5, dtype=torch.float32, device=Q.device)
    mass = torch.empty(max(1, n * BH * nbmax), dtype=torch.float32, device=Q.device) if with_mass else None
    nbytes = ctypes.c_size_t(0)
    _check(lib().s2o_block_truth_workspace_size(ctypes.byref(cfg), n, ctypes.byref(nbytes)),
           "s2o_block_truth_workspace_size")
    ws = torch.empty(nbytes.value, dtype=torch.uint8, device=Q.device)
    _check(lib().s2o_block_truth(ctypes.byref(cfg), _ptr(Q), _ptr(K), _ptr(perm), _ptr(nblocks),
                                 segs.ctypes.data, n, _ptr(stats), _ptr(mass), _ptr(ws), ws.numel(),
                                 _stream(stream)), "s2o_block_truth")
    return stats.view(n, BH, 5), (mass[:n * BH * nbmax].view(n, BH, nbmax) if with_mass else None)


def prefill_host(cfg: Config, Q_host, K_host, V_host, O_host, arena, nblocks_host=None,
                 out_dtype: int = OUT_BF16, stream=None):
    """Whole path from host tensors (pinned for speed) through the C ABI."""
    _check(lib().s2o_prefill_host(ctypes.byref(cfg), _ptr(Q_host), _ptr(K_host), _ptr(V_host), _ptr(O_host),
                                  out_dtype, _ptr(nblocks_host), _ptr(arena), arena.numel(), _stream(stream)),
           "s2o_prefill_host")
    return O_host


def last_device_error(stream=None) -> int:
    return lib().s2o_last_device_error(_stream(stream))


def last_launch_count() -> int:
    return lib().s2o_last_launch_count()


def stage_timing(enable: bool):
    """Turn per-kernel event timing of the plan calls on or off (this thread)."""
    _check(lib().s2o_stage_timing(1 if enable else 0), "s2o_stage_timing")


def last_stage_times() -> list[tuple[str, float]]:
    """(kernel name, device ms) of each kernel of the last plan call on this thread."""
    ms = (ctypes.c_float * 16)()
    names = (ctypes.c_char_p * 16)()
    n = lib().s2o_last_stage_times(ms, names, 16)
    if n < 0:
        raise S2OError(4, "s2o_last_stage_times")
    return [(names[i].decode(), float(ms[i])) for i in range(n)]


def status_string(code: int) -> str:
    return lib().s2o_status_string(code).decode()
