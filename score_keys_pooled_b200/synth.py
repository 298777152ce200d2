"""Seeded synthetic prefill inputs (Q, K, V as raw bf16 bits).

This module only draws and shapes random inputs; it holds none of the
method's arithmetic.  Both the library's tests/benchmarks and the CPU checker
take their inputs from here.

The pages evaluate on Llama-3.1-8B attention at up to 128K tokens (S2O,
gist.science technical summary, "Resultats Experimentaux"); no weights or
text are available here, so these inputs stand in with that layer's shape
(32 query heads, 8 KV heads, d = 128) and planted structure of the kinds the
pages describe in attention maps: sink tokens, vertical stripes and a local
band.

Recipe (one numpy PCG64 stream, seed 0 unless given):
  1. Q [B,Hq,N,d], K [B,Hkv,N,d], V [B,Hkv,N,d]: standard normal float32, in
     that order.
  2. For every (b, kvh) in order: u = standard normal d-vector / its norm;
     then the stripe positions rng.choice(range(4, N), n_stripe, replace=False).
  3. Keys 0-3 get +4u, stripe keys +3u, every query of the group +1.0u.
  4. Band (optional): q_i[0:32] += 1.5 p(i), k_j[0:32] += 1.5 p(j), with
     p[2k] = sin(i / 10000^(2k/32)), p[2k+1] = cos(same), k = 0..15.
  5. Round to bf16, nearest-even.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    tau: float
    planted: bool      # sinks, stripes and query drift along u
    band: bool         # sinusoidal local band in dims 0..31
    n_stripe: int


def stripe_count_fraction(N: int) -> int:
    return int(round(0.005 * N))


WORKLOADS = {
    # single head, 1K tokens: the size the CPU checker finishes in seconds
    "tiny_1k": Workload("tiny_1k", 1, 1, 1, 1024, 128, 1e-3, True, False, 8),
    # Llama-3.1-8B-shaped layer at 16K with sinks, 0.5% stripes and a band
    "llama_16k": Workload("llama_16k", 1, 32, 8, 16384, 128, 1e-3, True, True, stripe_count_fraction(16384)),
    # same generator at 32K: large enough to exceed L2, small enough to profile
    "llama_32k": Workload("llama_32k", 1, 32, 8, 32768, 128, 1e-3, True, True, stripe_count_fraction(32768)),
    # same generator at 128K: the headline prefill workload
    "llama_128k": Workload("llama_128k", 1, 32, 8, 131072, 128, 1e-3, True, True, stripe_count_fraction(131072)),
    # sinks + 8 stripes, no band, GQA 32/8 at 64K: the tau sweep workload
    "sweep_64k": Workload("sweep_64k", 1, 32, 8, 65536, 128, 1e-3, True, False, 8),
    # iid N(0,1), no planted structure, 128K: flat importance, worst-case sort
    "flat_128k": Workload("flat_128k", 1, 32, 8, 131072, 128, 1e-3, False, False, 0),
}

TAU_SWEEP = (0.0, 1e-4, 3e-4, 1e-3, 3e-3, 1e-2)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _band_code(n: int) -> np.ndarray:
    i = np.arange(n, dtype=np.float64)[:, None]
    k = np.arange(16, dtype=np.float64)[None, :]
    ang = i / np.power(10000.0, 2.0 * k / 32.0)
    p = np.empty((n, 32), dtype=np.float64)
    p[:, 0::2] = np.sin(ang)
    p[:, 1::2] = np.cos(ang)
    return p.astype(np.float32)


def generate(B: int, Hq: int, Hkv: int, N: int, d: int, *, planted: bool, band: bool,
             n_stripe: int, seed: int = 0):
    """Returns (Q, K, V) as uint16 bf16 bits, shapes [B,Hq,N,d], [B,Hkv,N,d] x2."""
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, Hq, N, d), dtype=np.float32)
    K = rng.standard_normal((B, Hkv, N, d), dtype=np.float32)
    V = rng.standard_normal((B, Hkv, N, d), dtype=np.float32)
    if planted:
        for b in range(B):
            for kvh in range(Hkv):
                u = rng.standard_normal(d)
                u = (u / np.linalg.norm(u)).astype(np.float32)
                ns = min(n_stripe, max(0, N - 4))
                stripes = rng.choice(np.arange(4, N), ns, replace=False) if ns else np.zeros(0, np.int64)
                K[b, kvh, :min(4, N)] += np.float32(4.0) * u
                K[b, kvh, stripes] += np.float32(3.0) * u
                Q[b, kvh * G:(kvh + 1) * G] += u
    if band:
        if d < 32:
            raise ValueError("band needs d >= 32")
        pc = np.float32(1.5) * _band_code(N)
        Q[..., :32] += pc
        K[..., :32] += pc
    return _round_rows(Q), _round_rows(K), _round_rows(V)


def _round_rows(x: np.ndarray) -> np.ndarray:
    """bf16 rounding one head at a time, to bound host memory at 128K."""
    out = np.empty(x.shape, dtype=np.uint16)
    for b in range(x.shape[0]):
        for h in range(x.shape[1]):
            out[b, h] = to_bf16_bits(x[b, h])
    return out


def generate_workload(w: Workload, seed: int = 0):
    return generate(w.B, w.Hq, w.Hkv, w.N, w.d, planted=w.planted, band=w.band,
                    n_stripe=w.n_stripe, seed=seed)
