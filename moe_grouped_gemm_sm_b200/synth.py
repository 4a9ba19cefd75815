"""Seeded synthetic inputs shared by the CUDA path's tests, the benchmark and the oracle's tests.

This module holds none of the GEMM's or the cast's arithmetic: it only draws numbers.
Every value comes from one counter-based generator, defined here in full so that any
reader can regenerate the same bytes:

* splitmix64 (S. Vigna's published finaliser; golden-ratio increment
  0x9E3779B97F4A7C15, multipliers 0xBF58476D1CE4E5B9 and 0x94D049BB133111EB,
  shifts 30/27/31). Draw ``i`` of stream ``seed`` is
  ``mix(seed * 0xD1B54A32D192ED03 + (i + 1) * 0x9E3779B97F4A7C15)`` (mod 2**64).
* uniform doubles ``u = (x >> 11) * 2**-53`` in [0, 1).
* normals by Box–Muller on consecutive pairs ``(u1, u2)``: ``r = sqrt(-2 ln(1 - u1))``,
  ``z0 = r cos(2 pi u2)``, ``z1 = r sin(2 pi u2)``.
* bf16 values: the fp64 normal times sigma is rounded to fp32 (round to nearest even),
  then to bf16 (round to nearest even on the fp32 bit pattern).

The workloads mirror the DeepSeek-V3/R1 GEMM shapes that the DeepGEMM pages time
(likun.im/craft/deepgemm, section 3 "数字要分清楚", the H800 performance table):
activations and weights N(0, 1), the optional C addend N(0, 0.1), contiguous MoE
groups of U{2048..6144} rows padded to 128, masked MoE with masked_m ~ U{64..256}.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_SEED_MUL = np.uint64(0xD1B54A32D192ED03)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

BASE_SEED = 2026
# stream offsets from the base seed
STREAM_A, STREAM_B, STREAM_C, STREAM_GROUPS, STREAM_GARBAGE = 0, 1, 2, 3, 4

_CHUNK = 1 << 22
_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))
    return _POOL


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64(seed: int, start: int, count: int) -> np.ndarray:
    """Draws ``start .. start+count-1`` of stream ``seed`` as uint64."""
    with np.errstate(over="ignore"):
        base = np.uint64(seed % (1 << 64)) * _SEED_MUL
        idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        return _mix(base + idx * _GAMMA)


def uniform01(seed: int, start: int, count: int) -> np.ndarray:
    x = splitmix64(seed, start, count)
    return (x >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal_f64(seed: int, count: int, start_pair: int = 0) -> np.ndarray:
    """``count`` N(0,1) doubles; normal j uses draws 2*(j//2) and 2*(j//2)+1 of the stream."""
    npairs = (count + 1) // 2
    u = uniform01(seed, 2 * start_pair, 2 * npairs)
    u1, u2 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log1p(-u1))
    t = 2.0 * np.pi * u2
    out = np.empty(2 * npairs, dtype=np.float64)
    out[0::2] = r * np.cos(t)
    out[1::2] = r * np.sin(t)
    return out[:count]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even of finite fp32 values to bf16, returned as uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rnd = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + rnd) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(seed: int, shape, sigma: float = 1.0) -> np.ndarray:
    """bf16 bit patterns (uint16) of N(0, sigma^2) draws, filled in row-major order."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)

    def fill(s):
        cnt = min(_CHUNK, n - s)
        # chunks start on even draw indices so the pairing never straddles two chunks
        z = normal_f64(seed, cnt, start_pair=s // 2)
        out[s:s + cnt] = f32_to_bf16_bits((z * sigma).astype(np.float32))

    starts = range(0, n, _CHUNK)
    if n > 2 * _CHUNK:
        list(_pool().map(fill, starts))
    else:
        for s in starts:
            fill(s)
    return out.reshape(shape)


def uniform_int(seed: int, count: int, lo: int, hi: int) -> np.ndarray:
    """``count`` integers in [lo, hi] (inclusive) as ``lo + x mod (hi - lo + 1)``."""
    x = splitmix64(seed, 0, count)
    return (lo + (x % np.uint64(hi - lo + 1)).astype(np.int64)).astype(np.int64)


def seed_for(base: int, stream: int, salt: int = 0) -> int:
    """Seed of one tensor: the base seed plus its stream offset, with an optional per-shape salt."""
    return base + stream + 1000 * salt


# ---------------------------------------------------------------------------------------------
# Workload recipes
# ---------------------------------------------------------------------------------------------

def dense_inputs(M: int, N: int, K: int, with_c: bool, base: int = BASE_SEED, salt: int = 0):
    """bf16 A [M,K], B [N,K] ~ N(0,1) and C [M,N] ~ N(0,0.1) (None when absent)."""
    a = normal_bf16(seed_for(base, STREAM_A, salt), (M, K))
    b = normal_bf16(seed_for(base, STREAM_B, salt), (N, K))
    c = normal_bf16(seed_for(base, STREAM_C, salt), (M, N), sigma=0.1) if with_c else None
    return a, b, c


def contiguous_layout(G: int, lo: int = 2048, hi: int = 6144, align: int = 128,
                      base: int = BASE_SEED, salt: int = 0):
    """Per-expert row counts m_g ~ U{lo..hi}, each group padded up to ``align`` rows.

    Returns (m_per_group, grouped_layout int32 [M_sum]) where padding rows hold -1.
    """
    m = uniform_int(seed_for(base, STREAM_GROUPS, salt), G, lo, hi)
    padded = (m + align - 1) // align * align
    layout = np.full(int(padded.sum()), -1, dtype=np.int32)
    off = 0
    for g in range(G):
        layout[off:off + int(m[g])] = g
        off += int(padded[g])
    return m, layout


def contiguous_inputs(G: int, N: int, K: int, lo: int = 2048, hi: int = 6144,
                      base: int = BASE_SEED, salt: int = 0):
    """A [M_sum,K] (padding rows hold N(0,1) garbage too), B [G,N,K], grouped_layout."""
    m, layout = contiguous_layout(G, lo, hi, base=base, salt=salt)
    M_sum = layout.shape[0]
    a = normal_bf16(seed_for(base, STREAM_A, salt), (M_sum, K))
    b = normal_bf16(seed_for(base, STREAM_B, salt), (G, N, K))
    return m, layout, a, b


def masked_inputs(G: int, M_max: int, N: int, K: int, lo: int = 64, hi: int = 256,
                  base: int = BASE_SEED, salt: int = 0):
    """A [G,M_max,K] with N(0,1) valid rows and N(0,10^2) garbage rows >= masked_m[g]."""
    masked_m = uniform_int(seed_for(base, STREAM_GROUPS, salt), G, lo, hi).astype(np.int32)
    a = normal_bf16(seed_for(base, STREAM_A, salt), (G, M_max, K))
    garbage = normal_bf16(seed_for(base, STREAM_GARBAGE, salt), (G, M_max, K), sigma=10.0)
    rows = np.arange(M_max)[None, :, None]
    a = np.where(rows >= masked_m[:, None, None], garbage, a).astype(np.uint16)
    b = normal_bf16(seed_for(base, STREAM_B, salt), (G, N, K))
    return masked_m, a, b


def sentinel_bf16() -> int:
    """bf16 bit pattern written into D before a masked call; rows >= masked_m must keep it."""
    return 0xDEAD
