"""Python access to the C oracle (``oracle/dg_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()`` and by the
benchmark's CPU-baseline / reference leg. The library's product path never imports it.

All arrays are numpy; bf16 values travel as their uint16 bit patterns and e4m3 values as
their uint8 codes. Results of the GEMMs are fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dg_oracle.c")
_LIB = os.path.join(_HERE, "libdg_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compiles the oracle with gcc (fp-contract off, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                               "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P, I, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.dgo_e4m3_decode.restype = D
        L.dgo_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.dgo_e4m3_encode_satrne.restype = ctypes.c_uint8
        L.dgo_e4m3_encode_satrne.argtypes = [ctypes.c_float]
        L.dgo_bf16_to_f32.restype = ctypes.c_float
        L.dgo_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.dgo_cast_per_token.argtypes = [P, I, I, P, P]
        L.dgo_cast_per_block.argtypes = [P, I, I, I, P, P]
        L.dgo_transform_sf.argtypes = [P, I, I, I, P]
        L.dgo_gemm_nt.argtypes = [P, P, P, P, P, I, I, I, P, I, P]
        L.dgo_m_grouped_contiguous.argtypes = [P, P, P, P, P, P, I, I, I, I, P, I, P]
        L.dgo_m_grouped_masked.argtypes = [P, P, P, P, P, P, I, I, I, I, P]
        L.dgo_cast_per_channel.argtypes = [P, I, I, P, P]
        L.dgo_cast_per_token_scatter.argtypes = [P, P, I, I, I, P, P]
        L.dgo_ue8m0_of_amax.restype = ctypes.c_uint8
        L.dgo_ue8m0_of_amax.argtypes = [ctypes.c_float]
        L.dgo_cast_per_token_ue8m0.argtypes = [P, I, I, P, P]
        L.dgo_cast_per_block_ue8m0.argtypes = [P, I, I, I, P, P]
        L.dgo_k_grouped_tn.argtypes = [P, P, P, P, P, P, I, I, I, P]
        for f in ("dgo_cast_per_token", "dgo_cast_per_block", "dgo_transform_sf", "dgo_gemm_nt",
                  "dgo_m_grouped_contiguous", "dgo_m_grouped_masked", "dgo_num_threads",
                  "dgo_cast_per_channel", "dgo_k_grouped_tn", "dgo_cast_per_token_ue8m0",
                  "dgo_cast_per_block_ue8m0", "dgo_cast_per_token_scatter"):
            getattr(L, f).restype = I
        _lib = L
    return _lib


def _p(arr):
    return None if arr is None else arr.ctypes.data_as(ctypes.c_void_p)


def _c(arr, dtype):
    return None if arr is None else np.ascontiguousarray(arr, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (code {rc})")


def pad4(x: int) -> int:
    return (x + 3) // 4 * 4


def num_threads() -> int:
    return lib().dgo_num_threads()


def e4m3_decode(code: int) -> float:
    return lib().dgo_e4m3_decode(int(code))


def e4m3_encode(y: float) -> int:
    return lib().dgo_e4m3_encode_satrne(float(y))


def e4m3_table() -> np.ndarray:
    """fp64 value of every e4m3 code (NaN for the two NaN codes)."""
    return np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)


def cast_per_token(x_bf16: np.ndarray):
    """x [M,K] bf16 bits -> (q [M,K] uint8, sfa [Kb, pad4(M)] fp32; padding entries 0)."""
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    q = np.empty((M, K), np.uint8)
    sfa = np.zeros((K // 128, pad4(M)), np.float32)
    _check(lib().dgo_cast_per_token(_p(x), M, K, _p(q), _p(sfa)), "cast_per_token")
    return q, sfa


def cast_per_token_scatter(x_bf16: np.ndarray, dst: np.ndarray, M_sum: int, q_init=None, sfa_init=None):
    """Per-token cast of x [T,K] written at rows dst[t] of the contiguous layout: returns
    (q [M_sum,K] uint8, sfa [Kb, pad4(M_sum)] fp32), starting from q_init / sfa_init (zeros when
    None) for the rows no token maps to."""
    x = _c(x_bf16, np.uint16)
    T, K = x.shape
    d = _c(dst, np.int32)
    q = np.zeros((M_sum, K), np.uint8) if q_init is None else np.array(q_init, np.uint8, copy=True)
    sfa = np.zeros((K // 128, pad4(M_sum)), np.float32) if sfa_init is None else np.array(sfa_init, np.float32,
                                                                                           copy=True)
    _check(lib().dgo_cast_per_token_scatter(_p(x), _p(d), T, K, M_sum, _p(q), _p(sfa)), "cast_per_token_scatter")
    return q, sfa


def cast_per_block(x_bf16: np.ndarray):
    """x [N,K] or [G,N,K] bf16 bits -> (q same shape, sfb [G?, ceil(N/128), Kb] fp32)."""
    x = _c(x_bf16, np.uint16)
    squeeze = x.ndim == 2
    if squeeze:
        x = x[None]
    G, N, K = x.shape
    q = np.empty((G, N, K), np.uint8)
    sfb = np.empty((G, (N + 127) // 128, K // 128), np.float32)
    _check(lib().dgo_cast_per_block(_p(x), G, N, K, _p(q), _p(sfb)), "cast_per_block")
    return (q[0], sfb[0]) if squeeze else (q, sfb)


def transform_sf(sf_kmajor: np.ndarray) -> np.ndarray:
    """[MN, Kb] or [B, MN, Kb] fp32 -> [Kb, pad4(MN)] or [B, Kb, pad4(MN)] (tail zero)."""
    s = _c(sf_kmajor, np.float32)
    squeeze = s.ndim == 2
    if squeeze:
        s = s[None]
    B, MN, Kb = s.shape
    out = np.empty((B, Kb, pad4(MN)), np.float32)
    _check(lib().dgo_transform_sf(_p(s), B, MN, Kb, _p(out)), "transform_sf")
    return out[0] if squeeze else out


def gemm_nt(a, sfa, b, sfb, c=None, rows=None) -> np.ndarray:
    """fp64 D (or the listed rows of D) for the dense block-scaled NT GEMM."""
    a = _c(a, np.uint8); b = _c(b, np.uint8)
    sfa = _c(sfa, np.float32); sfb = _c(sfb, np.float32); c = _c(c, np.uint16)
    M, K = a.shape
    N = b.shape[0]
    assert sfa.shape == (K // 128, pad4(M)), sfa.shape
    assert sfb.shape == ((N + 127) // 128, K // 128), sfb.shape
    r = None if rows is None else _c(rows, np.int32)
    R = M if r is None else r.shape[0]
    out = np.empty((R, N), np.float64)
    _check(lib().dgo_gemm_nt(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), M, N, K, _p(r), R, _p(out)),
           "gemm_nt")
    return out


def m_grouped_contiguous(a, sfa, b, sfb, grouped_layout, c=None, rows=None) -> np.ndarray:
    a = _c(a, np.uint8); b = _c(b, np.uint8)
    sfa = _c(sfa, np.float32); sfb = _c(sfb, np.float32); c = _c(c, np.uint16)
    gl = _c(grouped_layout, np.int32)
    M_sum, K = a.shape
    G, N, _ = b.shape
    r = None if rows is None else _c(rows, np.int32)
    R = M_sum if r is None else r.shape[0]
    out = np.empty((R, N), np.float64)
    _check(lib().dgo_m_grouped_contiguous(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), _p(gl), M_sum, N, K,
                                          G, _p(r), R, _p(out)), "m_grouped_contiguous")
    return out


def m_grouped_masked(a, sfa, b, sfb, masked_m, c=None) -> np.ndarray:
    a = _c(a, np.uint8); b = _c(b, np.uint8)
    sfa = _c(sfa, np.float32); sfb = _c(sfb, np.float32); c = _c(c, np.uint16)
    mm = _c(masked_m, np.int32)
    G, M_max, K = a.shape
    N = b.shape[1]
    out = np.empty((G, M_max, N), np.float64)
    _check(lib().dgo_m_grouped_masked(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), _p(mm), G, M_max, N, K,
                                      _p(out)), "m_grouped_masked")
    return out


def tolerance_ok(d: np.ndarray, ref: np.ndarray, rel: float = 2.0 ** -7, abs_rms: float = 1e-2):
    """Per-element bound |D - ref| <= rel·|ref| + abs_rms·rms(ref); returns (ok, worst ratio)."""
    ref = np.asarray(ref, np.float64)
    d = np.asarray(d, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    bound = rel * np.abs(ref) + abs_rms * rms
    err = np.abs(d - ref)
    ratio = float(np.max(err / np.maximum(bound, 1e-300))) if ref.size else 0.0
    return bool(np.all(err <= bound)), ratio


def gemm_layout(a, sfa, b, sfb, layout: str, c=None, rows=None) -> np.ndarray:
    """fp64 D for the dense block-scaled GEMM in the layouts the pages name ([likun] §一/§二:
    fp8_gemm_{nt,nn,tn,tt}). The first letter is A's storage, the second B's:
      A "n": [M,K] (K contiguous)    A "t": [K,M] (M contiguous)
      B "t": [N,K] (K contiguous)    B "n": [K,N] (N contiguous)
    so that D[m,n] = C[m,n] + sum_k A_log[m,k]·B_log[n,k] with the same scales in every layout
    (sfa [Kb][pad4(M)] per 1x128 slice of A along K, sfb [Nb][Kb] per 128x128 block). Moving an
    operand from MN-major to K-major storage is a transpose (data movement only), after which
    the NT definition applies."""
    layout = layout.lower()
    assert layout in ("nt", "nn", "tn", "tt"), layout
    a = np.asarray(a)
    b = np.asarray(b)
    a_k = np.ascontiguousarray(a.T) if layout[0] == "t" else a
    b_k = np.ascontiguousarray(b.T) if layout[1] == "n" else b
    return gemm_nt(a_k, sfa, b_k, sfb, c, rows=rows)


def cast_per_channel(x_bf16: np.ndarray):
    """x [T,C] bf16 bits (T % 128 == 0) -> (q [T,C] uint8, sf [T/128, pad4(C)] fp32): one scale
    per channel per 128-token block (the recipe (1,1,128) of the K-grouped GEMM)."""
    x = _c(x_bf16, np.uint16)
    T, C = x.shape
    q = np.empty((T, C), np.uint8)
    sf = np.zeros((T // 128, pad4(C)), np.float32)
    _check(lib().dgo_cast_per_channel(_p(x), T, C, _p(q), _p(sf)), "cast_per_channel")
    return q, sf


def k_grouped_tn(a, sfa, b, sfb, ks, c=None) -> np.ndarray:
    """fp64 D [G,M,N] of the K-grouped TN GEMM: a [sum_K, M], b [sum_K, N] e4m3 codes,
    sfa [sum_K/128, pad4(M)], sfb [sum_K/128, pad4(N)] fp32, ks [G] group sizes (multiples of
    128), c fp32 [G,M,N] or None."""
    a = _c(a, np.uint8); b = _c(b, np.uint8)
    sfa = _c(sfa, np.float32); sfb = _c(sfb, np.float32); c = _c(c, np.float32)
    ks = _c(ks, np.int32)
    G = ks.shape[0]
    M, N = a.shape[1], b.shape[1]
    assert a.shape[0] == b.shape[0] == int(ks.sum()), (a.shape, b.shape, ks)
    assert sfa.shape == (a.shape[0] // 128, pad4(M)) and sfb.shape == (b.shape[0] // 128, pad4(N))
    out = np.empty((G, M, N), np.float64)
    _check(lib().dgo_k_grouped_tn(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), _p(ks), G, M, N, _p(out)),
           "k_grouped_tn")
    return out


# ------------------------------------------------------------------------------------------
# UE8M0 (power-of-two) scales ([likun] §五: packed UE8M0 on SM100, four per 32-bit word)
# ------------------------------------------------------------------------------------------

def ue8m0_of_amax(amax: float) -> int:
    return int(lib().dgo_ue8m0_of_amax(float(amax)))


def cast_per_token_ue8m0(x_bf16: np.ndarray):
    """x [M,K] bf16 bits -> (q [M,K] uint8, sfa packed uint32 [ceil(Kb/4), pad4(M)])."""
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    Kb = K // 128
    q = np.empty((M, K), np.uint8)
    sf = np.zeros(((Kb + 3) // 4, pad4(M)), np.uint32)
    _check(lib().dgo_cast_per_token_ue8m0(_p(x), M, K, _p(q), _p(sf)), "cast_per_token_ue8m0")
    return q, sf


def cast_per_block_ue8m0(x_bf16: np.ndarray):
    """x [N,K] or [G,N,K] bf16 bits -> (q same shape, sfb packed uint32 [G?, Nb, ceil(Kb/4)])."""
    x = _c(x_bf16, np.uint16)
    squeeze = x.ndim == 2
    if squeeze:
        x = x[None]
    G, N, K = x.shape
    Kb = K // 128
    q = np.empty((G, N, K), np.uint8)
    sf = np.empty((G, (N + 127) // 128, (Kb + 3) // 4), np.uint32)
    _check(lib().dgo_cast_per_block_ue8m0(_p(x), G, N, K, _p(q), _p(sf)), "cast_per_block_ue8m0")
    return (q[0], sf[0]) if squeeze else (q, sf)


def ue8m0_bytes_to_f32(b) -> np.ndarray:
    """Scale values 2^(byte - 127) of UE8M0 bytes."""
    return np.ldexp(np.float32(1.0), np.asarray(b, np.int32) - 127).astype(np.float32)


def unpack_sfa_ue8m0(packed: np.ndarray, Kb: int) -> np.ndarray:
    """[ceil(Kb/4), ld] packed words -> fp32 [Kb, ld]: K block kb is byte kb % 4 of word kb // 4."""
    p = np.asarray(packed, np.uint32)
    kb = np.arange(Kb)
    bytes_ = (p[kb // 4] >> (8 * (kb % 4))[:, None].astype(np.uint32)) & 0xFF
    return ue8m0_bytes_to_f32(bytes_)


def unpack_sfb_ue8m0(packed: np.ndarray, Kb: int) -> np.ndarray:
    """[G?, Nb, ceil(Kb/4)] packed words -> fp32 [G?, Nb, Kb]."""
    p = np.asarray(packed, np.uint32)
    kb = np.arange(Kb)
    bytes_ = (p[..., kb // 4] >> (8 * (kb % 4)).astype(np.uint32)) & 0xFF
    return ue8m0_bytes_to_f32(bytes_)


def gemm_nt_ue8m0(a, sfa_packed, b, sfb_packed, c=None, rows=None) -> np.ndarray:
    """fp64 D of the NT GEMM with UE8M0 scales: the same definition as gemm_nt, the scales
    being the powers of two the packed bytes encode."""
    K = np.asarray(a).shape[1]
    Kb = K // 128
    return gemm_nt(a, unpack_sfa_ue8m0(sfa_packed, Kb), b, unpack_sfb_ue8m0(sfb_packed, Kb), c, rows=rows)
