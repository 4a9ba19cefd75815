"""ctypes binding of ``include/dg.h``: the same entry points with the same argument order.

Each function accepts torch tensors (their ``data_ptr()`` is passed), plain integers (device
addresses) or None for optional pointers, and ``stream`` as a ``torch.cuda.Stream``, a raw
``cudaStream_t`` integer or None (the current torch stream). Nothing here computes anything:
every step runs in the CUDA library, and a non-OK status raises ``DgError``.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_PATH = os.path.join(HERE, "libdg_b200.so")
HEADER = os.path.join(ROOT, "include", "dg.h")

STATUS = {0: "DG_OK", 1: "DG_ERR_INVALID_ARG", 2: "DG_ERR_ALIGNMENT", 3: "DG_ERR_UNSUPPORTED",
          4: "DG_ERR_CUDA", 5: "DG_ERR_TIMEOUT", 6: "DG_ERR_DEVICE"}
DG_OK, DG_ERR_INVALID_ARG, DG_ERR_ALIGNMENT, DG_ERR_UNSUPPORTED = 0, 1, 2, 3
DG_ERR_CUDA, DG_ERR_TIMEOUT, DG_ERR_DEVICE = 4, 5, 6


class DgError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


_lib = None


def declared_functions():
    """Names of the functions that ``include/dg.h`` exports (lines starting with DG_API)."""
    text = open(HEADER).read()
    return re.findall(r"^DG_API\s+[^(]*?\b(dg_\w+)\s*\(", text, flags=re.M)


def load():
    """Loads libdg_b200.so; raises if it has not been built (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m moe_grouped_gemm_sm_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        P, I = ctypes.c_void_p, ctypes.c_int
        sig = {
            "dg_fp8_gemm_nt": [P, P, P, P, P, P, I, I, I, P],
            "dg_fp8_gemm_nt_noalloc": [P, P, P, P, P, P, I, I, I, P],
            "dg_m_grouped_fp8_gemm_nt_contiguous": [P, P, P, P, P, P, P, I, I, I, I, P],
            "dg_m_grouped_fp8_gemm_nt_masked": [P, P, P, P, P, P, P, I, I, I, I, I, P],
            "dg_transform_sf": [P, P, I, I, I, P],
            "dg_cast_fp8_per_token": [P, P, P, I, I, I, P],
            "dg_cast_fp8_per_block": [P, P, P, I, I, I, P],
            "dg_cast_fp8_per_channel": [P, P, P, I, I, P],
            "dg_cast_fp8_per_token_ue8m0": [P, P, P, I, I, I, P],
            "dg_cast_fp8_per_token_scatter": [P, P, P, P, I, I, I, P],
            "dg_cast_fp8_per_block_ue8m0": [P, P, P, I, I, I, P],
            "dg_sf_ld": [I],
            "dg_get_device_error": [P],
            "dg_status_string": [I],
            "dg_fp8_gemm_nt_ue8m0": [P, P, P, P, P, P, I, I, I, P],
            "dg_fp8_gemm_nn": [P, P, P, P, P, P, I, I, I, P],
            "dg_fp8_gemm_tn": [P, P, P, P, P, P, I, I, I, P],
            "dg_fp8_gemm_tt": [P, P, P, P, P, P, I, I, I, P],
            "dg_k_grouped_fp8_gemm_tn_contiguous": [P, P, P, P, P, P, P, P, I, I, I, P],
            "dg_last_kernel": [],
            "dg_last_launch_count": [],
            "dg_allocated_bytes": [],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = {"dg_status_string": ctypes.c_char_p, "dg_last_kernel": ctypes.c_char_p,
                         "dg_allocated_bytes": ctypes.c_longlong}.get(name, I)
        _lib = L
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _call(name, *args):
    rc = getattr(load(), name)(*args)
    if rc != DG_OK:
        raise DgError(name, rc)


def dg_fp8_gemm_nt(a, sfa, b, sfb, c, d, M, N, K, stream=None):
    _call("dg_fp8_gemm_nt", _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(c), _ptr(d), M, N, K, _stream(stream))


def dg_fp8_gemm_nt_noalloc(a, sfa, b, sfb, c, d, M, N, K, stream=None):
    _call("dg_fp8_gemm_nt_noalloc", _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(c), _ptr(d), M, N, K,
          _stream(stream))


def dg_fp8_gemm_nt_ue8m0(a, sfa, b, sfb, c, d, M, N, K, stream=None):
    _call("dg_fp8_gemm_nt_ue8m0", _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(c), _ptr(d), M, N, K, _stream(stream))


def dg_fp8_gemm_nn(a, sfa, b, sfb, c, d, M, N, K, stream=None):
    _call("dg_fp8_gemm_nn", _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(c), _ptr(d), M, N, K, _stream(stream))


def dg_fp8_gemm_tn(a, sfa, b, sfb, c, d, M, N, K, stream=None):
    _call("dg_fp8_gemm_tn", _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(c), _ptr(d), M, N, K, _stream(stream))


def dg_fp8_gemm_tt(a, sfa, b, sfb, c, d, M, N, K, stream=None):
    _call("dg_fp8_gemm_tt", _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(c), _ptr(d), M, N, K, _stream(stream))


def dg_k_grouped_fp8_gemm_tn_contiguous(a, sfa, b, sfb, c, d, ks, ks_device, G, M, N, stream=None):
    """``ks`` is a sequence of G host integers (passed as a C int array), ``ks_device`` the same
    values in an int32 device tensor."""
    arr = (ctypes.c_int * len(ks))(*[int(k) for k in ks])
    _call("dg_k_grouped_fp8_gemm_tn_contiguous", _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(c), _ptr(d),
          ctypes.cast(arr, ctypes.c_void_p), _ptr(ks_device), G, M, N, _stream(stream))


def dg_m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, c, d, grouped_layout, M_sum, N, K, G, stream=None):
    _call("dg_m_grouped_fp8_gemm_nt_contiguous", _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(c), _ptr(d),
          _ptr(grouped_layout), M_sum, N, K, G, _stream(stream))


def dg_m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, c, d, masked_m, expected_m, G, M_max, N, K, stream=None):
    _call("dg_m_grouped_fp8_gemm_nt_masked", _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(c), _ptr(d),
          _ptr(masked_m), expected_m, G, M_max, N, K, _stream(stream))


def dg_transform_sf(sf_kmajor, sf_mnmajor, batch, MN, Kb, stream=None):
    _call("dg_transform_sf", _ptr(sf_kmajor), _ptr(sf_mnmajor), batch, MN, Kb, _stream(stream))


def dg_cast_fp8_per_token(x, q, sfa, batch, M, K, stream=None):
    _call("dg_cast_fp8_per_token", _ptr(x), _ptr(q), _ptr(sfa), batch, M, K, _stream(stream))


def dg_cast_fp8_per_block(x, q, sfb, batch, N, K, stream=None):
    _call("dg_cast_fp8_per_block", _ptr(x), _ptr(q), _ptr(sfb), batch, N, K, _stream(stream))


def dg_cast_fp8_per_token_scatter(x, dst_rows, q, sfa, T, M_sum, K, stream=None):
    _call("dg_cast_fp8_per_token_scatter", _ptr(x), _ptr(dst_rows), _ptr(q), _ptr(sfa), T, M_sum, K, _stream(stream))


def dg_cast_fp8_per_token_ue8m0(x, q, sfa, batch, M, K, stream=None):
    _call("dg_cast_fp8_per_token_ue8m0", _ptr(x), _ptr(q), _ptr(sfa), batch, M, K, _stream(stream))


def dg_cast_fp8_per_block_ue8m0(x, q, sfb, batch, N, K, stream=None):
    _call("dg_cast_fp8_per_block_ue8m0", _ptr(x), _ptr(q), _ptr(sfb), batch, N, K, _stream(stream))


def dg_cast_fp8_per_channel(x, q, sf, T, C, stream=None):
    _call("dg_cast_fp8_per_channel", _ptr(x), _ptr(q), _ptr(sf), T, C, _stream(stream))


def dg_sf_ld(mn: int) -> int:
    return load().dg_sf_ld(mn)


def dg_get_device_error(stream=None) -> int:
    """Status code (0 = DG_OK) of the device error word; reading it clears it."""
    return load().dg_get_device_error(_stream(stream))


def dg_status_string(status: int) -> str:
    return load().dg_status_string(status).decode()


def dg_last_kernel() -> str:
    """Name of the GEMM kernel the calling thread's last GEMM call launched."""
    return load().dg_last_kernel().decode()


def dg_last_launch_count() -> int:
    """Number of kernels the calling thread's last GEMM call launched."""
    return int(load().dg_last_launch_count())


def dg_allocated_bytes() -> int:
    """Device memory (bytes) the library has allocated with cudaMalloc so far."""
    return int(load().dg_allocated_bytes())
