"""torch-tensor conveniences over the C ABI: they allocate outputs with torch and pass
pointers. All arithmetic happens in libdg_b200.so.

Layouts (see include/dg.h): e4m3 tensors are torch.uint8 holding the codes; ``sfa`` is fp32
[batch?][Kb][pad4(M)] (MN-major), ``sfb`` fp32 [G?][ceil(N/128)][Kb]; C and D are bf16.
"""
from __future__ import annotations

import torch

from . import _lib


def _pad4(x: int) -> int:
    return (x + 3) // 4 * 4


def _check_cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensors must live on a CUDA device")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")


def cast_per_token(x: torch.Tensor, stream=None):
    """bf16 [M,K] or [batch,M,K] -> (e4m3 codes uint8 same shape, sfa fp32 [batch?][Kb][pad4(M)])."""
    _check_cuda(x)
    assert x.dtype == torch.bfloat16
    squeeze = x.dim() == 2
    xb = x.unsqueeze(0) if squeeze else x
    B, M, K = xb.shape
    q = torch.empty((B, M, K), dtype=torch.uint8, device=x.device)
    sfa = torch.zeros((B, K // 128, _pad4(M)), dtype=torch.float32, device=x.device)
    _lib.dg_cast_fp8_per_token(xb, q, sfa, B, M, K, stream)
    return (q[0], sfa[0]) if squeeze else (q, sfa)


def cast_per_block(w: torch.Tensor, stream=None):
    """bf16 [N,K] or [G,N,K] -> (e4m3 codes uint8 same shape, sfb fp32 [G?][ceil(N/128)][Kb])."""
    _check_cuda(w)
    assert w.dtype == torch.bfloat16
    squeeze = w.dim() == 2
    wb = w.unsqueeze(0) if squeeze else w
    G, N, K = wb.shape
    q = torch.empty((G, N, K), dtype=torch.uint8, device=w.device)
    sfb = torch.empty((G, (N + 127) // 128, K // 128), dtype=torch.float32, device=w.device)
    _lib.dg_cast_fp8_per_block(wb, q, sfb, G, N, K, stream)
    return (q[0], sfb[0]) if squeeze else (q, sfb)


def transform_sf(sf_kmajor: torch.Tensor, stream=None) -> torch.Tensor:
    """fp32 [MN,Kb] or [batch,MN,Kb] -> [Kb,pad4(MN)] or [batch,Kb,pad4(MN)]."""
    _check_cuda(sf_kmajor)
    squeeze = sf_kmajor.dim() == 2
    s = sf_kmajor.unsqueeze(0) if squeeze else sf_kmajor
    B, MN, Kb = s.shape
    out = torch.empty((B, Kb, _pad4(MN)), dtype=torch.float32, device=s.device)
    _lib.dg_transform_sf(s, out, B, MN, Kb, stream)
    return out[0] if squeeze else out


def fp8_gemm_nt(a, sfa, b, sfb, c=None, out=None, stream=None) -> torch.Tensor:
    """D = C + A·Bᵀ; a [M,K] codes, b [N,K] codes; returns bf16 [M,N]."""
    _check_cuda(a, sfa, b, sfb, c, out)
    M, K = a.shape
    N = b.shape[0]
    d = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    _lib.dg_fp8_gemm_nt(a, sfa, b, sfb, c, d, M, N, K, stream)
    return d


def m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, grouped_layout, c=None, out=None, stream=None):
    """a [M_sum,K], b [G,N,K], grouped_layout int32 [M_sum]; returns bf16 [M_sum,N]."""
    _check_cuda(a, sfa, b, sfb, grouped_layout, c, out)
    M_sum, K = a.shape
    G, N, _ = b.shape
    d = out if out is not None else torch.empty((M_sum, N), dtype=torch.bfloat16, device=a.device)
    _lib.dg_m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, c, d, grouped_layout, M_sum, N, K, G, stream)
    return d


def m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, masked_m, expected_m, c=None, out=None, stream=None):
    """a [G,M_max,K], b [G,N,K], masked_m int32 [G] (device); returns bf16 [G,M_max,N]
    (rows >= masked_m[g] keep whatever ``out`` held)."""
    _check_cuda(a, sfa, b, sfb, masked_m, c, out)
    G, M_max, K = a.shape
    N = b.shape[1]
    d = out if out is not None else torch.empty((G, M_max, N), dtype=torch.bfloat16, device=a.device)
    _lib.dg_m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, c, d, masked_m, expected_m, G, M_max, N, K, stream)
    return d
