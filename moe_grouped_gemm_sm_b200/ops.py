"""torch-tensor conveniences over the C ABI: they allocate outputs with torch and pass
pointers. All arithmetic happens in libdg_b200.so.

Layouts (see include/dg.h): e4m3 tensors are torch.uint8 holding the codes; ``sfa`` is fp32
[batch?][Kb][pad4(M)] (MN-major), ``sfb`` fp32 [G?][ceil(N/128)][Kb]; C and D are bf16 (fp32 for
the K-grouped GEMM); UE8M0 scales are int32 words of four packed bytes.

Each function checks that its tensors are contiguous CUDA tensors, allocates what it returns
(or writes ``out``) and makes one C-ABI call on ``stream`` (default: the current stream).
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


def cast_per_token_scatter(x, dst_rows, M_sum, stream=None):
    """bf16 [T,K] tokens and int32 [T] destination rows (device) -> (e4m3 [M_sum,K], sfa fp32
    [Kb][pad4(M_sum)]) in the contiguous grouped layout; rows no token maps to stay zero."""
    _check_cuda(x, dst_rows)
    assert x.dtype == torch.bfloat16 and dst_rows.dtype == torch.int32
    T, K = x.shape
    q = torch.zeros((M_sum, K), dtype=torch.uint8, device=x.device)
    sfa = torch.zeros((K // 128, _pad4(M_sum)), dtype=torch.float32, device=x.device)
    _lib.dg_cast_fp8_per_token_scatter(x, dst_rows, q, sfa, T, M_sum, K, stream)
    return q, sfa


def cast_per_token_ue8m0(x, stream=None):
    """bf16 [M,K] -> (e4m3 [M,K], packed UE8M0 sfa int32 [ceil(Kb/4)][pad4(M)])."""
    _check_cuda(x)
    assert x.dtype == torch.bfloat16
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    sfa = torch.zeros(((K // 128 + 3) // 4, _pad4(M)), dtype=torch.int32, device=x.device)
    _lib.dg_cast_fp8_per_token_ue8m0(x, q, sfa, 1, M, K, stream)
    return q, sfa


def cast_per_block_ue8m0(w, stream=None):
    """bf16 [N,K] -> (e4m3 [N,K], packed UE8M0 sfb int32 [ceil(N/128)][ceil(Kb/4)])."""
    _check_cuda(w)
    assert w.dtype == torch.bfloat16
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    sfb = torch.zeros(((N + 127) // 128, (K // 128 + 3) // 4), dtype=torch.int32, device=w.device)
    _lib.dg_cast_fp8_per_block_ue8m0(w, q, sfb, 1, N, K, stream)
    return q, sfb


def fp8_gemm_nt_ue8m0(a, sfa, b, sfb, c=None, out=None, stream=None) -> torch.Tensor:
    """D = C + A·Bᵀ with packed UE8M0 scales (cast_per_token_ue8m0 / cast_per_block_ue8m0)."""
    _check_cuda(a, sfa, b, sfb, c, out)
    M, K = a.shape
    N = b.shape[0]
    d = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    _lib.dg_fp8_gemm_nt_ue8m0(a, sfa, b, sfb, c, d, M, N, K, stream)
    return d


def fp8_gemm(layout, a, sfa, b, sfb, c=None, out=None, stream=None) -> torch.Tensor:
    """The dense GEMM in layout "nt", "nn", "tn" or "tt" (A then B: "n" = K contiguous for A,
    "t" = M contiguous; for B "t" = [N,K], "n" = [K,N]); sfa fp32 [Kb][pad4(M)], sfb fp32
    [ceil(N/128)][Kb] for the logical operands; returns bf16 [M,N]."""
    _check_cuda(a, sfa, b, sfb, c, out)
    if layout not in ("nt", "nn", "tn", "tt"):
        raise ValueError(f"layout {layout!r}")
    K, M = (a.shape[0], a.shape[1]) if layout[0] == "t" else (a.shape[1], a.shape[0])
    N = b.shape[1] if layout[1] == "n" else b.shape[0]
    d = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    getattr(_lib, "dg_fp8_gemm_" + layout)(a, sfa, b, sfb, c, d, M, N, K, stream)
    return d


def cast_per_channel(x, stream=None):
    """bf16 [T,C] token-major (T % 128 == 0) -> (e4m3 [T,C], sf fp32 [T/128][pad4(C)])."""
    _check_cuda(x)
    assert x.dtype == torch.bfloat16
    T, C = x.shape
    q = torch.empty((T, C), dtype=torch.uint8, device=x.device)
    sf = torch.zeros((T // 128, _pad4(C)), dtype=torch.float32, device=x.device)
    _lib.dg_cast_fp8_per_channel(x, q, sf, T, C, stream)
    return q, sf


def k_grouped_fp8_gemm_tn_contiguous(a, sfa, b, sfb, ks, c=None, out=None, stream=None) -> torch.Tensor:
    """a e4m3 [sum_K,M] and b e4m3 [sum_K,N] (token-major, from cast_per_channel), ks the G group
    sizes (host ints, multiples of 128); returns fp32 D [G,M,N] with D[g] = C[g] + A_gᵀ·B_g."""
    _check_cuda(a, sfa, b, sfb, c, out)
    ks = [int(k) for k in ks]
    M, N = a.shape[1], b.shape[1]
    ks_dev = torch.tensor(ks, dtype=torch.int32, device=a.device)
    d = out if out is not None else torch.empty((len(ks), M, N), dtype=torch.float32, device=a.device)
    _lib.dg_k_grouped_fp8_gemm_tn_contiguous(a, sfa, b, sfb, c, d, ks, ks_dev, len(ks), M, N, stream)
    return d
