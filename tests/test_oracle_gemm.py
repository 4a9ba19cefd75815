"""Pins of the oracle's GEMMs: D = C + A·Bᵀ in NT layout (likun.im/craft/deepgemm §一) with
block-wise scales (aitangshan.cn/news/1491278 技术原理 §4), and the M-grouped contiguous /
masked variants (likun.im §二; zwt0204.github.io "DeepGEMM deep dive", §"它的核心思路")."""
from fractions import Fraction

import numpy as np
import pytest
import torch

from moe_grouped_gemm_sm_b200 import synth


def torch_decode(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def rand_codes(rng, shape):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x3C                 # no NaN codes
    return c


def pad4(x):
    return (x + 3) // 4 * 4


def exact_reference(a, sfa, b, sfb, c=None):
    """Rational arithmetic: C + sum_kb sfa·sfb·sum_k a·b, with operand values from torch."""
    M, K = a.shape
    N = b.shape[0]
    av, bv = torch_decode(a), torch_decode(b)
    out = np.empty((M, N))
    for m in range(M):
        for n in range(N):
            tot = Fraction(0)
            for kb in range(K // 128):
                s = sum(Fraction(float(av[m, k])) * Fraction(float(bv[n, k]))
                        for k in range(kb * 128, kb * 128 + 128))
                tot += Fraction(float(sfa[kb, m])) * Fraction(float(sfb[n // 128, kb])) * s
            if c is not None:
                tot += Fraction(float(synth.bf16_bits_to_f32(c[m, n])))
            out[m, n] = float(tot)
    return out


@pytest.mark.parametrize("M,N,K,seed", [(1, 1, 128, 0), (3, 4, 256, 1), (4, 2, 384, 2)])
def test_brute_force_tiny(oracle, M, N, K, seed):
    rng = np.random.default_rng(seed)
    a, b = rand_codes(rng, (M, K)), rand_codes(rng, (N, K))
    sfa = np.zeros((K // 128, pad4(M)), np.float32)
    sfa[:, :M] = rng.uniform(0.01, 3, (K // 128, M)).astype(np.float32)
    sfb = rng.uniform(0.01, 3, ((N + 127) // 128, K // 128)).astype(np.float32)
    c = synth.normal_bf16(100 + seed, (M, N), sigma=0.1)
    for cc in (None, c):
        d = oracle.gemm_nt(a, sfa, b, sfb, cc)
        ref = exact_reference(a, sfa, b, sfb, cc)
        assert np.allclose(d, ref, rtol=1e-14, atol=0), (d, ref)


def test_closed_form_all_ones(oracle):
    M, N, K = 5, 130, 512
    a = np.full((M, K), 0x38, np.uint8)          # e4m3 1.0
    b = np.full((N, K), 0x38, np.uint8)
    sa, sb = np.float32(0.375), np.float32(2.5)
    sfa = np.full((K // 128, pad4(M)), sa, np.float32)
    sfb = np.full((2, K // 128), sb, np.float32)
    d = oracle.gemm_nt(a, sfa, b, sfb)
    assert np.all(d == K * float(sa) * float(sb))


def test_identity_selector_pins_indices(oracle):
    """A[m,k] = 1 at k = m only: D[m,n] = sfa[m, m/128]·sfb[n/128, m/128]·B[n,m]. A swapped
    operand, a transposed scale or a wrong K-block index changes the result."""
    M, N, K = 256, 260, 384
    rng = np.random.default_rng(5)
    a = np.zeros((M, K), np.uint8)
    a[np.arange(M), np.arange(M)] = 0x38
    b = rand_codes(rng, (N, K))
    sfa = np.zeros((K // 128, pad4(M)), np.float32)
    sfa[:, :M] = rng.uniform(0.5, 2, (K // 128, M)).astype(np.float32)
    sfb = rng.uniform(0.5, 2, (3, K // 128)).astype(np.float32)
    d = oracle.gemm_nt(a, sfa, b, sfb)
    bv = torch_decode(b)
    m = np.arange(M)[:, None]
    n = np.arange(N)[None, :]
    expect = sfa[m // 128, m].astype(np.float64) * sfb[n // 128, m // 128] * bv[n, m]
    assert np.array_equal(d, expect)


def test_transpose_symmetry_with_block_constant_scales(oracle):
    """With sfa constant over 128-row blocks, swapping the operands transposes D exactly."""
    M, N, K = 136, 200, 256
    rng = np.random.default_rng(6)
    a, b = rand_codes(rng, (M, K)), rand_codes(rng, (N, K))
    blk_a = rng.uniform(0.5, 2, ((M + 127) // 128, K // 128)).astype(np.float32)
    blk_b = rng.uniform(0.5, 2, ((N + 127) // 128, K // 128)).astype(np.float32)
    sfa = np.zeros((K // 128, pad4(M)), np.float32)
    sfa[:, :M] = blk_a[np.arange(M) // 128].T
    sfb_as_sfa = np.zeros((K // 128, pad4(N)), np.float32)
    sfb_as_sfa[:, :N] = blk_b[np.arange(N) // 128].T
    d1 = oracle.gemm_nt(a, sfa, b, blk_b)
    d2 = oracle.gemm_nt(b, sfb_as_sfa, a, blk_a)
    assert np.array_equal(d1, d2.T)


def test_power_of_two_block_invariance(oracle):
    """Codes of one (row, K-block) times 2^j with that scale times 2^-j: D is bit-identical."""
    M, N, K = 6, 40, 384
    rng = np.random.default_rng(8)
    # codes with exponent field 3..10 so +-2 binades stay in the normal range
    e = rng.integers(3, 11, size=(M, K)).astype(np.uint8)
    mant = rng.integers(0, 8, size=(M, K)).astype(np.uint8)
    sign = rng.integers(0, 2, size=(M, K)).astype(np.uint8)
    a = (sign << 7) | (e << 3) | mant
    b = rand_codes(rng, (N, K))
    sfa = np.zeros((K // 128, pad4(M)), np.float32)
    sfa[:, :M] = (2.0 ** rng.integers(-8, 0, size=(K // 128, M))).astype(np.float32)
    sfb = rng.uniform(0.5, 2, (1, K // 128)).astype(np.float32)
    d0 = oracle.gemm_nt(a, sfa, b, sfb)
    for j in (2, -2):
        a2, s2 = a.copy(), sfa.copy()
        m, kb = 3, 1
        blk = a2[m, kb * 128:(kb + 1) * 128].copy()
        ex = ((blk >> 3) & 15).astype(np.int32) + j
        a2[m, kb * 128:(kb + 1) * 128] = (blk & 0x87) | (ex.astype(np.uint8) << 3)
        s2[kb, m] = s2[kb, m] * np.float32(2.0 ** -j)
        assert np.array_equal(torch_decode(a2[m, kb * 128:(kb + 1) * 128]),
                              torch_decode(blk) * 2.0 ** j)
        assert np.array_equal(oracle.gemm_nt(a2, s2, b, sfb), d0)


def test_c_addend_and_row_sampling(oracle):
    M, N, K = 40, 96, 256
    x = synth.normal_bf16(20, (M, K)); w = synth.normal_bf16(21, (N, K))
    a, sfa = oracle.cast_per_token(x)
    b, sfb = oracle.cast_per_block(w)
    c = synth.normal_bf16(22, (M, N), sigma=0.1)
    d0 = oracle.gemm_nt(a, sfa, b, sfb)
    dc = oracle.gemm_nt(a, sfa, b, sfb, c)
    assert np.allclose(dc - d0, synth.bf16_bits_to_f32(c).astype(np.float64), rtol=0, atol=1e-12)
    rows = np.array([39, 0, 17, 17], np.int32)
    assert np.array_equal(oracle.gemm_nt(a, sfa, b, sfb, c, rows=rows), dc[rows])


def test_dequantised_product_close_to_bf16_product(oracle):
    """The block-scaled product approximates the unquantised bf16 product (sanity of scales)."""
    M, N, K = 32, 64, 1024
    x = synth.normal_bf16(23, (M, K)); w = synth.normal_bf16(24, (N, K))
    a, sfa = oracle.cast_per_token(x)
    b, sfb = oracle.cast_per_block(w)
    d = oracle.gemm_nt(a, sfa, b, sfb)
    exact = synth.bf16_bits_to_f32(x).astype(np.float64) @ synth.bf16_bits_to_f32(w).astype(np.float64).T
    rel = np.sqrt(np.mean((d - exact) ** 2) / np.mean(exact ** 2))
    assert rel < 0.05, rel


def test_contiguous_equals_concatenated_dense(oracle):
    G, N, K = 3, 136, 256
    m, layout, x, w = synth.contiguous_inputs(G, N, K, lo=100, hi=300, salt=1)
    a, sfa = oracle.cast_per_token(x)
    b, sfb = oracle.cast_per_block(w)
    c = synth.normal_bf16(30, (layout.shape[0], N), sigma=0.1)
    d = oracle.m_grouped_contiguous(a, sfa, b, sfb, layout, c)
    off = 0
    for g in range(G):
        rows = np.arange(off, off + int(m[g]))
        ref = oracle.gemm_nt(a, sfa, b[g], sfb[g], c, rows=rows)
        assert np.array_equal(d[rows], ref)
        padded = (int(m[g]) + 127) // 128 * 128
        assert np.all(np.isnan(d[off + int(m[g]):off + padded]))
        off += padded
    assert off == layout.shape[0]
    sel = np.array([5, layout.shape[0] - 1, 130], np.int32)
    assert np.array_equal(oracle.m_grouped_contiguous(a, sfa, b, sfb, layout, c, rows=sel), d[sel],
                          equal_nan=True)


def test_masked_equals_per_expert_dense(oracle):
    G, M_max, N, K = 4, 96, 72, 256
    masked_m, x, w = synth.masked_inputs(G, M_max, N, K, lo=0, hi=96, salt=2)
    masked_m[0] = 0
    masked_m[1] = M_max
    a = np.empty((G, M_max, K), np.uint8)
    sfa = np.empty((G, K // 128, pad4(M_max)), np.float32)
    for g in range(G):
        a[g], sfa[g] = oracle.cast_per_token(x[g])
    b, sfb = oracle.cast_per_block(w)
    d = oracle.m_grouped_masked(a, sfa, b, sfb, masked_m)
    for g in range(G):
        mm = int(masked_m[g])
        ref = oracle.gemm_nt(a[g], sfa[g], b[g], sfb[g])
        assert np.array_equal(d[g, :mm], ref[:mm])
        assert np.all(np.isnan(d[g, mm:]))
    # garbage rows never influence valid rows: rewrite them and compare
    a2 = a.copy()
    for g in range(G):
        a2[g, int(masked_m[g]):] = 0x7E
    d2 = oracle.m_grouped_masked(a2, sfa, b, sfb, masked_m)
    assert np.array_equal(np.nan_to_num(d2, nan=7.0), np.nan_to_num(d, nan=7.0))


def test_masked_m_clamped(oracle):
    G, M_max, N, K = 2, 8, 16, 128
    rng = np.random.default_rng(9)
    a = rand_codes(rng, (G, M_max, K)); b = rand_codes(rng, (G, N, K))
    sfa = np.ones((G, 1, 8), np.float32); sfb = np.ones((G, 1, 1), np.float32)
    d = oracle.m_grouped_masked(a, sfa, b, sfb, np.array([-3, 99], np.int32))
    assert np.all(np.isnan(d[0])) and not np.any(np.isnan(d[1]))


def test_rejects_bad_arguments(oracle):
    with pytest.raises(ValueError):
        oracle.cast_per_token(np.zeros((2, 100), np.uint16))      # K not a multiple of 128
    a = np.zeros((2, 128), np.uint8)
    with pytest.raises(ValueError):
        oracle.gemm_nt(a, np.ones((1, 4), np.float32), a, np.ones((1, 1), np.float32),
                       rows=np.array([2], np.int32))              # row out of range
