"""Pins of the oracle's UE8M0 (power-of-two) scales: likun.im/craft/deepgemm §五 (on SM100 the
scales are packed UE8M0, four per 32-bit word) and §二 (disable_ue8m0_cast in the fp8 GEMM's
signature). Reading: s is the smallest power of two with s >= amax/448 (the fp32 quotient that
defines the fp32 scale), stored as its exponent + 127; q = e4m3(x / s) as for the fp32 scales;
four K blocks' bytes per word, K block kb at bits 8·(kb % 4)."""
from fractions import Fraction

import numpy as np
import pytest
import torch

from moe_grouped_gemm_sm_b200 import synth


def f32(x):
    return np.float32(x)


@pytest.mark.parametrize("amax", [448.0, 449.0, 1.0, 3.5, 896.0, 895.9, 1e-30, 2.0 ** -100, 6.0e4, 0.001953125])
def test_scale_is_the_smallest_power_of_two_at_least_amax_over_448(oracle, amax):
    b = oracle.ue8m0_of_amax(amax)
    s = 2.0 ** (b - 127)
    r = float(f32(amax) / f32(448.0))
    assert s >= r and s / 2 < r


def test_zero_block_and_exact_powers(oracle):
    assert oracle.ue8m0_of_amax(0.0) == 127
    for e in range(-20, 21):
        assert oracle.ue8m0_of_amax(448.0 * 2.0 ** e) == 127 + e     # r exactly 2^e: that power


def test_per_token_codes_are_the_exact_scaling(oracle):
    """x / s is exact (a power of two), so the codes are torch's float8 conversion of x·2^-e
    wherever no value saturates; the amax element lands in (224, 448]."""
    M, K = 33, 512
    x = synth.normal_bf16(7, (M, K))
    q, sf = oracle.cast_per_token_ue8m0(x)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    Kb = K // 128
    s = oracle.unpack_sfa_ue8m0(sf, Kb)[:, :M].T                   # [M, Kb]
    y = xf / np.repeat(s, 128, axis=1)
    assert np.all(np.abs(y) <= 448.0)
    ref = torch.from_numpy(y.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)
    for m in range(M):
        for kb in range(Kb):
            blk = np.abs(y[m, kb * 128:(kb + 1) * 128])
            assert 224.0 < blk.max() <= 448.0


def test_packing_four_per_word(oracle):
    """Byte t of word kq is K block 4·kq + t; bytes past the last K block are 127."""
    M, K = 5, 128 * 6
    x = synth.normal_bf16(8, (M, K))
    x = (x.astype(np.int32) + 0).astype(np.uint16)
    # give every K block a different magnitude so that a byte mix-up shows
    xf = synth.bf16_bits_to_f32(x).copy()
    for kb in range(6):
        xf[:, kb * 128:(kb + 1) * 128] *= 2.0 ** (3 * kb)
    x = synth.f32_to_bf16_bits(xf)
    q, sf = oracle.cast_per_token_ue8m0(x)
    assert sf.shape == (2, 8)
    for m in range(M):
        for kb in range(6):
            amax = np.abs(synth.bf16_bits_to_f32(x[m, kb * 128:(kb + 1) * 128])).max()
            assert (int(sf[kb // 4, m]) >> (8 * (kb % 4))) & 0xFF == oracle.ue8m0_of_amax(amax)
        assert (int(sf[1, m]) >> 16) & 0xFF == 127 and (int(sf[1, m]) >> 24) == 127


def test_per_block_matches_per_token_on_a_block_constant_tensor(oracle):
    """A weight whose 128x128 blocks each hold one row pattern repeated: the block's amax is
    its rows' amax, so the per-block scale equals the per-token scale of any of its rows."""
    N, K = 256, 384
    row = synth.normal_bf16(9, (1, K))
    w = np.repeat(row, N, axis=0)
    qb, sfb = oracle.cast_per_block_ue8m0(w)
    qt, sfa = oracle.cast_per_token_ue8m0(w)
    assert np.array_equal(qb, qt)
    Kb = K // 128
    ub = oracle.unpack_sfb_ue8m0(sfb, Kb)
    ua = oracle.unpack_sfa_ue8m0(sfa, Kb)
    for nb in range(2):
        assert np.array_equal(ub[nb], ua[:, 0])


def test_ue8m0_gemm_is_exact_rational(oracle):
    """With power-of-two scales every product and partial sum is exact: the oracle equals the
    rational value of the definition, element by element (catches an unpacking that reads the
    wrong block's scale)."""
    M, N, K = 3, 130, 640
    x = synth.normal_bf16(10, (M, K))
    w = synth.normal_bf16(11, (N, K))
    a, sfa = oracle.cast_per_token_ue8m0(x)
    b, sfb = oracle.cast_per_block_ue8m0(w)
    d = oracle.gemm_nt_ue8m0(a, sfa, b, sfb)
    av = torch.from_numpy(a).view(torch.float8_e4m3fn).double().numpy()
    bv = torch.from_numpy(b).view(torch.float8_e4m3fn).double().numpy()
    Kb = K // 128
    for m in range(M):
        for n in (0, 1, 127, 128, 129):
            tot = Fraction(0)
            for kb in range(Kb):
                sa = 2 ** ((int(sfa[kb // 4, m]) >> (8 * (kb % 4)) & 0xFF) - 127)
                sb = 2 ** ((int(sfb[n // 128, kb // 4]) >> (8 * (kb % 4)) & 0xFF) - 127)
                s = sum(Fraction(float(av[m, k])) * Fraction(float(bv[n, k])) for k in range(kb * 128, kb * 128 + 128))
                tot += Fraction(sa) * Fraction(sb) * s
            assert d[m, n] == float(tot)
