"""Pins of the oracle's layout variants and of its K-grouped GEMM.

- fp8_gemm_{nt,nn,tn,tt} (likun.im/craft/deepgemm §一, "fp8_fp4_gemm_{nt,nn,tn,tt}"; §二
  "同类: _nn / _tn / _tt"): the first letter is A's storage ("n" = [M,K], "t" = [K,M]), the
  second B's ("t" = [N,K], "n" = [K,N]); the product and the scales are those of the NT GEMM.
- k_grouped_fp8_gemm_tn_contiguous (likun.im §一, "沿 K 轴分组的 k_grouped_fp8_gemm_tn（MoE 反向）";
  §二, ks_cpu and recipe (1,1,128)): the K dimension (tokens) is cut into groups, A [sum_K, M]
  and B [sum_K, N] are token-major, one scale per channel per 128 tokens.

Each pin is independent of the oracle's own code: exact rational brute force over
torch-decoded codes, closed forms, and reduction to the already-pinned NT oracle and
per-token cast through a transposition."""
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


def pow2(rng, shape, lo=-3, hi=3):
    return np.ldexp(1.0, rng.integers(lo, hi + 1, size=shape)).astype(np.float32)


# ------------------------------------------------------------------------------------------
# layouts
# ------------------------------------------------------------------------------------------

def brute_layout(a, sfa, b, sfb, layout, M, N, K, c=None):
    """Rational D[m,n] = C + sum_kb sfa[kb,m]·sfb[n/128,kb]·sum_k A_log[m,k]·B_log[n,k], with the
    stored index of each operand written out per layout."""
    av, bv = torch_decode(a), torch_decode(b)
    A = (lambda m, k: av[m, k]) if layout[0] == "n" else (lambda m, k: av[k, m])
    B = (lambda n, k: bv[n, k]) if layout[1] == "t" else (lambda n, k: bv[k, n])
    out = np.empty((M, N))
    for m in range(M):
        for n in range(N):
            tot = Fraction(0)
            for kb in range(K // 128):
                s = sum(Fraction(float(A(m, k))) * Fraction(float(B(n, k))) for k in range(kb * 128, kb * 128 + 128))
                tot += Fraction(float(sfa[kb, m])) * Fraction(float(sfb[n // 128, kb])) * s
            if c is not None:
                tot += Fraction(float(synth.bf16_bits_to_f32(c[m, n])))
            out[m, n] = float(tot)
    return out


@pytest.mark.parametrize("layout", ["nt", "nn", "tn", "tt"])
@pytest.mark.parametrize("M,N,K,seed", [(3, 5, 256, 0), (2, 130, 128, 1)])
def test_layouts_brute_force(oracle, layout, M, N, K, seed):
    rng = np.random.default_rng(seed)
    a_log, b_log = rand_codes(rng, (M, K)), rand_codes(rng, (N, K))
    a = a_log if layout[0] == "n" else np.ascontiguousarray(a_log.T)
    b = b_log if layout[1] == "t" else np.ascontiguousarray(b_log.T)
    sfa = np.zeros((K // 128, pad4(M)), np.float32)
    sfa[:, :M] = rng.uniform(0.01, 3, (K // 128, M)).astype(np.float32)
    sfb = rng.uniform(0.01, 3, ((N + 127) // 128, K // 128)).astype(np.float32)
    c = synth.normal_bf16(7 + seed, (M, N), sigma=0.1)
    for cc in (None, c):
        d = oracle.gemm_layout(a, sfa, b, sfb, layout, cc)
        ref = brute_layout(a, sfa, b, sfb, layout, M, N, K, cc)
        assert np.allclose(d, ref, rtol=1e-14, atol=0), layout


def test_layout_letters_are_not_interchangeable(oracle):
    """A square problem whose A is not symmetric: reading a stored operand in the other layout
    changes the result (a swapped letter would go unnoticed otherwise)."""
    rng = np.random.default_rng(5)
    M = N = K = 128
    a, b = rand_codes(rng, (M, K)), rand_codes(rng, (N, K))
    sfa = np.ones((1, M), np.float32)
    sfb = np.ones((1, 1), np.float32)
    outs = {lay: oracle.gemm_layout(a, sfa, b, sfb, lay) for lay in ("nt", "nn", "tn", "tt")}
    for x in outs:
        for y in outs:
            if x != y:
                assert not np.allclose(outs[x], outs[y])


# ------------------------------------------------------------------------------------------
# per-channel cast (recipe (1,1,128) along the token dimension)
# ------------------------------------------------------------------------------------------

def test_per_channel_cast_is_the_per_token_cast_of_the_transpose(oracle):
    """Quantising every channel over 128-token blocks is the per-token cast (pinned on its own)
    of the transposed tensor: the same codes, transposed back, and the same scale array."""
    T, C = 384, 200
    x = synth.normal_bf16(11, (T, C))
    q, sf = oracle.cast_per_channel(x)
    qt, sft = oracle.cast_per_token(np.ascontiguousarray(x.T))
    assert np.array_equal(q, qt.T)
    assert np.array_equal(sf, sft)


def test_per_channel_cast_amax_and_zero_block(oracle):
    T, C = 256, 8
    x = synth.normal_bf16(12, (T, C))
    x[128:, 3] = 0                                    # an all-zero block of one channel
    q, sf = oracle.cast_per_channel(x)
    xf = synth.bf16_bits_to_f32(x)
    for tb in range(2):
        for c in range(C):
            blk = xf[tb * 128:(tb + 1) * 128, c]
            if tb == 1 and c == 3:
                assert sf[tb, c] == 1.0 and np.all(q[128:, 3] == 0)
                continue
            i = int(np.argmax(np.abs(blk)))
            assert q[tb * 128 + i, c] in (0x7E, 0xFE)          # the amax element maps to +-448
            assert np.float32(sf[tb, c]) == np.float32(np.abs(blk).max()) / np.float32(448)


# ------------------------------------------------------------------------------------------
# K-grouped TN GEMM
# ------------------------------------------------------------------------------------------

def brute_k_grouped(a, sfa, b, sfb, ks, M, N, c=None):
    av, bv = torch_decode(a), torch_decode(b)
    G = len(ks)
    out = np.empty((G, M, N))
    k0 = 0
    for g in range(G):
        for m in range(M):
            for n in range(N):
                tot = Fraction(0)
                for kb in range(k0 // 128, (k0 + ks[g]) // 128):
                    s = sum(Fraction(float(av[k, m])) * Fraction(float(bv[k, n])) for k in range(kb * 128, kb * 128 + 128))
                    tot += Fraction(float(sfa[kb, m])) * Fraction(float(sfb[kb, n])) * s
                if c is not None:
                    tot += Fraction(float(c[g, m, n]))
                out[g, m, n] = float(tot)
        k0 += ks[g]
    return out


@pytest.mark.parametrize("ks,M,N,seed", [([128, 0, 256], 3, 5, 0), ([256], 2, 6, 1), ([128, 128], 5, 3, 2)])
def test_k_grouped_brute_force(oracle, ks, M, N, seed):
    rng = np.random.default_rng(seed)
    T = sum(ks)
    a, b = rand_codes(rng, (T, M)), rand_codes(rng, (T, N))
    sfa = np.zeros((T // 128, pad4(M)), np.float32)
    sfb = np.zeros((T // 128, pad4(N)), np.float32)
    sfa[:, :M] = rng.uniform(0.01, 3, (T // 128, M)).astype(np.float32)
    sfb[:, :N] = rng.uniform(0.01, 3, (T // 128, N)).astype(np.float32)
    c = rng.normal(size=(len(ks), M, N)).astype(np.float32)
    for cc in (None, c):
        d = oracle.k_grouped_tn(a, sfa, b, sfb, np.array(ks), cc)
        ref = brute_k_grouped(a, sfa, b, sfb, ks, M, N, cc)
        assert np.allclose(d, ref, rtol=1e-14, atol=0)


def test_k_grouped_closed_form(oracle):
    """All-ones operands (code 0x38 = 1.0) with constant scales: D[g] = ks[g]·s_a·s_b + C[g]."""
    ks = [256, 128, 0, 384]
    T, M, N = sum(ks), 4, 12
    a = np.full((T, M), 0x38, np.uint8)
    b = np.full((T, N), 0x38, np.uint8)
    sfa = np.full((T // 128, pad4(M)), 0.375, np.float32)
    sfb = np.full((T // 128, pad4(N)), 1.25, np.float32)
    c = np.arange(len(ks) * M * N, dtype=np.float32).reshape(len(ks), M, N)
    d = oracle.k_grouped_tn(a, sfa, b, sfb, np.array(ks), c)
    for g, k in enumerate(ks):
        assert np.array_equal(d[g], k * 0.375 * 1.25 + c[g].astype(np.float64))


def test_k_grouped_equals_per_group_nt_gemms(oracle):
    """With B's scales constant over each 128-channel block, group g is the (pinned) dense NT
    GEMM of the transposed token slices: D[g] = A_gᵀ·B_g with sfa_g and the block scales."""
    rng = np.random.default_rng(9)
    ks = [256, 128, 384]
    T, M, N = sum(ks), 130, 260
    a, b = rand_codes(rng, (T, M)), rand_codes(rng, (T, N))
    sfa = np.zeros((T // 128, pad4(M)), np.float32)
    sfa[:, :M] = rng.uniform(0.01, 3, (T // 128, M)).astype(np.float32)
    Nb = (N + 127) // 128
    blk = rng.uniform(0.01, 3, (Nb, T // 128)).astype(np.float32)     # [Nb][Kb] over all tokens
    sfb = np.zeros((T // 128, pad4(N)), np.float32)
    for n in range(N):
        sfb[:, n] = blk[n // 128]
    d = oracle.k_grouped_tn(a, sfa, b, sfb, np.array(ks))
    k0 = 0
    for g, k in enumerate(ks):
        kb0, kb1 = k0 // 128, (k0 + k) // 128
        ref = oracle.gemm_nt(np.ascontiguousarray(a[k0:k0 + k].T), np.ascontiguousarray(sfa[kb0:kb1]),
                             np.ascontiguousarray(b[k0:k0 + k].T), np.ascontiguousarray(blk[:, kb0:kb1]))
        assert np.array_equal(d[g], ref)
        k0 += k


def test_k_grouped_scale_is_per_channel(oracle):
    """Doubling sfb of one channel n in one token block doubles exactly that block's share of
    column n and nothing else (catches a scale indexed by the wrong channel or block)."""
    rng = np.random.default_rng(10)
    ks = [256]
    T, M, N = 256, 3, 7
    a, b = rand_codes(rng, (T, M)), rand_codes(rng, (T, N))
    sfa = np.zeros((2, pad4(M)), np.float32)
    sfa[:, :M] = pow2(rng, (2, M))
    sfb = np.zeros((2, pad4(N)), np.float32)
    sfb[:, :N] = pow2(rng, (2, N))
    d0 = oracle.k_grouped_tn(a, sfa, b, sfb, np.array(ks))
    sfb2 = sfb.copy()
    sfb2[1, 4] *= 2
    d1 = oracle.k_grouped_tn(a, sfa, b, sfb2, np.array(ks))
    sfb_only1 = np.zeros_like(sfb)
    sfb_only1[1] = sfb[1]
    share = oracle.k_grouped_tn(a, sfa, b, sfb_only1, np.array(ks))     # block 1's share
    diff = d1 - d0
    assert np.array_equal(diff[:, :, 4], share[:, :, 4])
    assert np.all(diff[:, :, [0, 1, 2, 3, 5, 6]] == 0)


def test_k_grouped_rejects_unaligned_groups(oracle):
    a = np.zeros((256, 4), np.uint8)
    with pytest.raises(ValueError):
        oracle.k_grouped_tn(a, np.ones((2, 4), np.float32), a, np.ones((2, 4), np.float32), np.array([100, 156]))
