"""GPU parity of the K-grouped TN GEMM of the MoE weight gradient (likun.im/craft/deepgemm §一,
"沿 K 轴分组的 k_grouped_fp8_gemm_tn（MoE 反向）"; §二, k_grouped_fp8_gemm_tn_contiguous with
ks_cpu and recipe (1,1,128)) and of its per-channel cast, against the oracle: the cast bit-exact,
the GEMM element by element within |D - ref| <= 2^-7·|ref| + 1e-2·rms(ref)."""
import numpy as np
import pytest
import torch

from moe_grouped_gemm_sm_b200 import _lib, build, synth
from tests.gpu_util import assert_close, bf16_dev, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def per_channel(x_bits):
    T, C = x_bits.shape
    x = bf16_dev(x_bits)
    q = torch.empty((T, C), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((T // 128, (C + 3) // 4 * 4), dtype=torch.float32, device="cuda")
    _lib.dg_cast_fp8_per_channel(x, q, sf, T, C)
    return q, sf


@pytest.mark.parametrize("T,C", [(128, 8), (384, 200), (1024, 4096), (256, 7168)])
def test_per_channel_cast_bit_exact(oracle, T, C):
    x = synth.normal_bf16(31 + C, (T, C))
    x[:128, 3] = 0                                          # an all-zero block: s = 1, codes 0
    q, sf = per_channel(x)
    torch.cuda.synchronize()
    qo, sfo = oracle.cast_per_channel(x)
    assert np.array_equal(host(q), qo)
    assert np.array_equal(host(sf)[:, :C], sfo[:, :C])


def kgrouped_case(oracle, ks, M, N, with_c, salt):
    T = int(sum(ks))
    dy = synth.normal_bf16(synth.seed_for(synth.BASE_SEED, synth.STREAM_A, salt), (T, M))
    x = synth.normal_bf16(synth.seed_for(synth.BASE_SEED, synth.STREAM_B, salt), (T, N))
    a, sfa = per_channel(dy)
    b, sfb = per_channel(x)
    ao, sfao = oracle.cast_per_channel(dy)
    bo, sfbo = oracle.cast_per_channel(x)
    assert np.array_equal(host(a), ao) and np.array_equal(host(b), bo)
    c = np.random.default_rng(salt).normal(size=(len(ks), M, N)).astype(np.float32) if with_c else None
    return (a, sfa, b, sfb, dev(c) if c is not None else None), (ao, sfao, bo, sfbo, c)


def run(ks, dv, M, N, d=None):
    a, sfa, b, sfb, c = dv
    G = len(ks)
    if d is None:
        d = torch.full((G, M, N), -7.0, dtype=torch.float32, device="cuda")
    _lib.dg_k_grouped_fp8_gemm_tn_contiguous(a, sfa, b, sfb, c, d, list(ks), dev(np.array(ks, np.int32)), G, M, N)
    return d


@pytest.mark.parametrize("ks,M,N", [([256, 0, 384, 128], 256, 384), ([128], 128, 128), ([384, 256], 208, 272),
                                    ([128, 128, 128], 512, 2112), ([640], 64, 4096)])
@pytest.mark.parametrize("with_c", [False, True])
def test_k_grouped_full_compare(oracle, ks, M, N, with_c):
    dv, hv = kgrouped_case(oracle, ks, M, N, with_c, salt=M + N + len(ks))
    d = run(ks, dv, M, N)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_OK
    ref = oracle.k_grouped_tn(*hv[:4], np.array(ks), hv[4])
    got = host(d).astype(np.float64)
    for g in range(len(ks)):
        if ks[g] == 0:                                      # an empty group: D = C exactly
            expect = hv[4][g].astype(np.float64) if with_c else np.zeros((M, N))
            assert np.array_equal(got[g], expect)
        else:
            assert_close(got[g], ref[g], f"k-grouped ks={ks} M={M} N={N} group {g}")


def test_k_grouped_c_aliases_d_and_is_deterministic(oracle):
    ks, M, N = [256, 128], 256, 256
    dv, hv = kgrouped_case(oracle, ks, M, N, True, salt=3)
    d = dv[4].clone()
    run(ks, (*dv[:4], d), M, N, d=d)                         # accumulate into the gradient in place
    d2 = run(ks, dv, M, N)
    torch.cuda.synchronize()
    assert torch.equal(d, d2)
    ref = oracle.k_grouped_tn(*hv[:4], np.array(ks), hv[4])
    for g in range(len(ks)):
        assert_close(host(d)[g].astype(np.float64), ref[g], f"in-place group {g}")


@pytest.mark.slow
@pytest.mark.parametrize("M,N", [(4096, 7168), (7168, 2048)])
def test_k_grouped_page_shape_sampled_rows(oracle, M, N):
    """The MoE weight gradient of the page's expert shapes: G = 8 groups of U{2048..6144}
    tokens padded to 128; rows of D checked on a sample (a row of D depends only on its column
    of A, so the oracle runs on those columns)."""
    m, layout = synth.contiguous_layout(8, salt=200 + N)
    ks = [int((k + 127) // 128 * 128) for k in m]
    dv, hv = kgrouped_case(oracle, ks, M, N, False, salt=200 + N)
    d = run(ks, dv, M, N)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_OK
    rows = np.array(sorted({0, 127, 128, 255, M - 1} | set(np.random.default_rng(N).integers(0, M, 3).tolist())))
    ao, sfao, bo, sfbo, _ = hv
    a_s = np.ascontiguousarray(ao[:, rows])
    sfa_s = np.zeros((sfao.shape[0], (len(rows) + 3) // 4 * 4), np.float32)
    sfa_s[:, :len(rows)] = sfao[:, rows]
    ref = oracle.k_grouped_tn(a_s, sfa_s, bo, sfbo, np.array(ks))
    got = host(d)
    for g in range(8):
        assert_close(got[g][rows].astype(np.float64), ref[g], f"k-grouped {M}x{N} group {g}")


def test_k_grouped_bad_device_group_size_sets_the_error_word(oracle):
    """The device copy of ks disagrees with the host's (not a multiple of 128): the group is
    computed as empty and DG_ERR_DEVICE is reported; the other groups are exact."""
    ks, M, N = [256, 128], 128, 128
    dv, hv = kgrouped_case(oracle, ks, M, N, False, salt=9)
    a, sfa, b, sfb, _ = dv
    d = torch.full((2, M, N), -7.0, dtype=torch.float32, device="cuda")
    assert _lib.dg_get_device_error() == _lib.DG_OK
    _lib.dg_k_grouped_fp8_gemm_tn_contiguous(a, sfa, b, sfb, None, d, ks, dev(np.array([100, 284], np.int32)), 2, M, N)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_ERR_DEVICE
    got = host(d)
    assert np.all(got[0] == 0)                              # group 0 empty: D = C = 0
    # group 1 read as 284 tokens from offset 0 is also rejected (not a multiple of 128)
    assert np.all(got[1] == 0)


def test_k_grouped_rejects_unaligned_host_sizes():
    a = torch.zeros((256, 128), dtype=torch.uint8, device="cuda")
    sf = torch.ones((2, 128), dtype=torch.float32, device="cuda")
    d = torch.empty((1, 128, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(_lib.DgError) as e:
        _lib.dg_k_grouped_fp8_gemm_tn_contiguous(a, sf, a, sf, None, d, [200], dev(np.array([200], np.int32)), 1,
                                                 128, 128)
    assert e.value.status == _lib.DG_ERR_INVALID_ARG
