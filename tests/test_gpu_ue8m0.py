"""GPU parity of the UE8M0 (power-of-two scale) path against the oracle: the casts bit-exact
(codes and packed scale words), the block-scaled-MMA GEMM element by element within
|D - ref| <= 2^-7·|ref| + 1e-2·rms(ref). likun.im/craft/deepgemm §五 (SM100: packed UE8M0, four
per 32-bit word) and §二 (disable_ue8m0_cast)."""
import numpy as np
import pytest
import torch

from moe_grouped_gemm_sm_b200 import _lib, build, synth
from tests.gpu_util import assert_close, bf16_dev, bf16_host_f64, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def cast_token(x_bits):
    M, K = x_bits.shape
    Kq = (K // 128 + 3) // 4
    q = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((Kq, (M + 3) // 4 * 4), dtype=torch.int32, device="cuda")
    _lib.dg_cast_fp8_per_token_ue8m0(bf16_dev(x_bits), q, sf, 1, M, K)
    return q, sf


def cast_block(w_bits):
    N, K = w_bits.shape
    Kq = (K // 128 + 3) // 4
    q = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    sf = torch.zeros(((N + 127) // 128, Kq), dtype=torch.int32, device="cuda")
    _lib.dg_cast_fp8_per_block_ue8m0(bf16_dev(w_bits), q, sf, 1, N, K)
    return q, sf


def words(t):
    return host(t).view(np.uint32)


@pytest.mark.parametrize("M,K", [(1, 128), (33, 640), (128, 512), (300, 7168), (4096, 1536)])
def test_per_token_ue8m0_cast_bit_exact(oracle, M, K):
    x = synth.normal_bf16(M + K, (M, K))
    x[0, :128] = 0                                          # a zero slice: byte 127, codes 0
    q, sf = cast_token(x)
    torch.cuda.synchronize()
    qo, sfo = oracle.cast_per_token_ue8m0(x)
    assert np.array_equal(host(q), qo)
    assert np.array_equal(words(sf)[:, :M], sfo[:, :M])


@pytest.mark.parametrize("N,K", [(128, 128), (2112, 640), (256, 7168), (7168, 512)])
def test_per_block_ue8m0_cast_bit_exact(oracle, N, K):
    w = synth.normal_bf16(N * 3 + K, (N, K))
    q, sf = cast_block(w)
    torch.cuda.synchronize()
    qo, sfo = oracle.cast_per_block_ue8m0(w)
    assert np.array_equal(host(q), qo)
    assert np.array_equal(words(sf), sfo)


def operands(oracle, M, N, K, with_c, salt):
    x, w, c = synth.dense_inputs(M, N, K, with_c, salt=salt)
    a, sfa = cast_token(x)
    b, sfb = cast_block(w)
    ao, sfao = oracle.cast_per_token_ue8m0(x)
    bo, sfbo = oracle.cast_per_block_ue8m0(w)
    assert np.array_equal(host(a), ao) and np.array_equal(host(b), bo)
    return (a, sfa, b, sfb, bf16_dev(c) if c is not None else None), (ao, sfao, bo, sfbo, c)


SHAPES = [(128, 224, 256), (256, 448, 512), (200, 2112, 1024), (64, 256, 128), (1000, 7168, 2048),
          (384, 4096, 384), (130, 16, 128)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("with_c", [False, True])
def test_ue8m0_gemm_full_compare(oracle, M, N, K, with_c):
    dv, hv = operands(oracle, M, N, K, with_c, salt=M + N + K)
    a, sfa, b, sfb, c = dv
    d = torch.full((M, N), -3.0, dtype=torch.bfloat16, device="cuda")
    _lib.dg_fp8_gemm_nt_ue8m0(a, sfa, b, sfb, c, d, M, N, K)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_OK
    ref = oracle.gemm_nt_ue8m0(*hv)
    assert_close(bf16_host_f64(d), ref, f"ue8m0 {M}x{N}x{K} c={with_c}")


def test_ue8m0_gemm_prefill_shape_sampled_and_deterministic(oracle):
    M, N, K = 4096, 7168, 7168
    dv, hv = operands(oracle, M, N, K, True, salt=77)
    a, sfa, b, sfb, c = dv
    d1 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    d2 = torch.empty_like(d1)
    _lib.dg_fp8_gemm_nt_ue8m0(a, sfa, b, sfb, c, d1, M, N, K)
    _lib.dg_fp8_gemm_nt_ue8m0(a, sfa, b, sfb, c, d2, M, N, K)
    torch.cuda.synchronize()
    assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))
    rows = np.array(sorted({0, 31, 32, 127, 128, 1000, 2047, 4095} |
                           set(np.random.default_rng(5).integers(0, M, 8).tolist())), np.int32)
    ref = oracle.gemm_nt_ue8m0(*hv[:4], hv[4], rows=rows)
    assert_close(bf16_host_f64(d1)[rows], ref, "ue8m0 4096x7168x7168")


def test_ue8m0_c_aliases_d(oracle):
    M, N, K = 256, 448, 1024
    dv, hv = operands(oracle, M, N, K, True, salt=12)
    a, sfa, b, sfb, c = dv
    d = c.clone()
    _lib.dg_fp8_gemm_nt_ue8m0(a, sfa, b, sfb, d, d, M, N, K)
    torch.cuda.synchronize()
    assert_close(bf16_host_f64(d), oracle.gemm_nt_ue8m0(*hv), "ue8m0 c aliases d")


def test_ue8m0_rejects_n_not_multiple_of_16():
    M, N, K = 128, 136, 128
    a = torch.zeros((M, K), dtype=torch.uint8, device="cuda")
    sfa = torch.zeros((1, M), dtype=torch.int32, device="cuda")
    b = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    sfb = torch.zeros((2, 1), dtype=torch.int32, device="cuda")
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_lib.DgError) as e:
        _lib.dg_fp8_gemm_nt_ue8m0(a, sfa, b, sfb, None, d, M, N, K)
    assert e.value.status == _lib.DG_ERR_INVALID_ARG
