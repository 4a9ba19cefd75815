"""GPU parity of the per-token cast written straight into the M-grouped contiguous layout (the
MoE dispatch in front of m_grouped_fp8_gemm_nt_contiguous, likun.im/craft/deepgemm §二), and of
that cast followed by the contiguous GEMM: the cast bit-exact against the oracle, the GEMM
within |D - ref| <= 2^-7·|ref| + 1e-2·rms(ref)."""
import numpy as np
import pytest
import torch

from moe_grouped_gemm_sm_b200 import _lib, build, ops, synth
from tests.gpu_util import assert_close, bf16_dev, bf16_host_f64, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def routing(G, lo, hi, salt):
    """Tokens in routing order (a seeded shuffle), each expert's tokens at the head of its
    128-aligned block of the contiguous layout: returns (dst_rows [T], grouped_layout [M_sum])."""
    m, layout = synth.contiguous_layout(G, lo, hi, salt=salt)
    rows = np.nonzero(layout >= 0)[0].astype(np.int32)          # rows that hold a token, by expert
    order = np.random.default_rng(salt).permutation(rows.size)
    dst = rows[order]                                             # token t -> its row
    return dst.astype(np.int32), layout


@pytest.mark.parametrize("G,K,lo,hi", [(3, 256, 1, 200), (8, 7168, 100, 400), (4, 2048, 129, 300)])
def test_scatter_cast_bit_exact(oracle, G, K, lo, hi):
    dst, layout = routing(G, lo, hi, salt=G + K)
    dst[::7] = -1                                                 # some dropped tokens
    T, M_sum = dst.size, layout.size
    x = synth.normal_bf16(G * K, (T, K))
    q = torch.full((M_sum, K), 0xAB, dtype=torch.uint8, device="cuda")
    sfa = torch.full((K // 128, (M_sum + 3) // 4 * 4), -1.0, dtype=torch.float32, device="cuda")
    _lib.dg_cast_fp8_per_token_scatter(bf16_dev(x), dev(dst), q, sfa, T, M_sum, K)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_OK
    qo, so = oracle.cast_per_token_scatter(x, dst, M_sum, np.full((M_sum, K), 0xAB, np.uint8),
                                           np.full((K // 128, (M_sum + 3) // 4 * 4), -1.0, np.float32))
    assert np.array_equal(host(q), qo)
    assert np.array_equal(host(sfa), so)


def test_scatter_cast_then_contiguous_gemm(oracle):
    G, N, K = 8, 1024, 2048
    dst, layout = routing(G, 100, 400, salt=5)
    T, M_sum = dst.size, layout.size
    x = synth.normal_bf16(61, (T, K))
    w = synth.normal_bf16(62, (G, N, K))
    b, sfb = ops.cast_per_block(bf16_dev(w))
    q = torch.zeros((M_sum, K), dtype=torch.uint8, device="cuda")
    sfa = torch.ones((K // 128, M_sum), dtype=torch.float32, device="cuda")
    _lib.dg_cast_fp8_per_token_scatter(bf16_dev(x), dev(dst), q, sfa, T, M_sum, K)
    d = ops.m_grouped_fp8_gemm_nt_contiguous(q, sfa, b, sfb, dev(layout))
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_OK
    qo, so = oracle.cast_per_token_scatter(x, dst, M_sum, np.zeros((M_sum, K), np.uint8),
                                           np.ones((K // 128, M_sum), np.float32))
    bo, sfbo = oracle.cast_per_block(w)
    rows = np.nonzero(layout >= 0)[0].astype(np.int32)
    ref = oracle.m_grouped_contiguous(qo, so, bo, sfbo, layout, None, rows=rows)
    assert_close(bf16_host_f64(d)[rows], ref, "scatter cast + contiguous GEMM")


def test_scatter_row_out_of_range_sets_the_error_word(oracle):
    T, K, M_sum = 4, 128, 128
    x = synth.normal_bf16(63, (T, K))
    dst = np.array([0, 200, 2, 3], np.int32)
    q = torch.zeros((M_sum, K), dtype=torch.uint8, device="cuda")
    sfa = torch.zeros((1, M_sum), dtype=torch.float32, device="cuda")
    assert _lib.dg_get_device_error() == _lib.DG_OK
    _lib.dg_cast_fp8_per_token_scatter(bf16_dev(x), dev(dst), q, sfa, T, M_sum, K)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_ERR_DEVICE
    qo, so = oracle.cast_per_token_scatter(x[[0, 2, 3]], np.array([0, 2, 3], np.int32), M_sum)
    assert np.array_equal(host(q), qo) and np.array_equal(host(sfa), so)
