"""GPU parity of the M-grouped contiguous and masked GEMMs (likun.im/craft/deepgemm §二;
zwt0204.github.io "DeepGEMM deep dive", grouped and masked layouts) against the oracle.
Masked: D is pre-filled with the 0xDEAD sentinel and every row >= masked_m[g] must keep it."""
import numpy as np
import pytest
import torch

from moe_grouped_gemm_sm_b200 import _lib, build, ops, synth
from tests.gpu_util import assert_close, bf16_dev, bf16_host_f64, dev, host

pytestmark = pytest.mark.gpu

SENTINEL = np.uint16(synth.sentinel_bf16())


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def sentinel_d(shape):
    arr = np.full(shape, SENTINEL, np.uint16)
    return bf16_dev(arr)


def contiguous_case(oracle, G, N, K, lo, hi, with_c, salt):
    m, layout, x, w = synth.contiguous_inputs(G, N, K, lo=lo, hi=hi, salt=salt)
    a, sfa = ops.cast_per_token(bf16_dev(x))
    b, sfb = ops.cast_per_block(bf16_dev(w))
    ao, sfao = oracle.cast_per_token(x)
    bo, sfbo = oracle.cast_per_block(w)
    assert np.array_equal(host(a), ao) and np.array_equal(host(b), bo)
    c = synth.normal_bf16(salt + 99, (layout.shape[0], N), sigma=0.1) if with_c else None
    return m, layout, (a, sfa, b, sfb, dev(layout), bf16_dev(c) if c is not None else None), (ao, sfao, bo, sfbo, layout, c)


@pytest.mark.parametrize("G,N,K,lo,hi", [(1, 128, 128, 1, 128), (3, 264, 256, 100, 300), (4, 2112, 384, 129, 260),
                                         (8, 136, 1024, 1, 400)])
@pytest.mark.parametrize("with_c", [False, True])
def test_contiguous_small(oracle, G, N, K, lo, hi, with_c):
    m, layout, dv, hv = contiguous_case(oracle, G, N, K, lo, hi, with_c, salt=G * 100 + N)
    a, sfa, b, sfb, gl, c = dv
    d = ops.m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, gl, c)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_OK
    ao, sfao, bo, sfbo, lay, ch = hv
    ref = oracle.m_grouped_contiguous(ao, sfao, bo, sfbo, lay, ch)
    valid = lay >= 0
    assert_close(bf16_host_f64(d)[valid], ref[valid], f"contiguous G={G} N={N} K={K}")


def test_contiguous_skips_padding_only_block(oracle):
    """A 128-row block whose first row is -1 is skipped: its D rows keep their old contents."""
    m, layout, dv, hv = contiguous_case(oracle, 2, 256, 256, 130, 200, False, salt=5)
    a, sfa, b, sfb, gl, _ = dv
    lay = layout.copy()
    lay[128:256] = -1                                          # second block of expert 0 -> padding
    d = sentinel_d((lay.shape[0], 256))
    ops.m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, dev(lay), None, out=d)
    torch.cuda.synchronize()
    dh = host(d.view(torch.int16)).view(np.uint16)
    assert np.all(dh[128:256] == SENTINEL)
    ref = oracle.m_grouped_contiguous(hv[0], hv[1], hv[2], hv[3], lay)
    valid = lay >= 0
    assert_close(bf16_host_f64(d)[valid], ref[valid], "contiguous with a skipped block")


def masked_case(oracle, G, M_max, N, K, lo, hi, with_c, salt):
    masked_m, x, w = synth.masked_inputs(G, M_max, N, K, lo=lo, hi=hi, salt=salt)
    a, sfa = ops.cast_per_token(bf16_dev(x))
    b, sfb = ops.cast_per_block(bf16_dev(w))
    ao = np.empty((G, M_max, K), np.uint8)
    sfao = np.empty((G, K // 128, (M_max + 3) // 4 * 4), np.float32)
    for g in range(G):
        ao[g], sfao[g] = oracle.cast_per_token(x[g])
    bo, sfbo = oracle.cast_per_block(w)
    assert np.array_equal(host(a), ao) and np.array_equal(host(sfa), sfao)
    c = synth.normal_bf16(salt + 7, (G, M_max, N), sigma=0.1) if with_c else None
    return masked_m, (a, sfa, b, sfb, bf16_dev(c) if c is not None else None), (ao, sfao, bo, sfbo, c)


def check_masked(oracle, masked_m, dv, hv, G, M_max, N, expected_m, what):
    a, sfa, b, sfb, c = dv
    d = sentinel_d((G, M_max, N))
    ops.m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, dev(masked_m), expected_m, c, out=d)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_OK
    ref = oracle.m_grouped_masked(hv[0], hv[1], hv[2], hv[3], masked_m, hv[4])
    dh16 = host(d.view(torch.int16)).view(np.uint16)
    df = bf16_host_f64(d)
    for g in range(G):
        mm = int(masked_m[g])
        assert np.all(dh16[g, mm:] == SENTINEL), f"{what}: expert {g} wrote rows >= masked_m"
        if mm:
            assert_close(df[g, :mm], ref[g, :mm], f"{what} expert {g}")


@pytest.mark.parametrize("G,M_max,N,K,lo,hi", [(2, 64, 128, 128, 1, 64), (4, 256, 264, 256, 0, 256),
                                               (3, 300, 2112, 384, 100, 300), (16, 256, 136, 512, 64, 256)])
@pytest.mark.parametrize("with_c", [False, True])
def test_masked_small(oracle, G, M_max, N, K, lo, hi, with_c):
    masked_m, dv, hv = masked_case(oracle, G, M_max, N, K, lo, hi, with_c, salt=G * 10 + N + K)
    check_masked(oracle, masked_m, dv, hv, G, M_max, N, 192, f"masked G={G} N={N} K={K}")


@pytest.mark.parametrize("expected_m,kernel", [(32, "gemm_kernel"), (128, "gemm_kernel"),
                                               (192, "gemm_kernel (CTA pairs)"), (0, "gemm_kernel (CTA pairs)")])
def test_masked_expected_m_picks_the_tile(oracle, expected_m, kernel):
    """expected_m <= 128 takes 128-row tiles, above it 256-row CTA-pair tiles (0: M_max decides);
    both give the oracle's result on the same experts, and rows >= masked_m keep the sentinel."""
    G, M_max, N, K = 6, 256, 520, 384
    masked_m, dv, hv = masked_case(oracle, G, M_max, N, K, 0, 256, True, salt=61)
    check_masked(oracle, masked_m, dv, hv, G, M_max, N, expected_m, f"masked expected_m={expected_m}")
    assert _lib.dg_last_kernel() == kernel


def test_masked_edge_counts(oracle):
    """masked_m of 0, 1, 31, 32, 33, 127, 128, 129 and M_max: partial warp slabs and tiles."""
    G, M_max, N, K = 9, 160, 264, 256
    masked_m, dv, hv = masked_case(oracle, G, M_max, N, K, 0, 160, False, salt=4)
    masked_m[:] = [0, 1, 31, 32, 33, 127, 128, 129, 160]
    check_masked(oracle, masked_m, dv, hv, G, M_max, N, 64, "masked edge counts")


@pytest.mark.slow
@pytest.mark.parametrize("N,K", [(4096, 7168), (7168, 2048)])
def test_contiguous_page_shapes_sampled(oracle, N, K):
    G = 8
    m, layout, dv, hv = contiguous_case(oracle, G, N, K, 2048, 6144, False, salt=N)
    a, sfa, b, sfb, gl, c = dv
    d = ops.m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, gl, c)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_OK
    rows = []
    for t in range(0, layout.shape[0], 128):
        blk = np.nonzero(layout[t:t + 128] >= 0)[0]
        if blk.size:
            rows += [t + int(blk[0]), t + int(blk[-1])]
    rng = np.random.default_rng(N * 7 + K)
    valid_rows = np.nonzero(layout >= 0)[0]
    rows = np.array(sorted(set(rows[::3] + rng.choice(valid_rows, 16).tolist())), np.int32)
    ao, sfao, bo, sfbo, lay, _ = hv
    ref = oracle.m_grouped_contiguous(ao, sfao, bo, sfbo, lay, None, rows=rows)
    assert_close(bf16_host_f64(d)[rows], ref, f"contiguous G=8 N={N} K={K}")


@pytest.mark.slow
@pytest.mark.parametrize("N,K", [(4096, 7168), (7168, 2048)])
def test_masked_page_shapes(oracle, N, K):
    G, M_max = 16, 256
    masked_m, dv, hv = masked_case(oracle, G, M_max, N, K, 64, 256, False, salt=N + 1)
    a, sfa, b, sfb, c = dv
    d = sentinel_d((G, M_max, N))
    ops.m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, dev(masked_m), 192, c, out=d)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_OK
    dh16 = host(d.view(torch.int16)).view(np.uint16)
    df = bf16_host_f64(d)
    ao, sfao, bo, sfbo, _ = hv
    ref = oracle.m_grouped_masked(ao, sfao, bo, sfbo, masked_m)    # every valid row of every expert
    for g in range(G):
        mm = int(masked_m[g])
        assert np.all(dh16[g, mm:] == SENTINEL)
        assert_close(df[g, :mm], ref[g, :mm], f"masked G=16 N={N} K={K} expert {g}")
