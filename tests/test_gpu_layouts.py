"""GPU parity of the dense GEMM in the NN, TN and TT storage layouts (likun.im/craft/deepgemm
§一, "fp8_fp4_gemm_{nt,nn,tn,tt}"; §二, "同类: _nn / _tn / _tt") against the oracle, element by
element, within |D - ref| <= 2^-7·|ref| + 1e-2·rms(ref). The operands are the library's NT
casts (checked bit-exact against the oracle's), stored transposed where the layout says so."""
import numpy as np
import pytest
import torch

from moe_grouped_gemm_sm_b200 import _lib, build, ops, synth
from tests.gpu_util import assert_close, bf16_dev, bf16_host_f64, host

pytestmark = pytest.mark.gpu

ENTRY = {"nt": _lib.dg_fp8_gemm_nt, "nn": _lib.dg_fp8_gemm_nn, "tn": _lib.dg_fp8_gemm_tn, "tt": _lib.dg_fp8_gemm_tt}


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def operands(oracle, M, N, K, layout, with_c, salt):
    x, w, c = synth.dense_inputs(M, N, K, with_c, salt=salt)
    a, sfa = ops.cast_per_token(bf16_dev(x))
    b, sfb = ops.cast_per_block(bf16_dev(w))
    ao, sfao = oracle.cast_per_token(x)
    bo, sfbo = oracle.cast_per_block(w)
    assert np.array_equal(host(a), ao) and np.array_equal(host(b), bo)
    a_st = a.t().contiguous() if layout[0] == "t" else a          # A [K,M] for "t"
    b_st = b.t().contiguous() if layout[1] == "n" else b          # B [K,N] for "n"
    cd = bf16_dev(c) if c is not None else None
    return (a_st, sfa, b_st, sfb, cd), (host(a_st), sfao, host(b_st), sfbo, c)


SHAPES = [(128, 256, 256), (256, 384, 512), (64, 128, 384), (208, 272, 640), (512, 2112, 1024), (384, 4096, 256)]


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("with_c", [False, True])
def test_layout_full_compare(oracle, layout, M, N, K, with_c):
    dv, hv = operands(oracle, M, N, K, layout, with_c, salt=M + 3 * N + K)
    a, sfa, b, sfb, c = dv
    d = torch.full((M, N), -3.0, dtype=torch.bfloat16, device="cuda")
    ENTRY[layout](a, sfa, b, sfb, c, d, M, N, K)
    torch.cuda.synchronize()
    assert _lib.dg_get_device_error() == _lib.DG_OK
    ref = oracle.gemm_layout(*hv[:4], layout, hv[4])
    assert_close(bf16_host_f64(d), ref, f"{layout} {M}x{N}x{K} c={with_c}")


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
def test_layout_prefill_shape_sampled(oracle, layout):
    """A prefill-size problem (CTA pairs, several waves) on sampled rows."""
    M, N, K = 4096, 4096, 7168
    dv, hv = operands(oracle, M, N, K, layout, True, salt=17)
    a, sfa, b, sfb, c = dv
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ENTRY[layout](a, sfa, b, sfb, c, d, M, N, K)
    torch.cuda.synchronize()
    rows = np.array(sorted({0, 127, 128, 255, 1000, 2047, 2048, 4095} |
                           set(np.random.default_rng(K + len(layout)).integers(0, M, 8).tolist())), np.int32)
    a_k = np.ascontiguousarray(hv[0].T) if layout[0] == "t" else hv[0]
    b_k = np.ascontiguousarray(hv[2].T) if layout[1] == "n" else hv[2]
    ref = oracle.gemm_nt(a_k, hv[1], b_k, hv[3], hv[4], rows=rows)
    assert_close(bf16_host_f64(d)[rows], ref, f"{layout} 4096x4096x7168")


def test_layouts_agree_with_nt(oracle):
    """The four layouts compute the same product: within the bound of one another's oracle, and
    deterministic call after call."""
    M, N, K = 256, 512, 1024
    outs = {}
    for layout in ("nt", "nn", "tn", "tt"):
        dv, hv = operands(oracle, M, N, K, layout, True, salt=5)
        a, sfa, b, sfb, c = dv
        d1 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        d2 = torch.empty_like(d1)
        ENTRY[layout](a, sfa, b, sfb, c, d1, M, N, K)
        ENTRY[layout](a, sfa, b, sfb, c, d2, M, N, K)
        torch.cuda.synchronize()
        assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))
        outs[layout] = bf16_host_f64(d1)
    ref = oracle.gemm_layout(*operands(oracle, M, N, K, "nt", True, salt=5)[1][:4], "nt",
                             synth.dense_inputs(M, N, K, True, salt=5)[2])
    for layout, o in outs.items():
        assert_close(o, ref, f"{layout} vs the NT product")


def test_unaligned_mn_major_rows_are_rejected():
    M, N, K = 136, 256, 128                              # M % 16 != 0 with A MN-major
    a = torch.zeros((K, M), dtype=torch.uint8, device="cuda")
    sfa = torch.ones((1, 136), dtype=torch.float32, device="cuda")
    b = torch.zeros((K, N), dtype=torch.uint8, device="cuda")
    sfb = torch.ones((2, 1), dtype=torch.float32, device="cuda")
    d = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    for f in (_lib.dg_fp8_gemm_tn, _lib.dg_fp8_gemm_tt):
        with pytest.raises(_lib.DgError) as e:
            f(a, sfa, b, sfb, None, d, M, N, K)
        assert e.value.status == _lib.DG_ERR_INVALID_ARG
