"""The torch conveniences of ``ops`` for the newer entry points (UE8M0 casts and GEMM, the NN /
TN / TT layouts, the per-channel cast and the K-grouped GEMM, the scattering cast), each against
the oracle: casts bit-exact, GEMMs within |D - ref| <= 2^-7·|ref| + 1e-2·rms(ref). They only
allocate and marshal; these tests pin their shapes and argument order."""
import numpy as np
import pytest
import torch

from moe_grouped_gemm_sm_b200 import build, ops, synth
from tests.gpu_util import assert_close, bf16_dev, bf16_host_f64, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def test_ops_ue8m0(oracle):
    M, N, K = 200, 272, 640
    x, w, c = synth.dense_inputs(M, N, K, True, salt=71)
    a, sfa = ops.cast_per_token_ue8m0(bf16_dev(x))
    b, sfb = ops.cast_per_block_ue8m0(bf16_dev(w))
    ao, sfao = oracle.cast_per_token_ue8m0(x)
    bo, sfbo = oracle.cast_per_block_ue8m0(w)
    assert np.array_equal(host(a), ao) and np.array_equal(host(b), bo)
    assert np.array_equal(host(sfa).view(np.uint32)[:, :M], sfao[:, :M])
    assert np.array_equal(host(sfb).view(np.uint32), sfbo)
    d = ops.fp8_gemm_nt_ue8m0(a, sfa, b, sfb, bf16_dev(c))
    torch.cuda.synchronize()
    assert_close(bf16_host_f64(d), oracle.gemm_nt_ue8m0(ao, sfao, bo, sfbo, c), "ops ue8m0")


@pytest.mark.parametrize("layout", ["nt", "nn", "tn", "tt"])
def test_ops_layouts(oracle, layout):
    M, N, K = 192, 272, 512
    x, w, c = synth.dense_inputs(M, N, K, True, salt=72)
    a, sfa = ops.cast_per_token(bf16_dev(x))
    b, sfb = ops.cast_per_block(bf16_dev(w))
    a_s = a.t().contiguous() if layout[0] == "t" else a          # stored operands of the layout
    b_s = b.t().contiguous() if layout[1] == "n" else b
    d = ops.fp8_gemm(layout, a_s, sfa, b_s, sfb, bf16_dev(c))
    torch.cuda.synchronize()
    ref = oracle.gemm_layout(host(a_s), host(sfa), host(b_s), host(sfb), layout, c)
    assert_close(bf16_host_f64(d), ref, f"ops layout {layout}")


def test_ops_k_grouped(oracle):
    ks, M, N = [256, 0, 384, 128], 96, 160
    T = sum(ks)
    dy = synth.normal_bf16(73, (T, M))
    xin = synth.normal_bf16(74, (T, N))
    a, sfa = ops.cast_per_channel(bf16_dev(dy))
    b, sfb = ops.cast_per_channel(bf16_dev(xin))
    ao, sfao = oracle.cast_per_channel(dy)
    bo, sfbo = oracle.cast_per_channel(xin)
    assert np.array_equal(host(a), ao) and np.array_equal(host(b), bo)
    assert np.array_equal(host(sfa)[:, :M], sfao[:, :M]) and np.array_equal(host(sfb)[:, :N], sfbo[:, :N])
    c = np.random.default_rng(75).normal(size=(len(ks), M, N)).astype(np.float32)
    d = ops.k_grouped_fp8_gemm_tn_contiguous(a, sfa, b, sfb, ks, c=dev(c))
    torch.cuda.synchronize()
    ref = oracle.k_grouped_tn(ao, sfao, bo, sfbo, np.array(ks, np.int32), c)
    assert_close(host(d).astype(np.float64), ref, "ops k-grouped")


def test_ops_scatter_cast(oracle):
    T, K, M_sum = 300, 384, 512
    x = synth.normal_bf16(76, (T, K))
    rng = np.random.default_rng(77)
    dst = np.full(T, -1, np.int32)
    keep = rng.choice(T, 250, replace=False)
    dst[keep] = rng.choice(M_sum, 250, replace=False).astype(np.int32)
    q, sfa = ops.cast_per_token_scatter(bf16_dev(x), dev(dst), M_sum)
    torch.cuda.synchronize()
    qo, sfo = oracle.cast_per_token_scatter(x, dst, M_sum, q_init=np.zeros((M_sum, K), np.uint8),
                                            sfa_init=np.zeros((K // 128, (M_sum + 3) // 4 * 4), np.float32))
    assert np.array_equal(host(q), qo)
    assert np.array_equal(host(sfa), sfo)
