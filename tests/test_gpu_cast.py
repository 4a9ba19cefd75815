"""GPU parity of the FP8 casts and the scale-layout transform: bit-exact against the oracle
(every e4m3 code, every fp32 scale), through the C ABI."""
import numpy as np
import pytest
import torch

from moe_grouped_gemm_sm_b200 import _lib, build, ops, synth
from tests.gpu_util import bf16_dev, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


@pytest.mark.parametrize("batch,M,K", [(1, 1, 128), (1, 37, 384), (1, 128, 7168), (1, 300, 1024),
                                       (3, 65, 640), (1, 4096, 512), (2, 256, 7168)])
def test_cast_per_token_bit_exact(oracle, batch, M, K):
    x = synth.normal_bf16(1000 + M + K, (batch, M, K))
    xd = bf16_dev(x)
    ld = (M + 3) // 4 * 4
    q = torch.empty((batch, M, K), dtype=torch.uint8, device="cuda")
    sfa = torch.full((batch, K // 128, ld), -7.0, dtype=torch.float32, device="cuda")
    _lib.dg_cast_fp8_per_token(xd, q, sfa, batch, M, K)
    torch.cuda.synchronize()
    qh, sh = host(q), host(sfa)
    for b in range(batch):
        qo, so = oracle.cast_per_token(x[b])
        assert np.array_equal(qh[b], qo)
        assert np.array_equal(sh[b][:, :M].view(np.uint32), so[:, :M].view(np.uint32))
        assert np.all(sh[b][:, M:] == -7.0), "padding entries must not be written"


def test_cast_per_token_special_values(oracle):
    M, K = 8, 256
    x = synth.normal_bf16(5, (M, K))
    x[0, :128] = 0                                         # amax 0 -> s = 1
    x[0, 7] = 0x8000                                       # -0
    vals = np.array([448.0, 2.0 ** -9, 3 * 2.0 ** -10, 2.0 ** -10, -7 * 2.0 ** -9, 1e-30], np.float32)
    x[1, :6] = synth.f32_to_bf16_bits(vals)                # subnormal outputs
    x[1, 6:128] = 0
    x[2, :] = synth.f32_to_bf16_bits(np.full(K, 3.0e38, np.float32))   # huge, all equal
    x[3, 128:] = synth.f32_to_bf16_bits(np.float32(2.0 ** -126) * np.arange(128, dtype=np.float32))
    q, sfa = ops.cast_per_token(bf16_dev(x))
    qo, so = oracle.cast_per_token(x)
    assert np.array_equal(host(q), qo)
    assert np.array_equal(host(sfa)[:, :M], so[:, :M])


@pytest.mark.parametrize("G,N,K", [(1, 1, 128), (1, 200, 256), (2, 128, 384), (1, 2112, 1024),
                                   (3, 136, 7168)])
def test_cast_per_block_bit_exact(oracle, G, N, K):
    w = synth.normal_bf16(2000 + N + K, (G, N, K))
    q, sfb = ops.cast_per_block(bf16_dev(w))
    torch.cuda.synchronize()
    qo, so = oracle.cast_per_block(w)
    assert np.array_equal(host(q), qo)
    assert np.array_equal(host(sfb).view(np.uint32), so.view(np.uint32))


@pytest.mark.parametrize("B,MN,Kb", [(1, 1, 1), (1, 37, 5), (2, 130, 56), (1, 4096, 56), (3, 33, 33)])
def test_transform_sf_exact(oracle, B, MN, Kb):
    rng = np.random.default_rng(B * 1000 + MN)
    s = rng.standard_normal((B, MN, Kb)).astype(np.float32)
    out = ops.transform_sf(dev(s))
    assert np.array_equal(host(out), oracle.transform_sf(s))


def test_cast_then_transform_roundtrip(oracle):
    """The per-token cast's MN-major scales equal the transform of its K-major scales."""
    x = synth.normal_bf16(77, (50, 512))
    _, sfa = ops.cast_per_token(bf16_dev(x))
    kmajor = sfa[:, :50].t().contiguous()
    assert torch.equal(ops.transform_sf(kmajor)[:, :50], sfa[:, :50])


def _all_finite_bf16(limit: float) -> np.ndarray:
    """Every finite bf16 bit pattern (both signs, both zeros) whose magnitude is <= limit."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    finite = (bits & 0x7F80) != 0x7F80
    mag = synth.bf16_bits_to_f32(bits & 0x7FFF)
    return bits[finite & (mag <= np.float32(limit))]


# amax values: ordinary ones, one whose scale is a subnormal fp32 (1/s still finite), one
# whose scale is so small that 1/s overflows, a huge one, and a bf16 subnormal amax.
SWEEP_AMAX = [1.0, 3.1875, 0.3, 57.75, 1.0e30, 448.0 * 2.0 ** -127, 2.0 ** -126, 2.0 ** -133]


@pytest.mark.parametrize("amax", SWEEP_AMAX)
def test_cast_per_token_every_bf16_value(oracle, amax):
    """Each row's K slice holds the amax first, then a run of the sweep of every finite bf16
    value up to that magnitude: every code decision of the cast for that scale is checked."""
    a_bits = np.uint16(synth.f32_to_bf16_bits(np.array([amax], np.float32))[0])
    amax_f = float(synth.bf16_bits_to_f32(np.array([a_bits], np.uint16))[0])
    vals = _all_finite_bf16(amax_f)
    rows = (vals.size + 126) // 127
    x = np.zeros((rows, 128), np.uint16)
    flat = np.zeros(rows * 127, np.uint16)
    flat[:vals.size] = vals
    x[:, 0] = a_bits
    x[:, 1:] = flat.reshape(rows, 127)
    q, sfa = ops.cast_per_token(bf16_dev(x))
    torch.cuda.synchronize()
    qo, so = oracle.cast_per_token(x)
    assert np.array_equal(host(q), qo)
    assert np.array_equal(host(sfa)[:, :rows].view(np.uint32), so[:, :rows].view(np.uint32))


@pytest.mark.parametrize("amax", [3.1875, 448.0 * 2.0 ** -127, 1.0e30])
def test_cast_per_block_every_bf16_value(oracle, amax):
    a_bits = np.uint16(synth.f32_to_bf16_bits(np.array([amax], np.float32))[0])
    amax_f = float(synth.bf16_bits_to_f32(np.array([a_bits], np.uint16))[0])
    vals = _all_finite_bf16(amax_f)
    per_block = 128 * 128 - 1
    nblk = (vals.size + per_block - 1) // per_block
    w = np.zeros((nblk * 128, 128), np.uint16)
    flat = np.zeros(nblk * per_block, np.uint16)
    flat[:vals.size] = vals
    for b in range(nblk):
        blk = np.concatenate([np.array([a_bits], np.uint16), flat[b * per_block:(b + 1) * per_block]])
        w[b * 128:(b + 1) * 128] = blk.reshape(128, 128)
    q, sfb = ops.cast_per_block(bf16_dev(w))
    torch.cuda.synchronize()
    qo, so = oracle.cast_per_block(w)
    assert np.array_equal(host(q), qo)
    assert np.array_equal(host(sfb).view(np.uint32), so.view(np.uint32))
