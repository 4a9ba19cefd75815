"""The seeded generator: published splitmix64 outputs, determinism, distributions and the
bf16 rounding (checked against torch's own fp32 -> bf16 conversion)."""
import numpy as np
import torch

from moe_grouped_gemm_sm_b200 import synth


def test_splitmix64_published_sequence():
    # splitmix64 started from state 0 (seed 0 here): the first outputs of the published generator
    got = synth.splitmix64(0, 0, 3).tolist()
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_streams_are_deterministic_and_offset():
    a = synth.splitmix64(5, 0, 100)
    b = synth.splitmix64(5, 40, 60)
    assert np.array_equal(a[40:], b)
    assert not np.array_equal(synth.splitmix64(6, 0, 100), a)


def test_normal_moments_and_chunking():
    z = synth.normal_f64(1, 200001)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    x1 = synth.normal_bf16(3, (1000, 64))
    x2 = synth.normal_bf16(3, (1000, 64))
    assert np.array_equal(x1, x2)
    # chunk boundaries do not change values
    old = synth._CHUNK
    try:
        synth._CHUNK = 1 << 10
        x3 = synth.normal_bf16(3, (1000, 64))
    finally:
        synth._CHUNK = old
    assert np.array_equal(x1, x3)


def test_bf16_rounding_matches_torch():
    f = (synth.normal_f64(9, 50000) * 3).astype(np.float32)
    ours = synth.f32_to_bf16_bits(f)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_workload_recipes():
    m, layout = synth.contiguous_layout(8)
    assert np.all((m >= 2048) & (m <= 6144))
    assert layout.shape[0] % 128 == 0
    off = 0
    for g in range(8):
        pad = (int(m[g]) + 127) // 128 * 128
        assert np.all(layout[off:off + int(m[g])] == g) and np.all(layout[off + int(m[g]):off + pad] == -1)
        off += pad
    mm, a, b = synth.masked_inputs(4, 256, 16, 128)
    assert a.shape == (4, 256, 128) and b.shape == (4, 16, 128)
    assert np.all((mm >= 64) & (mm <= 256))
    assert np.all(np.isfinite(synth.bf16_bits_to_f32(a)))
