"""Pins of the oracle's casts (per-token 1x128, per-block 128x128) and of the scale-layout
transform. Block-wise scaling: aitangshan.cn/news/1491278, 技术原理 §4; the scale layout:
likun.im/craft/deepgemm §五. None of these re-types the oracle's formula; each checks a
property that any correct cast must have, or a library route (torch's float8_e4m3fn)."""
import numpy as np
import pytest
import torch

from moe_grouped_gemm_sm_b200 import synth


def bf16_to_f32(x):
    return synth.bf16_bits_to_f32(x)


def test_amax_element_maps_to_448(oracle):
    x = synth.normal_bf16(11, (37, 512))
    q, sfa = oracle.cast_per_token(x)
    xf = bf16_to_f32(x).reshape(37, 4, 128)
    idx = np.abs(xf).argmax(axis=2)
    qr = q.reshape(37, 4, 128)
    for m in range(37):
        for kb in range(4):
            code = qr[m, kb, idx[m, kb]]
            assert code & 0x7F == 0x7E, (m, kb, hex(code))


def test_scale_and_layout(oracle):
    M, K = 13, 384
    x = synth.normal_bf16(12, (M, K))
    q, sfa = oracle.cast_per_token(x)
    assert sfa.shape == (3, 16)                 # [Kb][pad4(M)]
    xf = bf16_to_f32(x).reshape(M, 3, 128)
    amax = np.abs(xf).max(axis=2)
    # the scale times 448 recovers amax to fp32 rounding, and the layout is MN-major
    assert np.allclose(sfa[:, :M].T * 448.0, amax, rtol=2 ** -22, atol=0)
    assert np.all(sfa[:, M:] == 0)


def test_dequant_error_bound(oracle):
    """|e4m3(q)·s - x| is at most half a grid step at x/s, times s (nearest rounding)."""
    M, K = 64, 1024
    x = synth.normal_bf16(13, (M, K))
    q, sfa = oracle.cast_per_token(x)
    t = oracle.e4m3_table()
    xf = bf16_to_f32(x).astype(np.float64).reshape(M, K // 128, 128)
    s = sfa[:, :M].T.astype(np.float64)[:, :, None]
    y = np.abs(xf / s)
    # grid step: 2^-9 below 2^-6, else 2^(floor(log2 y) - 3)
    e = np.floor(np.log2(np.maximum(y, 2.0 ** -6)))
    step = np.where(y < 2.0 ** -6, 2.0 ** -9, 2.0 ** (e - 3))
    deq = t[q.reshape(M, K // 128, 128)] * s
    err = np.abs(deq - xf)
    assert np.all(err <= 0.5 * step * s * (1 + 1e-6) + 1e-30)


def test_matches_torch_float8_route(oracle):
    """y = x / s in IEEE fp32, then torch's round-to-nearest-even float8_e4m3fn conversion."""
    M, K = 50, 768
    x = synth.normal_bf16(14, (M, K))
    q, sfa = oracle.cast_per_token(x)
    xt = torch.from_numpy(bf16_to_f32(x).copy()).reshape(M, K // 128, 128)
    amax = xt.abs().amax(dim=2, keepdim=True)
    s = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
    y = xt / s
    assert torch.all(y.abs() < 464)
    tq = y.to(torch.float8_e4m3fn).view(torch.uint8).reshape(M, K).numpy()
    assert np.array_equal(q, tq)
    assert np.array_equal(sfa[:, :M].T, s.reshape(M, K // 128).numpy())


def test_power_of_two_invariance(oracle):
    """Scaling x by 2^j leaves every code unchanged and scales every scale by exactly 2^j."""
    x = synth.normal_bf16(15, (9, 256))
    q0, s0 = oracle.cast_per_token(x)
    for j in (-5, 3):
        xj = synth.f32_to_bf16_bits(bf16_to_f32(x) * np.float32(2.0 ** j))
        assert np.array_equal(bf16_to_f32(xj), bf16_to_f32(x) * np.float32(2.0 ** j))
        qj, sj = oracle.cast_per_token(xj)
        assert np.array_equal(q0, qj)
        assert np.array_equal(sj[:, :9], s0[:, :9] * np.float32(2.0 ** j))


def test_zero_slice_and_signed_zero(oracle):
    x = synth.normal_bf16(16, (2, 256))
    x[0, :128] = 0
    x[0, 5] = 0x8000                            # -0.0
    q, sfa = oracle.cast_per_token(x)
    assert sfa[0, 0] == 1.0
    assert np.all(q[0, :128][np.arange(128) != 5] == 0x00)
    assert q[0, 5] == 0x80
    assert sfa[1, 0] != 1.0


def test_subnormal_outputs(oracle):
    """A slice with one large value pushes the small ones onto the E4M3 subnormal grid."""
    x = np.zeros((1, 128), np.uint16)
    vals = np.array([448.0, 2.0 ** -9, 3 * 2.0 ** -10, 2.0 ** -10, 5 * 2.0 ** -11, -7 * 2.0 ** -9], np.float32)
    x[0, :6] = synth.f32_to_bf16_bits(vals)
    q, sfa = oracle.cast_per_token(x)
    assert sfa[0, 0] == 1.0                     # amax 448 -> s = 1 exactly
    # 2^-9 -> 0x01; 1.5·2^-9 ties between 1 and 2 -> even (2); 0.5·2^-9 ties between 0 and 1 -> 0;
    # 1.25·2^-9 -> 1; -7·2^-9 -> 0x87
    assert q[0, :6].tolist() == [0x7E, 0x01, 0x02, 0x00, 0x01, 0x87]


def test_per_block_partial_and_identity(oracle):
    N, K = 200, 256                             # second 128-row block holds 72 valid rows
    x = synth.normal_bf16(17, (N, K))
    q, sfb = oracle.cast_per_block(x)
    assert sfb.shape == (2, 2)
    xf = bf16_to_f32(x)
    for nb in range(2):
        rows = slice(nb * 128, min(N, nb * 128 + 128))
        for kb in range(2):
            amax = np.abs(xf[rows, kb * 128:(kb + 1) * 128]).max()
            assert sfb[nb, kb] == np.float32(amax) / np.float32(448.0)
    # a single-row matrix: per-block and per-token casts coincide
    q1, s1 = oracle.cast_per_block(x[:1])
    q2, s2 = oracle.cast_per_token(x[:1])
    assert np.array_equal(q1, q2) and np.array_equal(s1[0], s2[:, 0])
    # batch dimension: each batch entry is cast on its own
    xb = np.stack([x, x[::-1].copy()])
    qb, sb = oracle.cast_per_block(xb)
    assert np.array_equal(qb[0], q) and np.array_equal(sb[0], sfb)
    qr, sr = oracle.cast_per_block(x[::-1].copy())
    assert np.array_equal(qb[1], qr) and np.array_equal(sb[1], sr)


def test_transform_sf_matches_numpy_transpose(oracle):
    rng = np.random.default_rng(3)
    for B, MN, Kb in ((1, 7, 3), (3, 130, 5), (2, 4, 1)):
        s = rng.standard_normal((B, MN, Kb)).astype(np.float32)
        out = oracle.transform_sf(s)
        ld = (MN + 3) // 4 * 4
        assert out.shape == (B, Kb, ld)
        assert np.array_equal(out[:, :, :MN], np.transpose(s, (0, 2, 1)))
        assert np.all(out[:, :, MN:] == 0)
    # the per-token cast's sfa equals transform_sf of the same scales laid out K-major
    x = synth.normal_bf16(18, (6, 384))
    _, sfa = oracle.cast_per_token(x)
    assert np.array_equal(oracle.transform_sf(np.ascontiguousarray(sfa[:, :6].T)), sfa)


def test_scatter_cast_is_the_per_token_cast_moved_to_its_rows(oracle):
    """The cast into the contiguous layout (tokens routed to the rows of their expert's block)
    is the per-token cast of each token, placed at its destination row; rows no token maps to
    keep what they held, and a dropped token (-1) writes nothing."""
    T, K, M_sum = 40, 384, 128
    x = synth.normal_bf16(51, (T, K))
    rng = np.random.default_rng(3)
    dst = rng.permutation(M_sum)[:T].astype(np.int32)
    dst[5] = -1
    q0 = np.full((M_sum, K), 0xAB, np.uint8)
    s0 = np.full((K // 128, M_sum), -1.0, np.float32)
    q, sfa = oracle.cast_per_token_scatter(x, dst, M_sum, q0, s0)
    qt, st = oracle.cast_per_token(x)
    for t in range(T):
        if dst[t] >= 0:
            assert np.array_equal(q[dst[t]], qt[t])
            assert np.array_equal(sfa[:, dst[t]], st[:, t])
    untouched = np.setdiff1d(np.arange(M_sum), dst[dst >= 0])
    assert np.all(q[untouched] == 0xAB) and np.all(sfa[:, untouched] == -1.0)


def test_scatter_cast_rejects_a_row_taken_twice(oracle):
    x = synth.normal_bf16(52, (3, 128))
    with pytest.raises(ValueError):
        oracle.cast_per_token_scatter(x, np.array([1, 4, 1], np.int32), 8)
