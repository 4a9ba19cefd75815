"""Pins of the oracle's E4M3 codec against the OCP OFP8 E4M3 definition and torch's own
float8_e4m3fn conversion (an independent library routine)."""
import math
import random

import numpy as np
import pytest
import torch


def torch_decode_all():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_decode_matches_torch_for_every_code(oracle):
    ours = oracle.e4m3_table()
    ref = torch_decode_all()
    nan_ours = np.isnan(ours)
    assert np.array_equal(nan_ours, np.isnan(ref))
    assert sorted(np.nonzero(nan_ours)[0].tolist()) == [0x7F, 0xFF]
    assert np.array_equal(ours[~nan_ours], ref[~nan_ours])


def test_decode_structure(oracle):
    t = oracle.e4m3_table()
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0), "positive codes must be strictly increasing"
    assert t[0x7E] == 448.0
    assert t[0x01] == 2.0 ** -9
    assert t[0x08] == 2.0 ** -6
    assert t[0x38] == 1.0
    for c in range(0x7F):
        assert t[c | 0x80] == -t[c] or (t[c] == 0 and math.copysign(1, t[c | 0x80]) < 0)


def test_roundtrip_every_finite_code(oracle):
    t = oracle.e4m3_table()
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert oracle.e4m3_encode(t[c]) == c, hex(c)


def test_midpoints_round_to_even(oracle):
    t = oracle.e4m3_table()
    for c in range(0x7E):
        mid = (t[c] + t[c + 1]) / 2.0           # exact in fp32: at most 5 significant bits
        assert float(np.float32(mid)) == mid
        even = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode(mid) == even, (hex(c), mid)
        assert oracle.e4m3_encode(-mid) == even | 0x80
        # just off the midpoint goes to the nearer neighbour
        lo = float(np.nextafter(np.float32(mid), np.float32(0)))
        hi = float(np.nextafter(np.float32(mid), np.float32(1e9)))
        assert oracle.e4m3_encode(lo) == c
        assert oracle.e4m3_encode(hi) == c + 1


def test_saturation(oracle):
    for y in (448.0, 448.5, 463.9, 464.0, 480.0, 1e6, 3.0e38):
        assert oracle.e4m3_encode(y) == 0x7E
        assert oracle.e4m3_encode(-y) == 0xFE
    assert oracle.e4m3_encode(0.0) == 0x00
    assert oracle.e4m3_encode(-0.0) == 0x80


def brute_nearest(t, y):
    """Nearest finite code by exhaustive scan; ties to the even code; saturate at 448."""
    a = abs(y)
    if a >= 448.0:
        code = 0x7E
    else:
        best = None
        for c in range(0x7F):
            d = abs(t[c] - a)
            if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
                best = (d, c)
        code = best[1]
    return code | (0x80 if math.copysign(1.0, y) < 0 else 0)


def test_encode_matches_brute_force_and_torch(oracle):
    t = oracle.e4m3_table()
    rng = random.Random(7)
    ys = []
    for _ in range(3000):
        e = rng.uniform(-12, 9.2)
        ys.append(float(np.float32(rng.choice((-1, 1)) * 2.0 ** e)))
    ys += [float(np.float32(x)) for x in (1e-30, -1e-30, 2.0 ** -10, 2.0 ** -10 * 1.0000001, 3 * 2.0 ** -11)]
    ours = np.array([oracle.e4m3_encode(y) for y in ys], np.uint8)
    brute = np.array([brute_nearest(t, y) for y in ys], np.uint8)
    assert np.array_equal(ours, brute)
    # torch's conversion rounds to nearest even but overflows to NaN above the range:
    # compare where |y| < 464 (values in [448, 464) round to 448 in both).
    ysf = torch.tensor(ys, dtype=torch.float32)
    mask = ysf.abs() < 464
    tq = ysf[mask].to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours[mask.numpy()], tq)


def test_bf16_decode(oracle):
    for bits in (0x0000, 0x8000, 0x3F80, 0xBF80, 0x4000, 0x0001, 0x7F7F, 0x3DCD):
        t = torch.from_numpy(np.array([bits], np.uint16).view(np.int16)).view(torch.bfloat16)
        ref = t.float().item()
        got = oracle.lib().dgo_bf16_to_f32(bits)
        assert got == ref and math.copysign(1, got) == math.copysign(1, ref)
