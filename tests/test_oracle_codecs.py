"""Pins for the oracle's E2M1 / UE4M3 codecs (CPU only).

Each pin checks the oracle against something other than itself: the bit-level
format definitions, torch's own float8_e4m3fn conversion, and the rounding
midpoints of the E2M1 grid.
"""
import numpy as np
import pytest
import torch

from oracle import codecs


def _e2m1_from_bits(c: int) -> float:
    """Bit-level E2M1 definition: s | e1 e0 | m, bias 1, subnormal when e == 0."""
    s = -1.0 if (c >> 3) & 1 else 1.0
    e = (c >> 1) & 3
    m = c & 1
    if e == 0:
        return s * 0.5 * m                 # 2^(1-1) * (m/2)
    return s * 2.0 ** (e - 1) * (1.0 + m / 2.0)


def test_e2m1_decode_matches_bit_definition():
    for c in range(16):
        assert codecs.e2m1_decode(np.array([c]))[0] == _e2m1_from_bits(c)
        assert np.signbit(codecs.e2m1_decode(np.array([c]))[0]) == bool(c & 8)


def test_ue4m3_decode_matches_torch_float8():
    codes = torch.arange(0, 127, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = codecs.ue4m3_decode(codes.numpy())
    np.testing.assert_array_equal(got, ref)
    assert np.isnan(codecs.ue4m3_decode(np.array([0x7F]))[0])
    assert codecs.ue4m3_decode(np.array([0x7E]))[0] == 448.0
    assert codecs.ue4m3_decode(np.array([1]))[0] == 2.0 ** -9


@pytest.mark.parametrize("x,code", [
    (0.0, 0x0), (0.24, 0x0), (0.25, 0x0), (0.26, 0x1), (0.5, 0x1),
    (0.75, 0x2), (1.0, 0x2), (1.25, 0x2), (1.26, 0x3), (1.5, 0x3),
    (1.75, 0x4), (2.0, 0x4), (2.5, 0x4), (2.51, 0x5), (3.0, 0x5),
    (3.5, 0x6), (4.0, 0x6), (5.0, 0x6), (5.01, 0x7), (6.0, 0x7), (7.0, 0x7), (1e30, 0x7),
    (-0.0, 0x8), (-0.1, 0x8), (-0.75, 0xA), (-2.5, 0xC), (-3.5, 0xE), (-5.0, 0xE), (-9.0, 0xF),
])
def test_e2m1_encode_midpoints(x, code):
    assert int(codecs.e2m1_encode(np.float32(x))) == code


def test_e2m1_encode_decode_identity():
    for c in range(16):
        v = codecs.e2m1_decode(np.array([c]))[0]
        assert int(codecs.e2m1_encode(np.float32(v))) == c


def test_ue4m3_encode_decode_identity():
    codes = np.arange(127)
    vals = codecs.ue4m3_decode(codes).astype(np.float32)
    np.testing.assert_array_equal(codecs.ue4m3_encode(vals), codes)


def test_ue4m3_encode_matches_torch_rne_in_range():
    # torch's fp32 -> float8_e4m3fn conversion is round-to-nearest-even; in range it must agree.
    g = torch.Generator().manual_seed(7)
    x = torch.cat([
        torch.rand(200000, generator=g) * 448.0,
        torch.rand(100000, generator=g) * 2.0 ** -6,               # subnormal range
        torch.exp2(torch.rand(100000, generator=g) * 14 - 9),      # log-uniform
        torch.tensor(codecs.UE4M3_GRID[:-1] + np.diff(codecs.UE4M3_GRID) / 2, dtype=torch.float32),  # ties
    ]).to(torch.float32).clamp(max=448.0)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = codecs.ue4m3_encode(x.numpy())
    np.testing.assert_array_equal(got, ref)


def test_ue4m3_encode_saturates():
    assert int(codecs.ue4m3_encode(np.float32(464.0))) == 0x7E
    assert int(codecs.ue4m3_encode(np.float32(1e30))) == 0x7E
    # 2^-10 is exactly half of the smallest subnormal: tie -> even code 0.
    assert int(codecs.ue4m3_encode(np.float32(2.0 ** -10))) == 0
    assert int(codecs.ue4m3_encode(np.float32(3 * 2.0 ** -10))) == 2   # tie 1|2 -> even 2


def test_e2m1_encode_matches_nearest_value_bruteforce():
    # independent brute force: scan the 16 decoded codes, nearest magnitude, even mantissa on ties
    rng = np.random.default_rng(3)
    xs = np.concatenate([rng.uniform(-8, 8, 20000), np.arange(-7, 7.01, 0.125)]).astype(np.float32)
    got = codecs.e2m1_encode(xs)
    for x, c in zip(xs, got):
        best, bd = None, None
        for cand in range(8):
            d = abs(abs(float(x)) - _e2m1_from_bits(cand))
            if bd is None or d < bd or (d == bd and cand % 2 == 0):
                best, bd = cand, d
        best |= 8 if np.signbit(x) else 0
        assert c == best, (x, c, best)
