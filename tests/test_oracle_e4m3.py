"""Pins of the oracle's E4M3 codec (decode table and RNE/satfinite encoder).

Each pin is independent of the code it checks: closed-form special values of
the format, torch's own float8_e4m3fn conversion (a library routine), and a
brute-force nearest-value search written here.
"""
import math

import numpy as np
import pytest
import torch

from oracle import e4m3


def test_decode_special_values(O):
    d = O.e4m3_table()
    assert d[0x00] == 0.0 and not math.copysign(1, d[0x00]) < 0
    assert d[0x80] == 0.0 and math.copysign(1, d[0x80]) < 0      # -0
    assert d[0x7E] == 448.0 and d[0xFE] == -448.0                  # largest finite
    assert math.isnan(d[0x7F]) and math.isnan(d[0xFF])             # the only NaNs
    assert d[0x38] == 1.0                                          # exponent bias 7
    assert d[0x08] == 2.0 ** -6                                    # smallest normal
    assert d[0x01] == 2.0 ** -9                                    # smallest subnormal
    assert d[0x07] == 7 * 2.0 ** -9                                # largest subnormal
    assert d[0x3F] == 1.875 and d[0x40] == 2.0
    assert np.isfinite(d).sum() == 254


def test_decode_monotonic_and_symmetric(O):
    d = O.e4m3_table()
    assert np.all(np.diff(d[:127]) > 0)
    assert np.array_equal(d[128:255], -d[:127])


def test_decode_matches_torch_float8(O):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = O.e4m3_table()
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(ours))
    assert np.array_equal(ref[fin], ours[fin])
    assert np.array_equal(np.signbit(ref[fin]), np.signbit(ours[fin]))


def _brute_encode(v: np.ndarray) -> np.ndarray:
    """Nearest of all 127 non-negative finite values by explicit distance;
    ties to the even code; |v| >= 448 saturates."""
    pos = np.array([e4m3.DECODE[c] for c in range(127)])
    out = np.empty(v.shape, np.uint8)
    for i, x in enumerate(v.astype(np.float64)):
        a = min(abs(x), 448.0)
        dist = np.abs(pos - a)
        best = np.flatnonzero(dist == dist.min())
        code = best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]
        out[i] = code | (0x80 if math.copysign(1.0, x) < 0 else 0)
    return out


def test_encode_midpoints_and_neighbours(O):
    pos = O.e4m3_table()[:127]
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (pos[:-1] + pos[1:]) / 2)   # midpoints exact in fp32
    up = np.nextafter(mids, np.float32(np.inf))
    dn = np.nextafter(mids, np.float32(0))
    v = np.concatenate([mids, up, dn, pos.astype(np.float32)])
    v = np.concatenate([v, -v])
    assert np.array_equal(O.e4m3_encode(v), _brute_encode(v))
    # ties go to the even code: 1.0625 lies between 1.0 (0x38) and 1.125 (0x39)
    assert O.e4m3_encode(np.float32([1.0625]))[0] == 0x38
    assert O.e4m3_encode(np.float32([1.1875]))[0] == 0x3A       # between 0x39 and 0x3A -> even
    assert O.e4m3_encode(np.float32([2.0 ** -10]))[0] == 0x00   # half the smallest subnormal -> 0
    assert O.e4m3_encode(np.float32([3 * 2.0 ** -10]))[0] == 0x02


def test_encode_saturates(O):
    v = np.float32([448, 449, 463.9, 464, 480, 1e4, 3e38, np.inf, -448, -500, -np.inf])
    assert list(O.e4m3_encode(v)) == [0x7E] * 8 + [0xFE] * 3


def test_encode_sign_of_zero(O):
    v = np.float32([0.0, -0.0, -1e-30, 1e-30])
    assert list(O.e4m3_encode(v)) == [0x00, 0x80, 0x80, 0x00]


def test_encode_random_vs_brute_force(O):
    rng = np.random.default_rng(1)
    v = (rng.standard_normal(20000) * np.exp(rng.uniform(-12, 7, 20000))).astype(np.float32)
    assert np.array_equal(O.e4m3_encode(v), _brute_encode(v))


@pytest.mark.parametrize("start,stop,step", [(0, 0x43E00000, 997), (0x3C000000, 0x3C800000, 13)])
def test_encode_bit_pattern_sweep_vs_torch(O, start, stop, step):
    """Every step-th fp32 bit pattern in [0, 448] (and a dense sweep of one
    binade): torch's float8_e4m3fn cast is RNE there."""
    bits = np.arange(start, stop, step, dtype=np.uint32)
    v = bits.view(np.float32)
    v = np.concatenate([v, -v])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(v), ref)
