"""E4M3 ("FN" flavour of the OCP 8-bit floating point formats) for the oracle.

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline may import this package. It shares no code with the CUDA path.

transformers PR #47844 ("What does this PR do?") states that FP8 checkpoints
use E4M3 weights with 128 x 128 weight blocks and dynamically quantised
activations. The format itself is not spelled out on the pages; this module
takes the OCP E4M3FN reading: 1 sign bit, 4 exponent bits (bias 7), 3
mantissa bits, no infinities, NaN = S.1111.111, largest finite 448.

decode: the 256-entry table, written from the closed form of the format.
encode: nearest finite table value, ties to the even code, saturating to
+-448 (round-to-nearest-even with satfinite). The sign of zero is kept.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def _decode_one(code: int) -> float:
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


DECODE = np.array([_decode_one(c) for c in range(256)], dtype=np.float64)
DECODE.setflags(write=False)

# non-negative finite values, indexed by code 0..126 (monotonic in the code)
_POS = DECODE[:127].copy()


def decode(codes: np.ndarray) -> np.ndarray:
    """E4M3 codes (uint8) -> float64 values through the 256-entry table."""
    return DECODE[np.asarray(codes, dtype=np.uint8)]


def encode(v: np.ndarray) -> np.ndarray:
    """float32 values -> E4M3 codes: nearest representable value, ties to the
    even code, |v| >= 448 saturates to +-448. NaN inputs are not expected."""
    v = np.asarray(v, dtype=np.float32)
    a = np.abs(v).astype(np.float64)
    sat = a >= E4M3_MAX
    a_c = np.minimum(a, E4M3_MAX)
    hi = np.searchsorted(_POS, a_c, side="left")        # first table value >= a
    hi = np.minimum(hi, 126)
    lo = np.maximum(hi - 1, 0)
    exact = _POS[hi] == a_c
    d_lo = a_c - _POS[lo]
    d_hi = _POS[hi] - a_c
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(exact, hi, np.where(pick_hi, hi, lo))
    code = np.where(sat, 126, code).astype(np.uint8)
    sign = np.signbit(v).astype(np.uint8) << 7
    return code | sign
