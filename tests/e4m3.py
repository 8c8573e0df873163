"""Host-side FP8 e4m3 (the "fn" variant: no infinities, 0x7F / 0xFF = NaN,
largest finite 448) for the decode tests: exact decoding of codes, and
quantisation by round-to-nearest-even with saturation to +-448.  Written from
the format's definition (1 sign bit, 4 exponent bits with bias 7, 3 mantissa
bits, subnormals at exponent field 0); independent of the CUDA path."""
import numpy as np


def decode(codes) -> np.ndarray:
    """e4m3 codes (uint8) -> float64 values (NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes, np.uint8).astype(np.int64)
    s = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 15
    m = c & 7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    out = s * mag
    return np.where((e == 15) & (m == 7), np.nan, out)


_POS = decode(np.arange(127, dtype=np.uint8))  # codes 0..126, increasing, 0 .. 448


def quantize(y) -> np.ndarray:
    """float32 values -> e4m3 codes: nearest value, ties to the even code,
    magnitudes above 448 saturate to 448, NaN -> 0x7F; the sign is kept
    (a negative value that rounds to zero gives 0x80)."""
    y = np.asarray(y, np.float32)
    a = np.abs(y).astype(np.float64)
    a = np.minimum(a, 448.0)
    hi = np.searchsorted(_POS, a, side="left").clip(0, 126)
    lo = (hi - 1).clip(0, 126)
    d_hi = np.abs(_POS[hi] - a)
    d_lo = np.abs(a - _POS[lo])
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0))
    code = np.where(pick_lo, lo, hi).astype(np.uint8)
    code = np.where(np.signbit(y), code | np.uint8(0x80), code).astype(np.uint8)
    return np.where(np.isnan(y), np.uint8(0x7F), code).astype(np.uint8)
