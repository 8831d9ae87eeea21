"""MXFP8 codec: E4M3 elements with one E8M0 power-of-two scale per 32 values.

Test infrastructure only (see the package docstring).

What the pages fix (sitech.ge "Memory and quantization overhead"; ai4snews
paragraph 2; andresseo.expert "Memory Pressure From Long Sequences"): 8-bit
elements, one scaling factor per block of 32 consecutive values, chosen to
protect the numerical range.  Everything else is a reading:

* element format: OCP E4M3 ("FN"): bias 7, no infinities, S.1111.111 is NaN,
  largest finite 448, subnormals down to 2**-9.  Conversion rounds to nearest,
  ties to even, saturating to +-448, and keeps the sign of zero.
* shared scale: the power of two 2**e with the smallest integer e such that
  amax <= 448 * 2**e (no element can saturate), clamped to [-127, 127] and
  stored as the biased byte e + 127.  An all-zero block gets byte 0.
  Variant ("floor", the OCP MX v1.0 rule): e = floor(log2(amax)) - 8, 8 being
  the exponent of E4M3's largest power of two; the block maximum then scales
  into [256, 512) and elements above 448 saturate to 448.
* a block holding a NaN gets scale byte 0xFF and NaN codes (outside the
  tested contract; inputs are finite).

Gradient variant (E5M2 elements, the same E8M0 scales per 32 values): OCP E5M2
has bias 15, largest finite 57344 = 1.75 * 2**15, subnormals down to 2**-16,
infinities and NaNs; conversion rounds to nearest even and saturates to
+-57344.  Its round-up shared exponent is the smallest e with
amax <= 57344 * 2**e, its floor one floor(log2(amax)) - 15.

The implementation is brute force on purpose: decode all 256 codes from the
bit layout, and encode by picking the nearest table entry.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
BLOCK = 32


def e4m3_decode_table() -> np.ndarray:
    """float64 value of each of the 256 E4M3 codes (NaN for the two NaN codes)."""
    vals = np.empty(256, dtype=np.float64)
    for c in range(256):
        s = -1.0 if (c >> 7) & 1 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            vals[c] = np.nan
        elif e == 0:
            vals[c] = s * (m / 8.0) * 2.0 ** (1 - 7)
        else:
            vals[c] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


def e5m2_decode_table() -> np.ndarray:
    """float64 value of each of the 256 E5M2 codes (+-inf for 0x7C / 0xFC, NaN above)."""
    vals = np.empty(256, dtype=np.float64)
    for c in range(256):
        s = -1.0 if (c >> 7) & 1 else 1.0
        e = (c >> 2) & 0x1F
        m = c & 0x3
        if e == 0x1F:
            vals[c] = s * np.inf if m == 0 else np.nan
        elif e == 0:
            vals[c] = s * (m / 4.0) * 2.0 ** (1 - 15)
        else:
            vals[c] = s * (1.0 + m / 4.0) * 2.0 ** (e - 15)
    return vals


_TABLE = e4m3_decode_table()
# positive finite codes 0x00..0x7E are monotone in value
_POS = _TABLE[:0x7F].copy()
_TABLE5 = e5m2_decode_table()
_POS5 = _TABLE5[:0x7C].copy()          # positive finite E5M2 codes 0x00..0x7B
E5M2_MAX = 57344.0
FORMATS = ("e4m3", "e5m2")


def e4m3_encode(v) -> np.ndarray:
    """Round float values to E4M3 codes: nearest, ties to even code, saturate at 448."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    nan = np.isnan(v)
    a_c = np.where(nan, 0.0, np.minimum(a, E4M3_MAX))
    lo = np.searchsorted(_POS, a_c, side="right") - 1          # largest code with value <= a
    lo = np.clip(lo, 0, 0x7E)
    hi = np.minimum(lo + 1, 0x7E)
    d_lo = a_c - _POS[lo]
    d_hi = _POS[hi] - a_c
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi != lo) & (lo % 2 == 1))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(np.signbit(v), code | 0x80, code).astype(np.uint8)
    code = np.where(nan, np.where(np.signbit(v), 0xFF, 0x7F), code).astype(np.uint8)
    return code


def e4m3_decode(codes) -> np.ndarray:
    return _TABLE[np.asarray(codes, dtype=np.uint8)]


def e5m2_encode(v) -> np.ndarray:
    """Round float values to E5M2 codes: nearest, ties to even code, saturate at 57344."""
    v = np.asarray(v, dtype=np.float64)
    nan = np.isnan(v)
    a_c = np.where(nan, 0.0, np.minimum(np.abs(v), E5M2_MAX))
    lo = np.clip(np.searchsorted(_POS5, a_c, side="right") - 1, 0, 0x7B)
    hi = np.minimum(lo + 1, 0x7B)
    d_lo = a_c - _POS5[lo]
    d_hi = _POS5[hi] - a_c
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi != lo) & (lo % 2 == 1))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(np.signbit(v), code | 0x80, code).astype(np.uint8)
    return np.where(nan, np.where(np.signbit(v), 0xFF, 0x7F), code).astype(np.uint8)


def e5m2_decode(codes) -> np.ndarray:
    return _TABLE5[np.asarray(codes, dtype=np.uint8)]


SCALE_RULES = ("ceil", "floor")


def e8m0_exponent(amax, rule: str = "ceil", fmt: str = "e4m3") -> np.ndarray:
    """Shared exponent of a block with maximum magnitude ``amax`` (int64, clamped to [-127, 127]).

    ceil:  the smallest integer e with amax <= vmax * 2**e (vmax = 448 for E4M3, 57344 for E5M2).
    floor: floor(log2(amax)) - emax (emax = 8 for E4M3, 15 for E5M2; OCP MX v1.0).
    """
    if rule not in SCALE_RULES or fmt not in FORMATS:
        raise ValueError((rule, fmt))
    vmax, emax = (E4M3_MAX, 8) if fmt == "e4m3" else (E5M2_MAX, 15)
    amax = np.asarray(amax, dtype=np.float64)
    safe = np.where((amax > 0) & np.isfinite(amax), amax, 1.0)
    _, ex = np.frexp(safe)                  # safe = m * 2**ex, m in [0.5, 1)
    guess = ex.astype(np.int64) - 1 - emax  # floor(log2(amax)) - emax
    if rule == "floor":
        e = guess
    else:
        e = guess + 2
        # walk down while the next smaller exponent still covers amax (checks are exact in fp64)
        for _ in range(4):
            smaller_ok = safe <= vmax * np.exp2((e - 1).astype(np.float64))
            e = np.where(smaller_ok, e - 1, e)
    e = np.where(amax > 0, e, -127)
    return np.clip(e, -127, 127)


def quantize_blocks(x: np.ndarray, rule: str = "ceil", fmt: str = "e4m3"):
    """Quantise along the last axis in blocks of 32, with the shared-exponent ``rule`` and the
    element format ``fmt``.

    Returns (codes uint8, same shape as x; scale bytes uint8, shape [..., n/32]).
    """
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    if n % BLOCK:
        raise ValueError("last axis must be a multiple of 32")
    xb = x.reshape(x.shape[:-1] + (n // BLOCK, BLOCK))
    amax = np.max(np.abs(xb), axis=-1)
    has_nan = np.isnan(xb).any(axis=-1)
    e = e8m0_exponent(np.where(has_nan, 0.0, amax), rule, fmt)
    scaled = xb * np.exp2(-e.astype(np.float64))[..., None]
    codes = e4m3_encode(scaled) if fmt == "e4m3" else e5m2_encode(scaled)
    codes = np.where(has_nan[..., None], np.where(np.signbit(xb), 0xFF, 0x7F), codes).astype(np.uint8)
    sbytes = np.where(has_nan, 0xFF, e + 127).astype(np.uint8)
    return codes.reshape(x.shape), sbytes


def dequantize_blocks(codes: np.ndarray, sbytes: np.ndarray, fmt: str = "e4m3") -> np.ndarray:
    """Inverse of quantize_blocks (exact, float64)."""
    codes = np.asarray(codes, dtype=np.uint8)
    n = codes.shape[-1]
    dec = e4m3_decode(codes) if fmt == "e4m3" else e5m2_decode(codes)
    vals = dec.reshape(codes.shape[:-1] + (n // BLOCK, BLOCK))
    s = np.asarray(sbytes).astype(np.float64)
    scale = np.where(s == 255, np.nan, np.exp2(s - 127.0))
    return (vals * scale[..., None]).reshape(codes.shape)


def quantize_rowwise(x: np.ndarray, rule: str = "ceil", fmt: str = "e4m3"):
    """Blocks of 32 along each row (the last axis): codes [R, C], scales [R, C/32]."""
    return quantize_blocks(x, rule, fmt)


def quantize_colwise_t(x: np.ndarray, rule: str = "ceil", fmt: str = "e4m3"):
    """Blocks of 32 down each column, returned transposed: codes [C, R], scales [C, R/32]."""
    return quantize_blocks(np.swapaxes(np.asarray(x), -1, -2), rule, fmt)


def fake_quant(x: np.ndarray, axis: int, rule: str = "ceil", fmt: str = "e4m3") -> np.ndarray:
    """Dequantised value of x after MXFP8 quantisation with blocks of 32 along ``axis``."""
    xm = np.moveaxis(np.asarray(x, dtype=np.float64), axis, -1)
    c, s = quantize_blocks(xm, rule, fmt)
    return np.moveaxis(dequantize_blocks(c, s, fmt), -1, axis)
