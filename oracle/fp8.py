"""Per-tensor FP8: E4M3 (or E5M2) elements with one fp32 scale for the whole tensor.

Test infrastructure only (see the package docstring).

What the pages fix (ai4snews paragraph 2; sitech.ge "Memory and quantization
overhead"): the recipe trains in FP8 as well as MXFP8, both with 8-bit values;
MXFP8 is the one that adds a scaling factor per block of 32 values.  Plain FP8
therefore carries no block scales: one scaling factor serves a whole tensor.
Everything else is a reading:

* the tensor: each GEMM operand of each expert (an expert's weight matrix, its
  rows of x / a / dy / dh).  The grouped GEMM is a group of per-expert GEMMs,
  and every one of them gets its own operand scales.  With one scale per
  tensor the codes do not depend on the GEMM's K axis, so one quantisation of
  a tensor serves both GEMMs that read it (the transposed copy holds the same
  codes).
* current scaling: the scale comes from the tensor's own maximum magnitude at
  the time it is quantised, s = fp32(vmax / amax) (vmax = 448 for E4M3, 57344
  for E5M2; a correctly rounded fp32 division).  amax = 0 gives s = 1; a
  quotient beyond the fp32 range gives the largest finite fp32.
* element: code = RNE-saturating encode (oracle.mx) of the fp32 product
  fp32(v * s); its value is code / s.
"""
from __future__ import annotations

import numpy as np

from . import mx

VMAX = {"e4m3": mx.E4M3_MAX, "e5m2": mx.E5M2_MAX}
F32_MAX = np.float32(np.finfo(np.float32).max)


def scale(amax, fmt: str = "e4m3") -> np.ndarray:
    """fp32 scale(s) for tensor maxima ``amax`` (array or scalar, fp32 values)."""
    a = np.asarray(amax, dtype=np.float32)
    with np.errstate(divide="ignore", over="ignore"):
        s = np.float32(VMAX[fmt]) / np.where(a > 0, a, np.float32(1))
    s = np.where(np.isinf(s), F32_MAX, s)
    return np.where(a > 0, s, np.float32(1)).astype(np.float32)


def amax(v) -> np.float32:
    """Largest magnitude of the tensor (its values must be fp32-representable)."""
    v = np.asarray(v, dtype=np.float32)
    return np.float32(np.max(np.abs(v))) if v.size else np.float32(0)


def encode(v, s, fmt: str = "e4m3") -> np.ndarray:
    """Codes of the values v (fp32-representable) under the tensor scale s (fp32)."""
    v = np.asarray(v, dtype=np.float32)
    prod = (v * np.float32(s)).astype(np.float32)          # fp32 product, rounded to nearest
    enc = mx.e4m3_encode if fmt == "e4m3" else mx.e5m2_encode
    return enc(prod.astype(np.float64))


def quantize(v, fmt: str = "e4m3"):
    """Codes (uint8, the shape of v) and the fp32 scale of the tensor v."""
    s = scale(amax(v), fmt)
    return encode(v, s, fmt), np.float32(s)


def dequantize(codes, s, fmt: str = "e4m3") -> np.ndarray:
    dec = mx.e4m3_decode if fmt == "e4m3" else mx.e5m2_decode
    return dec(codes) / np.float64(s)


def fake_quant(v, fmt: str = "e4m3") -> np.ndarray:
    """Value of the tensor v after per-tensor FP8 quantisation (float64)."""
    c, s = quantize(v, fmt)
    return dequantize(c, s, fmt)
