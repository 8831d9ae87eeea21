"""Pins of the per-tensor FP8 oracle (oracle.fp8) against facts fixed by the formats and by
arithmetic (CPU only).

Per-tensor FP8 (ai4snews paragraph 2: FP8 and MXFP8 training; sitech.ge "Memory and quantization
overhead": 8-bit values, MXFP8 adding a scale per block of 32) keeps one fp32 scale per tensor.
The readings (current scaling, s = fp32(vmax / amax), code = RNE-saturating encode of fp32(v * s))
are pinned here by:
* hand vectors (tests/golden/fp8_per_tensor_hand_vectors.txt);
* the scale against exact rational division, rounded to fp32 by brute force;
* every code against a brute-force nearest search over the 256 decoded values;
* the tensor maximum landing on the largest code, invariance under power-of-two rescaling, and
  the half-step error bound of the element format;
* the layer: on operands whose values lie on the scaled E4M3 grid (each tensor's maximum
  448 * 2**k) the first GEMM of the "fp8" forward is exact.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import fp8, moe, mx

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fp8_per_tensor_hand_vectors.txt")
VMAX = {"e4m3": 448.0, "e5m2": 57344.0}
TOP = {"e4m3": 0x7E, "e5m2": 0x7B}


def _cases():
    out = []
    with open(GOLDEN) as fh:
        for line in fh:
            if not line.strip() or line.startswith("#"):
                continue
            name, fmt, vals, sc, codes = [c.strip() for c in line.split("|")]
            out.append((name, fmt, [float(v) for v in vals.split(",")], float(sc),
                        [int(c, 16) for c in codes.split(",")]))
    return out


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c[0])
def test_hand_vectors(case):
    _, fmt, vals, sc, codes = case
    v = np.array(vals, dtype=np.float32)
    assert np.array_equal(v.astype(np.float64), np.array(vals)), "a golden value is not an fp32 value"
    got_codes, got_s = fp8.quantize(v, fmt)
    assert float(got_s) == sc
    assert got_codes.tolist() == codes


def _nearest_f32(q: Fraction) -> np.float32:
    """The fp32 nearest to the rational q (ties to the even significand), by brute force over the
    neighbours of a first guess."""
    c = np.float32(float(q))
    cands = [np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))]
    cands = [x for x in cands if np.isfinite(x)]
    best = min(abs(Fraction(float(x)) - q) for x in cands)
    tied = [x for x in cands if abs(Fraction(float(x)) - q) == best]
    tied.sort(key=lambda x: int(np.array(x, dtype=np.float32).view(np.uint32)) & 1)
    return tied[0]


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_scale_is_the_correctly_rounded_quotient(fmt):
    rng = np.random.default_rng(7)
    amax = np.concatenate([
        (rng.standard_normal(300) * 10.0 ** rng.integers(-30, 30, 300)).astype(np.float32),
        np.array([1.0, 3.0, 7.0, 448.0, 1e-30, 6e4, 0.1, 1 / 3], dtype=np.float32),
    ])
    amax = np.abs(amax)
    got = fp8.scale(amax, fmt)
    for a, s in zip(amax, got):
        want = _nearest_f32(Fraction(VMAX[fmt]) / Fraction(float(a)))
        assert s == want, (a, s, want)


def test_scale_edge_cases():
    assert fp8.scale(np.float32(0.0)) == 1.0
    assert fp8.scale(np.float32(2.0 ** -120)) == np.finfo(np.float32).max   # quotient beyond fp32
    assert fp8.scale(np.float32(448.0)) == 1.0
    assert fp8.scale(np.float32(57344.0), "e5m2") == 1.0


def _brute_codes(v, s, fmt):
    """Each element: the fp32 product (exact in fp64, then rounded once), clipped to the largest
    finite value, and the nearest of the 256 decoded codes (ties to the even code)."""
    table = mx.e4m3_decode_table() if fmt == "e4m3" else mx.e5m2_decode_table()
    finite = np.isfinite(table)
    out = []
    for x in np.asarray(v, dtype=np.float32).ravel():
        p = float(np.float32(np.float64(x) * np.float64(s)))
        p = min(max(p, -VMAX[fmt]), VMAX[fmt])
        dist = np.where(finite, np.abs(table - p), np.inf)
        best = np.flatnonzero(dist == dist.min())
        same_sign = [c for c in best if (c >> 7) == (1 if np.signbit(p) else 0)] or list(best)
        out.append(min(same_sign, key=lambda c: (c & 1, c)))
    return np.array(out, dtype=np.uint8).reshape(np.shape(v))


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_codes_match_brute_force_nearest(fmt, seed):
    rng = np.random.default_rng(seed)
    v = (rng.standard_normal((6, 40)) * 2.0 ** rng.integers(-12, 12, (6, 1))).astype(np.float32)
    v[0, :4] = [0.0, -0.0, 1e-30, -1e-30]
    codes, s = fp8.quantize(v, fmt)
    assert np.array_equal(codes, _brute_codes(v, s, fmt))


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_tensor_maximum_takes_the_largest_code(fmt):
    rng = np.random.default_rng(3)
    for mag in (1e-20, 1e-3, 1.0, 300.0, 1e6, 1e25):
        v = (rng.standard_normal(500) * mag).astype(np.float32)
        codes, _ = fp8.quantize(v, fmt)
        i = int(np.argmax(np.abs(v)))
        assert codes[i] & 0x7F == TOP[fmt]
        assert (codes[i] >> 7) == (1 if v[i] < 0 else 0)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_power_of_two_rescaling_keeps_the_codes(fmt):
    rng = np.random.default_rng(4)
    v = rng.standard_normal((8, 64)).astype(np.float32)
    c0, s0 = fp8.quantize(v, fmt)
    for k in (-40, -7, -1, 1, 5, 60):
        c, s = fp8.quantize((v * np.float32(2.0 ** k)).astype(np.float32), fmt)
        assert np.array_equal(c, c0), k
        assert float(s) == float(s0) * 2.0 ** -k, k


@pytest.mark.parametrize("fmt,rel,sub", [("e4m3", 2.0 ** -4, 2.0 ** -10), ("e5m2", 2.0 ** -3, 2.0 ** -17)])
def test_round_trip_within_half_a_step(fmt, rel, sub):
    """Half a step of the element format: relative 2**-(m+1) for normal values (m mantissa bits),
    half the subnormal spacing below, both divided by the scale; the fp32 product adds at most
    2**-24 relative."""
    rng = np.random.default_rng(5)
    v = (rng.standard_normal(4000) * np.exp(rng.uniform(-8, 8, 4000))).astype(np.float32)
    codes, s = fp8.quantize(v, fmt)
    back = fp8.dequantize(codes, s, fmt)
    err = np.abs(back - v.astype(np.float64))
    bound = np.maximum(rel * np.abs(v), sub / float(s)) * (1 + 2.0 ** -20)
    assert np.all(err <= bound)
    assert np.count_nonzero(err) > 1000          # the bound is not met by doing nothing


def _grid_tensor(rng, shape, k):
    """Values on the E4M3 grid times 2**k, with the maximum 448 * 2**k in every row."""
    codes = rng.integers(0, 0x7F, shape).astype(np.uint8)
    codes = codes | (rng.integers(0, 2, shape).astype(np.uint8) << 7)
    v = mx.e4m3_decode(codes)
    v[..., 0] = 448.0
    return (v * 2.0 ** k).astype(np.float32)


def test_layer_first_gemm_exact_on_grid_operands():
    """x, W1 and W2 on the scaled grid with every tensor's maximum 448 * 2**k: each scale is 2**-k
    and the quantisation of the first GEMM's operands is exact, so the "fp8" h equals the fp64 h
    rounded to fp32.  A wrong scale, a rounding of an operand to another grid, or an operand
    quantised twice would change it."""
    rng = np.random.default_rng(6)
    T, d, f, E, k = 48, 64, 64, 3, 2
    x = _grid_tensor(rng, (T, d), -9)
    w1 = _grid_tensor(rng, (E, 2 * f, d), -12)
    w2 = _grid_tensor(rng, (E, d, f), -11)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    prob = rng.uniform(0.1, 1.0, (T, k)).astype(np.float32)
    _, st8 = moe.forward(x, idx, prob, w1, w2, "fp8")
    _, st64 = moe.forward(x, idx, prob, w1, w2, "fp64")
    assert np.array_equal(st8["h"], st64["h"].astype(np.float32))
    # a is rounded to bf16 before it is quantised (the fp8 reading), from the fp32 h
    a_ref = moe.bf16_round(moe.f32(moe.silu(st8["h"][:, :f].astype(np.float64)) * st8["h"][:, f:] *
                                   st8["p_perm"][:, None]))
    assert np.array_equal(st8["a"], a_ref)


def test_fp8_refuses_the_mxfp8_saved_h():
    x = np.zeros((4, 32), np.float32)
    with pytest.raises(ValueError):
        moe.forward(x, np.zeros((4, 1), np.int32), np.ones((4, 1), np.float32), np.zeros((1, 64, 32), np.float32),
                    np.zeros((1, 32, 32), np.float32), "fp8", saved_h="mxfp8")
