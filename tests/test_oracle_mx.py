"""Pins for the oracle's MXFP8 codec (CPU only).

Each check ties the oracle to something other than itself: hand vectors derived
from the format definitions, torch's own float8_e4m3fn conversion (an
independent library routine), exact invariants of a power-of-two block scale,
and brute-force searches.
"""
import os

import numpy as np
import pytest
import torch

from oracle import mx

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mxfp8_hand_vectors.txt")
GOLDEN_FLOOR = os.path.join(os.path.dirname(__file__), "golden", "mxfp8_hand_vectors_floor.txt")
GOLDEN_E5M2 = os.path.join(os.path.dirname(__file__), "golden", "mxfp8_e5m2_hand_vectors.txt")


def _parse_list(s):
    out = []
    for tok in s.split(","):
        tok = tok.strip()
        if " x" in tok:
            v, n = tok.split(" x")
            out += [v.strip()] * int(n)
        else:
            out.append(tok)
    return out


def _golden_cases(path=GOLDEN):
    cases = []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, vals, sbyte, codes = [p.strip() for p in line.split("|")]
        v = [float(x) for x in _parse_list(vals)]
        v = v + [0.0] * (32 - len(v))
        c = [int(x, 16) for x in _parse_list(codes)]
        cases.append((name, np.array(v), int(sbyte, 16), c))
    return cases


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c[0])
def test_hand_vectors(case):
    name, v, sbyte, codes = case
    q, s = mx.quantize_blocks(v[None, :])
    assert int(s[0, 0]) == sbyte
    assert [int(c) for c in q[0, :len(codes)]] == codes


@pytest.mark.parametrize("case", _golden_cases(GOLDEN_FLOOR), ids=lambda c: c[0])
def test_hand_vectors_floor_rule(case):
    name, v, sbyte, codes = case
    q, s = mx.quantize_blocks(v[None, :], rule="floor")
    assert int(s[0, 0]) == sbyte
    assert [int(c) for c in q[0, :len(codes)]] == codes


def test_floor_rule_brute_force_and_relation_to_round_up():
    """floor: 2**(e + 8) <= amax < 2**(e + 9) exactly; the round-up exponent is the floor one or one
    more (one more exactly when amax > 448 * 2**e_floor, the blocks the floor rule saturates)."""
    rng = np.random.default_rng(12)
    amax = np.abs(rng.standard_normal(5000)) * 2.0 ** rng.integers(-60, 60, 5000)
    amax = np.concatenate([amax, 448.0 * 2.0 ** np.arange(-20, 20), 2.0 ** np.arange(-20, 20),
                           np.nextafter(2.0 ** np.arange(-20, 20), 0)])
    ef = mx.e8m0_exponent(amax, "floor")
    ec = mx.e8m0_exponent(amax, "ceil")
    for a, f_, c_ in zip(amax, ef, ec):
        assert 2.0 ** (f_ + 8) <= a < 2.0 ** (f_ + 9)
        assert c_ == f_ + (1 if a > 448.0 * 2.0 ** f_ else 0)


def test_floor_rule_top_binade_and_saturation():
    rng = np.random.default_rng(13)
    x = _bf16_block(rng, 512, spread=30)
    q, s = mx.quantize_blocks(x, rule="floor")
    scaled = np.abs(x) * 2.0 ** -(s[:, 0].astype(np.float64) - 127)[:, None]
    assert np.all(np.max(scaled, axis=1) >= 256) and np.all(np.max(scaled, axis=1) < 512)
    top = q[np.arange(x.shape[0]), np.argmax(np.abs(x), axis=1)] & 0x7F
    assert np.all((top >= 0x78) & (top <= 0x7E))
    sat = np.max(scaled, axis=1) > 448
    assert sat.any() and np.all(top[sat] == 0x7E)
    # torch's float8 conversion of the scaled, clamped values gives the same codes
    ref = torch.from_numpy(np.clip(x * 2.0 ** -(s[:, :1].astype(np.float64) - 127), -448, 448).astype(np.float32))
    assert np.array_equal(ref.to(torch.float8_e4m3fn).view(torch.uint8).numpy(), q)


def test_decode_table_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = mx.e4m3_decode_table()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert np.array_equal(ref[~nan], ours[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def test_encode_matches_torch_rne_in_range():
    rng = np.random.default_rng(0)
    # dense sample over every binade of E4M3 plus all midpoints between adjacent codes
    pos = mx.e4m3_decode_table()[:0x7F]
    mids = (pos[:-1] + pos[1:]) / 2
    v = np.concatenate([pos, mids, -pos, -mids,
                        rng.uniform(-448, 448, 20000),
                        rng.standard_normal(20000) * 2.0 ** rng.integers(-12, 8, 20000)])
    v = v.astype(np.float32)  # torch converts from fp32 here
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = mx.e4m3_encode(v)
    assert np.array_equal(ref, ours)


def test_encode_saturates_and_roundtrips_all_codes():
    table = mx.e4m3_decode_table()
    finite = ~np.isnan(table)
    codes = np.arange(256)[finite]
    assert np.array_equal(mx.e4m3_encode(table[finite]), codes.astype(np.uint8))
    assert mx.e4m3_encode(np.array([449.0, 464.0, 1e6, -1e6])).tolist() == [0x7E, 0x7E, 0x7E, 0xFE]


def test_encode_is_nearest_by_brute_force():
    rng = np.random.default_rng(1)
    table = mx.e4m3_decode_table()
    fin = np.where(~np.isnan(table))[0]
    v = rng.uniform(-460, 460, 4000)
    got = mx.e4m3_encode(v)
    for x, c in zip(v, got):
        dist = np.abs(table[fin] - min(max(x, -448), 448))
        best = dist.min()
        assert abs(table[c] - min(max(x, -448), 448)) == best


def test_e8m0_rule_brute_force():
    rng = np.random.default_rng(2)
    amax = np.abs(rng.standard_normal(5000)) * 2.0 ** rng.integers(-60, 60, 5000)
    amax = np.concatenate([amax, 448.0 * 2.0 ** np.arange(-20, 20), 1.75 * 2.0 ** np.arange(-20, 20)])
    e = mx.e8m0_exponent(amax)
    for a, ei in zip(amax, e):
        assert a <= 448.0 * 2.0 ** ei
        assert a > 448.0 * 2.0 ** (ei - 1)


def test_e8m0_clamps():
    e = mx.e8m0_exponent(np.array([0.0, 2.0 ** -140, 3.0e38]))
    assert e.tolist() == [-127, -127, 120]


def _bf16_block(rng, n_blocks, spread=8):
    x = rng.standard_normal((n_blocks, 32)) * 2.0 ** rng.integers(-spread, spread, (n_blocks, 1))
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def test_power_of_two_scaling_invariance():
    rng = np.random.default_rng(3)
    x = _bf16_block(rng, 256)
    q0, s0 = mx.quantize_blocks(x)
    for sh in (-5, 1, 7):
        q1, s1 = mx.quantize_blocks(x * 2.0 ** sh)
        assert np.array_equal(q0, q1)
        assert np.array_equal(s1.astype(int), s0.astype(int) + sh)


def test_sign_flip_only_flips_sign_bits():
    rng = np.random.default_rng(4)
    x = _bf16_block(rng, 128)
    q0, s0 = mx.quantize_blocks(x)
    q1, s1 = mx.quantize_blocks(-x)
    assert np.array_equal(s0, s1)
    assert np.array_equal(q0 ^ 0x80, q1)


def test_amax_element_lands_in_top_binade_and_never_saturates():
    rng = np.random.default_rng(5)
    x = _bf16_block(rng, 512, spread=30)
    q, s = mx.quantize_blocks(x)
    idx = np.argmax(np.abs(x), axis=1)
    top = q[np.arange(x.shape[0]), idx] & 0x7F
    assert np.all((top >= 0x76) & (top <= 0x7E))
    scaled = np.abs(x) * 2.0 ** -(s[:, 0].astype(np.float64) - 127)[:, None]
    assert np.all(scaled <= 448.0)


def test_grid_values_roundtrip_exactly():
    rng = np.random.default_rng(6)
    table = mx.e4m3_decode_table()
    codes = rng.integers(0, 0x7F, (64, 32)).astype(np.uint8)
    codes[:, 0] = 0x7E                      # make every block's amax code 448 so its scale is exactly 2**sb
    codes |= (rng.integers(0, 2, codes.shape) * 0x80).astype(np.uint8)
    sb = rng.integers(-20, 20, 64)
    x = table[codes] * 2.0 ** sb[:, None]
    q, s = mx.quantize_blocks(x)
    assert np.array_equal(q, codes)
    assert np.array_equal(s[:, 0].astype(int), sb + 127)
    assert np.array_equal(mx.dequantize_blocks(q, s), x)


def test_colwise_is_rowwise_of_transpose_and_axes():
    rng = np.random.default_rng(7)
    x = _bf16_block(rng, 64).reshape(64, 32)
    x = np.concatenate([x, x * 3], axis=1)  # [64, 64]
    qc, sc = mx.quantize_colwise_t(x)
    assert qc.shape == (64, 64) and sc.shape == (64, 2)
    # element [r, c] of x lives at [c, r] of the transposed codes; its block is rows 32*(r//32)..
    r, c = 40, 5
    blk = x[32:64, c]
    e = mx.e8m0_exponent(np.max(np.abs(blk)))
    assert sc[c, 1] == e + 127
    assert qc[c, r] == mx.e4m3_encode(x[r, c] * 2.0 ** -e)


def test_fake_quant_error_bound():
    # relative error of an element in the top binade is at most half an E4M3 ulp (2**-4)
    rng = np.random.default_rng(8)
    x = _bf16_block(rng, 300)
    xq = mx.fake_quant(x, axis=1)
    amax = np.max(np.abs(x), axis=1, keepdims=True)
    err = np.abs(xq - x)
    # absolute error bound per element: half the spacing of the binade the scaled value falls in,
    # at most 2**-4 * |x| for normal codes and 2**-10 * 2**e for subnormal ones
    e = mx.e8m0_exponent(amax[:, 0])[:, None].astype(np.float64)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** (e - 10))
    assert np.all(err <= bound + 0.0)


# ---------------------------------------------------------------- E5M2 elements (gradient variant)
@pytest.mark.parametrize("case", _golden_cases(GOLDEN_E5M2), ids=lambda c: c[0])
def test_hand_vectors_e5m2(case):
    name, v, sbyte, codes = case
    q, s = mx.quantize_blocks(v[None, :], fmt="e5m2")
    assert int(s[0, 0]) == sbyte
    assert [int(c) for c in q[0, :len(codes)]] == codes


def test_e5m2_decode_table_matches_torch_float8():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e5m2).to(torch.float64).numpy()
    ours = mx.e5m2_decode_table()
    assert np.array_equal(np.isnan(ref), np.isnan(ours)) and np.array_equal(np.isinf(ref), np.isinf(ours))
    fin = np.isfinite(ref)
    assert np.array_equal(ref[fin], ours[fin])
    assert ours[0x7B] == 57344.0 and ours[0x01] == 2.0 ** -16


def test_e5m2_encode_matches_torch_rne_in_range():
    rng = np.random.default_rng(20)
    pos = mx.e5m2_decode_table()[:0x7C]
    mids = (pos[:-1] + pos[1:]) / 2
    v = np.concatenate([pos, mids, -pos, -mids, rng.uniform(-57344, 57344, 20000),
                        rng.standard_normal(20000) * 2.0 ** rng.integers(-20, 14, 20000)]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert np.array_equal(ref, mx.e5m2_encode(v))
    assert mx.e5m2_encode(np.array([57344.0, 60000.0, 1e9, -1e9])).tolist() == [0x7B, 0x7B, 0x7B, 0xFB]


@pytest.mark.parametrize("rule", ["ceil", "floor"])
def test_e5m2_exponent_rules_brute_force(rule):
    rng = np.random.default_rng(21)
    amax = np.abs(rng.standard_normal(5000)) * 2.0 ** rng.integers(-60, 60, 5000)
    amax = np.concatenate([amax, 57344.0 * 2.0 ** np.arange(-20, 20), 2.0 ** np.arange(-20, 20)])
    e = mx.e8m0_exponent(amax, rule, "e5m2")
    for a, ei in zip(amax, e):
        if rule == "ceil":
            assert 57344.0 * 2.0 ** (ei - 1) < a <= 57344.0 * 2.0 ** ei
        else:
            assert 2.0 ** (ei + 15) <= a < 2.0 ** (ei + 16)


def test_e5m2_blocks_roundtrip_grid_values_and_never_saturate():
    rng = np.random.default_rng(22)
    table = mx.e5m2_decode_table()
    codes = rng.integers(0, 0x7C, (64, 32)).astype(np.uint8)
    codes[:, 0] = 0x7B                      # every block's amax is 57344 * 2**sb
    codes |= (rng.integers(0, 2, codes.shape) * 0x80).astype(np.uint8)
    sb = rng.integers(-20, 20, 64)
    x = table[codes] * 2.0 ** sb[:, None]
    q, s = mx.quantize_blocks(x, fmt="e5m2")
    assert np.array_equal(q, codes) and np.array_equal(s[:, 0].astype(int), sb + 127)
    assert np.array_equal(mx.dequantize_blocks(q, s, fmt="e5m2"), x)
    y = _bf16_block(rng, 256, spread=30)
    q, s = mx.quantize_blocks(y, fmt="e5m2")
    assert not np.any((q & 0x7F) > 0x7B)    # no infinity or NaN code
