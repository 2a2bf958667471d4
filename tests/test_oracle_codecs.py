"""Pins for the oracle's NVFP4 codecs (CPU only).

Each test ties the oracle to something other than itself: the format
definition of the pages ("Full-Stack FP4", Section 2, paragraph "NVFP4
format"), an independent library codec (ml_dtypes, torch float8), exact
rational brute force, or hand-worked blocks under tests/golden/.
"""
import json
import math
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import nvfp4 as Q


# ---------------------------------------------------------------- E2M1 codes

def test_e2m1_all_codes_decode_like_library():
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    ours = Q.code_values(np.arange(16, dtype=np.uint8))
    assert np.array_equal(np.signbit(lib), np.signbit(ours))
    assert np.array_equal(np.abs(lib), np.abs(ours))
    assert sorted(set(np.abs(ours).tolist())) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_every_code_reencodes_to_itself():
    mags = Q.E2M1_MAGNITUDES
    assert np.array_equal(Q.e2m1_encode_magnitude(mags), np.arange(8, dtype=np.uint8))


def test_e2m1_encode_matches_library_rne_with_saturation():
    rng = np.random.default_rng(0)
    q = np.concatenate([
        rng.uniform(0, 7, 200000).astype(np.float32),
        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 6.5, 100.0], np.float32),
        np.nextafter(np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32), np.float32(0)),
        np.nextafter(np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32), np.float32(9)),
    ])
    lib = q.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0x7
    assert np.array_equal(Q.e2m1_encode_magnitude(q), lib)


# ---------------------------------------------------------------- E4M3 bytes

def test_e4m3_all_bytes_decode_like_two_libraries():
    b = np.arange(256, dtype=np.uint8)
    lib1 = b.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    lib2 = torch.from_numpy(b.copy()).view(torch.float8_e4m3fn).double().numpy()
    ours = Q.E4M3_VALUES
    for lib in (lib1, lib2):
        nan = np.isnan(lib)
        assert np.array_equal(nan, np.isnan(ours))
        assert np.array_equal(lib[~nan], ours[~nan])
    assert set(np.flatnonzero(np.isnan(ours)).tolist()) == {0x7F, 0xFF}
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def test_e4m3_encode_matches_library_rne_in_range():
    rng = np.random.default_rng(1)
    v = np.concatenate([
        np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), 300000)).astype(np.float32),
        (Q.E4M3_VALUES[1:0x7E] + Q.E4M3_VALUES[2:0x7F]).astype(np.float32) / 2,   # midpoints
        Q.E4M3_VALUES[:0x7F].astype(np.float32),
    ])
    v = v[v <= 448.0]
    lib = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(Q.e4m3_encode(v), lib)


def test_e4m3_encode_saturates_above_448():
    v = np.array([448.0, 460.0, 464.0, 480.0, 1e6, 3e38], np.float32)
    assert np.all(Q.e4m3_encode(v) == 0x7E)


# ---------------------------------------------------------------- tensor scale

@pytest.mark.parametrize("amax", [1e-30, 3e-6, 0.02, 0.9, 1.0, 6.0, 12.0, 2688.0, 2688.5, 1e6, 3e38])
def test_pow2_tensor_scale_is_smallest_power_of_two_covering_amax(amax):
    s = float(Q.global_scale(amax))
    e = math.log2(s)
    assert e == int(e)
    a = float(np.float32(amax))
    if Q.SG_EXP_MIN < e < Q.SG_EXP_MAX:
        assert Fraction(2688) * Fraction(s) >= Fraction(a)
        assert Fraction(2688) * Fraction(s) / 2 < Fraction(a)


def test_tensor_scale_of_zero_tensor_is_one():
    assert Q.global_scale(0.0) == 1.0
    c, s, g = Q.quantize_rows(np.zeros((2, 32), np.float32))
    assert g == 1.0 and not c.any() and not s.any()


# ---------------------------------------------------------------- hand-worked blocks

def _golden(golden_dir):
    with open(os.path.join(golden_dir, "hand_blocks.json")) as f:
        return json.load(f)["cases"]


def test_hand_worked_blocks(golden_dir):
    for case in _golden(golden_dir):
        x = np.array(case["x"], np.float32)[None, :]
        codes, scales, s_g = Q.quantize_rows(x)
        assert float(s_g) == case["s_g"], case["name"]
        assert [f"{b:02x}" for b in scales[0]] == case["scales_hex"], case["name"]
        assert [f"{b:02x}" for b in codes[0]] == case["codes_hex"], case["name"]
        for dt in (np.float64, np.float32):
            y = Q.dequantize_rows(codes, scales, s_g, dtype=dt)[0]
            want = np.array(case["dequantized"], dt)
            assert np.array_equal(y, want), case["name"]
            assert np.array_equal(np.signbit(y), np.signbit(want)), case["name"]


# ---------------------------------------------------------------- brute force

def _nearest_even_exact(value: Fraction, grid):
    """Exhaustive nearest search over (code, Fraction) pairs, tie -> even code."""
    best = None
    for code, g in grid:
        d = abs(value - g)
        if best is None or d < best[0] or (d == best[0] and code % 2 == 0):
            best = (d, code)
    return best[1]


_E2M1_GRID = [(i, Fraction(v)) for i, v in enumerate([0, 0.5, 1, 1.5, 2, 3, 4, 6])]
_E4M3_GRID = [(i, Fraction(Q.E4M3_VALUES[i])) for i in range(0x7F)]


def _brute_quantize_block(xs, s_g):
    s_g = np.float32(s_g)
    amax = max(abs(float(v)) for v in xs)
    v = np.float32(np.float32(amax) / (np.float32(6.0) * s_g))
    sb = 0x7E if v >= 448 else _nearest_even_exact(Fraction(float(v)), _E4M3_GRID)
    den = np.float32(np.float32(Q.E4M3_VALUES[sb]) * s_g)
    codes = []
    for x in xs:
        if den == 0:
            codes.append(0)
            continue
        q = np.float32(abs(x) / den)
        mag = 7 if q >= 6 else _nearest_even_exact(Fraction(float(q)), _E2M1_GRID)
        codes.append(mag | (8 if np.signbit(x) else 0))
    return sb, codes


def test_quantize_matches_exhaustive_rational_search_on_tiny_blocks():
    rng = np.random.default_rng(7)
    for trial in range(60):
        kind = trial % 4
        if kind == 0:
            x = rng.standard_normal((2, 16))
        elif kind == 1:   # values exactly on E2M1 ties after scaling
            x = rng.choice([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], (2, 16)) * rng.choice([-1, 1], (2, 16))
        elif kind == 2:   # wide dynamic range inside the tensor: subnormal and zero scales
            x = rng.standard_normal((2, 16)) * np.exp(rng.uniform(-14, 4, (2, 1)))
        else:
            x = rng.standard_t(3, (2, 16)) * 0.02
        x = x.astype(np.float32)
        codes, scales, s_g = Q.quantize_rows(x)
        nib = Q.unpack_codes(codes)
        for r in range(2):
            sb, want = _brute_quantize_block(x[r], s_g)
            assert scales[r, 0] == sb
            assert nib[r].tolist() == want


def test_textbook_amax_scale_mode_matches_brute_force():
    rng = np.random.default_rng(8)
    x = (rng.standard_normal((4, 32)) * 0.3).astype(np.float32)
    codes, scales, s_g = Q.quantize_rows(x, mode="amax")
    assert s_g == np.float32(np.float32(np.max(np.abs(x))) / np.float32(2688.0))
    nib = Q.unpack_codes(codes)
    for r in range(4):
        for blk in range(2):
            sb, want = _brute_quantize_block(x[r, 16 * blk:16 * blk + 16], s_g)
            assert scales[r, blk] == sb
            assert nib[r, 16 * blk:16 * blk + 16].tolist() == want


# ---------------------------------------------------------------- properties

def test_dequantised_value_is_nearest_grid_point_of_scaled_input():
    """For every unsaturated element, x_hat/den is the grid point nearest to x/den."""
    rng = np.random.default_rng(9)
    x = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    codes, scales, s_g = Q.quantize_rows(x)
    y = Q.dequantize_rows(codes, scales, s_g)
    den = np.repeat(Q.E4M3_VALUES[scales] * float(s_g), 16, axis=1)
    err = np.abs(np.abs(x.astype(np.float64)) / den - np.abs(y) / den)
    grid = Q.E2M1_MAGNITUDES
    q = np.abs(x) / den
    gap = np.diff(grid)[np.clip(np.searchsorted(grid, q) - 1, 0, 6)]
    unsat = q <= 6
    assert np.all(err[unsat] <= gap[unsat] / 2 + 1e-6)


def test_power_of_two_tensor_scale_invariance():
    """With a power-of-two s_g, multiplying s_g by 2^d leaves every dequantised
    value unchanged as long as no block scale becomes an E4M3 subnormal."""
    rng = np.random.default_rng(10)
    x = (rng.standard_t(3, (128, 512)) * 0.02).astype(np.float32)
    c0, s0, g0 = Q.quantize_rows(x)
    y0 = Q.dequantize_rows(c0, s0, g0)
    for d in range(1, 5):
        c, s, g = Q.quantize_rows(x, s_g=float(g0) * 2.0 ** d)
        normal = np.repeat(s >= 0x08, 16, axis=1)
        y = Q.dequantize_rows(c, s, g)
        assert np.array_equal(y[normal], y0[normal])
        assert np.array_equal(Q.unpack_codes(c)[normal], Q.unpack_codes(c0)[normal])


def test_float32_and_float64_dequantisation_agree_for_pow2_scale():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((32, 64)) * 5).astype(np.float32)
    c, s, g = Q.quantize_rows(x)
    assert np.array_equal(Q.dequantize_rows(c, s, g, np.float32).astype(np.float64),
                          Q.dequantize_rows(c, s, g, np.float64))


def test_column_quantisation_is_row_quantisation_of_transpose():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((48, 32)).astype(np.float32)
    c, s, g = Q.quantize_cols(x)
    assert c.shape == (32, 24) and s.shape == (32, 3)
    y = Q.dequantize_cols(c, s, g)
    assert y.shape == x.shape
    # blocks run down the columns: each 16-row slice of a column has one scale
    for j in range(32):
        for blk in range(3):
            col = x[16 * blk:16 * blk + 16, j]
            sb, want = _brute_quantize_block(col, g)
            assert s[j, blk] == sb
            assert Q.unpack_codes(c)[j, 16 * blk:16 * blk + 16].tolist() == want


def test_rejects_bad_input():
    with pytest.raises(ValueError):
        Q.quantize_rows(np.ones((2, 10), np.float32))
    with pytest.raises(ValueError):
        Q.quantize_rows(np.array([[np.nan] * 16], np.float32))
    with pytest.raises(TypeError):
        Q.quantize_rows(np.ones((2, 16), np.float64))


def test_exact_signed_zeros_keep_their_sign_bit():
    """E2M1 is sign-magnitude (1 sign, 2 exponent, 1 mantissa bit), so in a block with a
    non-zero scale a zero element keeps its sign: an exact -0.0 gets code 0x8 and +0.0
    gets 0x0.  A block whose scale rounds to 0 (here an all-zero block) is written as
    all-zero codes, signs included (the reading for a zero block scale)."""
    x = np.zeros((2, 32), np.float32)
    x[0, :16] = [-0.0, 0.0] * 8                       # all-zero block: scale byte 0
    x[0, 16:] = [4.0, -0.0, 0.0, -4.0] + [0.0] * 12   # live block with signed zeros
    x[1, :15] = 1.0
    x[1, 15] = -0.0                                   # last element of a live block
    codes, scales, _ = Q.quantize_rows(x)
    nib = Q.unpack_codes(codes)
    assert scales[0, 0] == 0 and np.all(nib[0, :16] == 0)
    assert scales[0, 1] != 0
    assert nib[0, 17] == 0x8 and nib[0, 18] == 0x0
    assert nib[0, 16] & 8 == 0 and nib[0, 19] & 8 == 8
    assert nib[1, 15] == 0x8 and np.all(nib[1, :15] == 0x7)   # the block amax maps to 6
