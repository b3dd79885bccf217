"""Pins for the oracle's MXFP4 format: E2M1 values, rounding, scale rule, round trips.

The oracle is checked here against facts fixed outside it: the E2M1 value
set, every tie case, hand-computed scale bytes, exact round trips of blocks
that are already on the grid, and a brute-force nearest-point search done in
numpy over a dense fp32 sweep.
"""
import os

import numpy as np
import pytest

import oracle


def _read_pairs(path, conv=float):
    rows = []
    with open(path) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                a, b = line.split()
                rows.append((conv(a), int(b)))
    return rows


def test_e2m1_value_set(golden_dir):
    with open(os.path.join(golden_dir, "e2m1_values.txt")) as f:
        vals = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert len(vals) == 16
    for code_s, val_s in vals:
        code, val = int(code_s), float(val_s)
        got = oracle.e2m1_value(code)
        assert got == val and np.signbit(got) == np.signbit(val), (code, got, val)


def test_e2m1_brute_force_all_codes():
    # every code decodes to a grid value and encodes back to itself at scale 2^0
    for code in range(16):
        v = oracle.e2m1_value(code)
        assert oracle.e2m1_code(v) == code, code


def test_e2m1_ties_and_saturation(golden_dir):
    for value, expected in _read_pairs(os.path.join(golden_dir, "e2m1_ties.txt")):
        assert oracle.e2m1_code(value) == expected, (value, expected)


def test_negative_zero_and_small_negatives():
    assert oracle.e2m1_code(-0.0) == 8
    assert oracle.e2m1_code(0.0) == 0
    assert oracle.e2m1_code(-0.1) == 8
    assert oracle.e2m1_code(0.1) == 0
    assert oracle.e2m1_code(-1e-40) == 8


def _grid():
    return np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def test_e2m1_dense_sweep_nearest_even():
    """All fp32 magnitudes in [2^-4, 2^4) with a 2^-7 relative step, plus each
    value's neighbours: the oracle's code is a nearest grid point, and on a tie
    the even one. Independent numpy brute force over the 8 magnitudes."""
    grid = _grid()
    base = np.arange(2 ** 23, dtype=np.uint32)[:: 2 ** 7]
    vals = []
    for exp in range(-4, 4):
        bits = ((exp + 127) << 23) | base
        vals.append(bits.view(np.float32))
    v = np.concatenate(vals)
    v = np.concatenate([v, np.nextafter(v, np.float32(0)), np.nextafter(v, np.float32(100))])
    # the midpoints themselves
    v = np.concatenate([v, (grid[1:] + grid[:-1]).astype(np.float32) / 2]).astype(np.float64)
    codes = oracle.e2m1_codes(v)
    mag = codes & 7
    d = np.abs(v[:, None] - grid[None, :])
    dmin = d.min(axis=1)
    assert np.all(d[np.arange(len(v)), mag] == dmin), "not a nearest grid point"
    tie = (d == dmin[:, None]).sum(axis=1) > 1
    assert np.all(mag[tie] % 2 == 0), "tie not resolved to the even code"
    assert np.all(codes < 8)
    # negatives mirror
    neg = oracle.e2m1_codes(-v)
    assert np.array_equal(neg, codes | 8)


def test_scale_bytes(golden_dir):
    for amax, expected in _read_pairs(os.path.join(golden_dir, "scale_examples.txt"),
                                      conv=float.fromhex):
        assert oracle.scale_exponent(amax) + 127 == expected, (amax, expected)


def test_scale_invariant_amax_over_scale_in_4_8():
    rng = np.random.default_rng(1)
    for _ in range(20000):
        amax = np.float32(np.exp(rng.uniform(-80, 80)))
        e = oracle.scale_exponent(amax)
        r = float(amax) / 2.0 ** e
        assert 4.0 <= r < 8.0, (amax, e)


def test_floor_log2_brute_force_over_exponents():
    for k in range(-149, 128):
        a = np.float32(2.0 ** k)
        assert oracle.floor_log2_f32(a) == k
        if k < 127:
            b = np.nextafter(np.float32(2.0 ** (k + 1)), np.float32(0))
            assert oracle.floor_log2_f32(b) == k


def test_zero_block_and_nonfinite_block():
    codes, s = oracle.quantize_blocks(np.zeros((1, 32), np.float32))
    assert s[0] == 0 and not codes.any()
    y = np.ones((1, 32), np.float32)
    y[0, 5] = np.inf
    codes, s = oracle.quantize_blocks(y)
    assert s[0] == 0xFF and not codes.any()
    y[0, 5] = np.nan
    codes, s = oracle.quantize_blocks(y)
    assert s[0] == 0xFF and not codes.any()


def test_exact_round_trip_of_grid_blocks():
    """Any block whose largest magnitude code is 6 or 7 (value 4 or 6), scaled
    by any byte b in [0, 252], decodes and re-quantises to the same (codes, b)."""
    rng = np.random.default_rng(2)
    grid = _grid()
    for b in range(0, 253):
        for top in (6, 7):
            codes = rng.integers(0, 16, size=32).astype(np.uint8)
            # keep the block maximum at `top`
            codes = np.where((codes & 7) > top, (codes & 8) | top, codes).astype(np.uint8)
            codes[rng.integers(0, 32)] = top | (8 if rng.integers(0, 2) else 0)
            vals = np.where(codes & 8, -1.0, 1.0) * grid[codes & 7] * 2.0 ** (b - 127)
            y = vals.astype(np.float32)
            assert np.array_equal(y.astype(np.float64), vals), "grid value not exact in fp32"
            c2, s2 = oracle.quantize_blocks(y[None, :])
            # +0 and -0 codes: the decoded value keeps its sign, so they survive too
            assert s2[0] == b, (b, top)
            assert np.array_equal(c2[0], codes), (b, top)


def test_bf16_round_pins():
    cases = [
        (1.0, 1.0),
        (1.0 + 2 ** -8, 1.0),                 # tie -> even (mantissa ...0)
        (1.0 + 3 * 2 ** -8, 1.0 + 2 ** -6),   # tie -> even (mantissa ...10)
        (1.0 + 2 ** -8 + 2 ** -30, 1.0 + 2 ** -7),
        (-3.0, -3.0),
        (2.0 ** -130, 2.0 ** -130),           # bf16 subnormal, exact
        (2.0 ** -140, 0.0),                   # below half the smallest bf16 subnormal
        (0.0, 0.0),
    ]
    got = oracle.bf16_round(np.array([c[0] for c in cases]))
    assert np.array_equal(got, np.array([c[1] for c in cases]))


def test_pack_order_low_nibble_first():
    # element 0 = 1.0 (code 2), element 1 = -6 (code 15), rest 0; scale 2^0 needs amax in [4, 8)
    y = np.zeros((1, 32), np.float32)
    y[0, 0] = 1.0
    y[0, 1] = -6.0
    q, s = oracle.rotate_quantize(y, oracle.ROT_NONE, bf16=False)
    assert s[0, 0] == 127
    assert q[0, 0] == (2 | (15 << 4))


def test_sf_layout_map():
    K = 640  # 20 blocks -> 5 atoms of 4 blocks
    rows = 300
    assert oracle.sf_bytes(rows, K) == 3 * 5 * 512
    assert oracle.sf_offset(0, 0, K) == 0
    assert oracle.sf_offset(0, 1, K) == 1
    assert oracle.sf_offset(1, 0, K) == 16
    assert oracle.sf_offset(32, 0, K) == 4
    assert oracle.sf_offset(96, 3, K) == 12 + 3
    assert oracle.sf_offset(0, 4, K) == 512
    assert oracle.sf_offset(128, 0, K) == 5 * 512
    offs = {oracle.sf_offset(r, b, K) for r in range(384) for b in range(20)}
    assert len(offs) == 384 * 20 and max(offs) < oracle.sf_bytes(rows, K)
    s = np.arange(rows * 20, dtype=np.uint32).astype(np.uint8).reshape(rows, 20)
    assert np.array_equal(oracle.sf_from_physical(oracle.sf_to_physical(s, K), rows, K), s)
