"""Pins for the oracle's norm prologue (row f3): row statistics against closed forms, the
identity case, and the fp32 order of the per-element affine steps."""
import math

import numpy as np
import pytest

import oracle


def test_layernorm_stats_closed_forms():
    n = 96
    rows = np.stack([np.arange(n, dtype=np.float32) * 0.5 + 7.0,      # arithmetic sequence
                     np.full(n, -3.25, np.float32)])                  # constant row
    mu, rstd = oracle.row_stats(rows, oracle.NORM_LAYER, 1e-5)
    var = (n * n - 1) / 12.0 * 0.25                                  # variance of k * 0.5
    assert mu[0] == pytest.approx(7.0 + 0.5 * (n - 1) / 2, abs=0, rel=1e-15)
    assert rstd[0] == pytest.approx(1.0 / math.sqrt(var + 1e-5), rel=1e-14)
    assert mu[1] == -3.25 and rstd[1] == pytest.approx(1.0 / math.sqrt(1e-5), rel=1e-14)


def test_rmsnorm_stats_closed_form():
    a = 1.75
    row = np.where(np.arange(64) % 2 == 0, a, -a).astype(np.float32)[None, :]
    mu, rstd = oracle.row_stats(row, oracle.NORM_RMS, 1e-6)
    assert mu[0] == 0.0
    assert rstd[0] == pytest.approx(1.0 / math.sqrt(a * a + 1e-6), rel=1e-14)


def test_identity_statistics_reduce_to_rotate_quantize():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((9, 128)).astype(np.float32)
    for mode in (oracle.ROT_NONE, oracle.ROT_HADAMARD32):
        q, s = oracle.norm_rotate_quantize(x, np.zeros(9), np.ones(9), None, None, mode)
        q2, s2 = oracle.rotate_quantize(x, mode, bf16=False)
        assert np.array_equal(q, q2) and np.array_equal(s, s2)


def test_affine_order_lands_on_the_grid():
    """((x - mu) * rstd) * g + b with mu = 3, rstd = 0.25, g = 2, b = 0.5 maps
    x = 2 t + 2 exactly to t: the codes are the E2M1 grid's, the scale byte 127 + 0."""
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    t = np.concatenate([grid, grid[::-1], grid, grid]).astype(np.float32)      # 32 values
    x = (2.0 * t + 2.0).astype(np.float32)[None, :]
    g = np.full(32, 2.0, np.float32)
    b = np.full(32, 0.5, np.float32)
    q, s = oracle.norm_rotate_quantize(x, np.array([3.0]), np.array([0.25]), g, b,
                                       oracle.ROT_NONE)
    want = np.array([oracle.e2m1_code(v) for v in t], np.uint8)
    assert np.array_equal(oracle.unpack_codes(q)[0], want)
    assert s[0, 0] == 127  # amax 6: floor(log2 6) - 2 = 0
