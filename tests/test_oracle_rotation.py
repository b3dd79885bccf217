"""Pins for the oracle's block rotations (Hadamard-32 and Kronecker A(x)B).

Checked against explicit matrices built here from their closed forms
(H_ij = (-1)^popcount(i & j) / sqrt(32); (A(x)B)[8i+k, 8j+l] = A_ij B_kl via
numpy.kron), orthogonality / invertibility identities, and the fp32 error
bounds of the stated evaluation orders.
"""
import math
from decimal import Decimal, getcontext

import numpy as np
import pytest

import oracle
import synth


def _sylvester(n=32):
    i = np.arange(n)
    pc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1.0, -1.0)


def test_inv_sqrt32_is_nearest_fp32():
    getcontext().prec = 60
    exact = Decimal(1) / Decimal(32).sqrt()
    c = oracle.inv_sqrt32()
    lo = np.nextafter(c, np.float32(0))
    hi = np.nextafter(c, np.float32(1))
    err = abs(Decimal(float(c)) - exact)
    assert err <= abs(Decimal(float(lo)) - exact)
    assert err <= abs(Decimal(float(hi)) - exact)


def test_unnormalised_butterfly_is_sylvester_integer_exact():
    H = _sylvester()
    cols = np.stack([oracle.fwht32_unnormalised(np.eye(32, dtype=np.float32)[j]) for j in range(32)],
                    axis=1)
    assert np.array_equal(cols, H)                   # column j = H e_j, exact integers
    assert np.array_equal(cols @ cols.T, 32 * np.eye(32))


def test_hadamard_orthonormal_in_fp32():
    Hn = oracle.rotate_blocks(np.eye(32, dtype=np.float32), oracle.ROT_HADAMARD32)
    # rows of the block-rotated identity are H e_j (H is symmetric)
    G = Hn.astype(np.float64) @ Hn.astype(np.float64).T
    assert np.max(np.abs(G - np.eye(32))) < 1e-6


def test_hadamard_matches_explicit_matrix():
    H = _sylvester() / math.sqrt(32.0)
    x = synth.normal_f32(0, 999, (200, 32))
    x[:, 3] *= 50.0
    y = oracle.rotate_blocks(x, oracle.ROT_HADAMARD32).astype(np.float64)
    ref = x.astype(np.float64) @ H.T
    # 5 add stages + 1 multiply: relative error per element <= ~6u of sum |x|/sqrt(32)
    bound = 8 * 2.0 ** -24 * (np.abs(x).astype(np.float64).sum(axis=1, keepdims=True) / math.sqrt(32))
    assert np.all(np.abs(y - ref) <= bound + 1e-30)
    # involution: H (H x) = x within fp32 error
    yy = oracle.rotate_blocks(y.astype(np.float32), oracle.ROT_HADAMARD32).astype(np.float64)
    assert np.max(np.abs(yy - x) / (np.abs(x).max(axis=1, keepdims=True))) < 1e-5


def test_kron_matches_numpy_kron():
    A, B = synth.kron_factors(0)
    T = np.kron(A.astype(np.float64), B.astype(np.float64))
    x = synth.normal_f32(0, 998, (300, 32))
    y = oracle.rotate_blocks(x, oracle.ROT_KRON_4x8, A, B).astype(np.float64)
    ref = x.astype(np.float64) @ T.T
    absT = np.kron(np.abs(A).astype(np.float64), np.abs(B).astype(np.float64))
    bound = 16 * 2.0 ** -24 * (np.abs(x).astype(np.float64) @ absT.T)
    assert np.all(np.abs(y - ref) <= bound)


def test_kron_identity_factors_is_identity():
    x = synth.normal_f32(0, 997, (10, 32))
    y = oracle.rotate_blocks(x, oracle.ROT_KRON_4x8, np.eye(4), np.eye(8))
    assert np.array_equal(y, x)


def test_kron_weight_factors_invert():
    A, B = synth.kron_factors(0)
    assert abs(np.linalg.det(A.astype(np.float64))) > 1e-3
    assert abs(np.linalg.det(B.astype(np.float64))) > 1e-3
    Ai = oracle.inverse(A)
    Bi = oracle.inverse(B)
    I = np.kron(A.astype(np.float64), B.astype(np.float64)) @ np.kron(Ai, Bi)
    assert np.max(np.abs(I - np.eye(32))) < 1e-12
    At, Bt = oracle.kron_weight_factors(A, B)
    assert np.max(np.abs(At.astype(np.float64) - Ai.T)) < 1e-6
    assert np.max(np.abs(Bt.astype(np.float64) - Bi.T)) < 1e-6


def test_rotation_invariance_of_dot_products():
    """(H x).(H w) = x.w and (T x).(T^-T w) = x.w, evaluated through the oracle's
    fp32 rotations: catches transposed factors and wrong conventions."""
    x = synth.normal_f32(0, 996, (64, 32))
    w = synth.normal_f32(0, 995, (64, 32), 0.02)
    base = np.sum(x.astype(np.float64) * w.astype(np.float64), axis=1)
    scale = np.sqrt(np.sum(x.astype(np.float64) ** 2, 1) * np.sum(w.astype(np.float64) ** 2, 1))
    hx = oracle.rotate_blocks(x, oracle.ROT_HADAMARD32).astype(np.float64)
    hw = oracle.rotate_blocks(w, oracle.ROT_HADAMARD32).astype(np.float64)
    assert np.max(np.abs(np.sum(hx * hw, 1) - base) / scale) < 1e-5
    A, B = synth.kron_factors(0)
    At, Bt = oracle.kron_weight_factors(A, B)
    tx = oracle.rotate_blocks(x, oracle.ROT_KRON_4x8, A, B).astype(np.float64)
    tw = oracle.rotate_blocks(w, oracle.ROT_KRON_4x8, At, Bt).astype(np.float64)
    assert np.max(np.abs(np.sum(tx * tw, 1) - base) / scale) < 1e-4
    # and a wrong convention (T^-1 instead of T^-T on w) breaks it
    Ai, Bi = oracle.inverse(A).astype(np.float32), oracle.inverse(B).astype(np.float32)
    bad = oracle.rotate_blocks(w, oracle.ROT_KRON_4x8, Ai, Bi).astype(np.float64)
    assert np.max(np.abs(np.sum(tx * bad, 1) - base) / scale) > 1e-3


def test_rotate_quantize_composes_rotation_and_quantisation():
    xb, _ = synth.activation_bf16(0, 8, 256, 0.02, 20.0)
    x32 = synth.bf16_bits_to_f32(xb)
    q, s = oracle.rotate_quantize(xb, oracle.ROT_HADAMARD32)
    y = oracle.rotate_blocks(x32.reshape(-1, 32), oracle.ROT_HADAMARD32)
    codes, sc = oracle.quantize_blocks(y)
    assert np.array_equal(oracle.unpack_codes(q).reshape(-1, 32), codes)
    assert np.array_equal(s.reshape(-1), sc)


def test_quantize_output_adds_bias_once_in_fp32_then_quantises():
    """MXFP4 output: row r of y + bias lands exactly on the E2M1 grid times 2^3, so the
    codes are the grid's codes and every scale byte is 127 + 3 (amax 48 = 6 * 2^3)."""
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    target = np.concatenate([grid, -grid[::-1], grid, -grid[::-1]]) * 8.0  # 32 values
    target[target == 0] = 0.0  # (y - b) + b is +0 in IEEE arithmetic, never -0
    bias = (np.arange(32) % 5 - 2).astype(np.float32) * np.float32(0.25)  # exact quarters
    y = np.stack([target - bias.astype(np.float64)] * 3).astype(np.float32)  # exact in fp32
    q, s = oracle.quantize_output(y, bias, oracle.ROT_NONE)
    codes = oracle.unpack_codes(q)
    want = np.array([oracle.e2m1_code(v / 8.0) for v in target], np.uint8)
    assert np.array_equal(codes, np.stack([want] * 3))
    assert np.all(s == 130)
    # no bias: the same as quantising y itself
    q0, s0 = oracle.quantize_output(y, None, oracle.ROT_HADAMARD32)
    q1, s1 = oracle.rotate_quantize(y, oracle.ROT_HADAMARD32, bf16=False)
    assert np.array_equal(q0, q1) and np.array_equal(s0, s1)


def test_quantize_output_rounds_the_sum_once():
    """y + bias is one fp32 rounding (ties to even): 1 + 2^-24 -> 1, 1 + 3 * 2^-24 -> 1 + 2^-22."""
    y = np.ones((1, 32), np.float32)
    b = np.zeros(32, np.float32)
    b[0], b[1] = 2.0 ** -24, 3 * 2.0 ** -24
    yb = (y + b[None, :]).astype(np.float32)
    assert yb[0, 0] == np.float32(1.0) and yb[0, 1] == np.float32(1.0 + 2.0 ** -22)
    q, s = oracle.quantize_output(y, b, oracle.ROT_NONE)
    q2, s2 = oracle.rotate_quantize(yb, oracle.ROT_NONE, bf16=False)
    assert np.array_equal(q, q2) and np.array_equal(s, s2)


# ---- larger Hadamard blocks (n = 64, 128 elements = 2, 4 MX blocks)

@pytest.mark.parametrize("n", [64, 128])
def test_larger_butterfly_is_sylvester_integer_exact(n):
    H = _sylvester(n)
    cols = oracle.fwht_unnormalised(np.eye(n, dtype=np.float32)).T  # column j = H e_j
    assert np.array_equal(cols, H)
    assert np.array_equal(cols @ cols.T, n * np.eye(n))


def test_larger_normalisers_are_nearest_fp32():
    getcontext().prec = 60
    for n in (64, 128):
        e = np.zeros((1, n), np.float32)
        e[0, 0] = 1.0
        c = oracle.hadamard_n(e)[0, 0]  # (H_n e_0)_0 = the normaliser itself
        exact = Decimal(1) / Decimal(n).sqrt()
        for nb in (np.nextafter(c, np.float32(0)), np.nextafter(c, np.float32(1))):
            assert abs(Decimal(float(c)) - exact) <= abs(Decimal(float(nb)) - exact)
    assert oracle.hadamard_n(np.eye(64, dtype=np.float32)[:1])[0, 0] == np.float32(0.125)


@pytest.mark.parametrize("n", [64, 128])
def test_larger_hadamard_matches_explicit_matrix_and_is_an_involution(n):
    H = _sylvester(n) / math.sqrt(n)
    x = synth.normal_f32(1, 998, (100, n))
    x[:, 5] *= 40.0
    y = oracle.hadamard_n(x).astype(np.float64)
    ref = x.astype(np.float64) @ H.T
    stages = int(math.log2(n))
    bound = (stages + 3) * 2.0 ** -24 * (np.abs(x).astype(np.float64).sum(axis=1, keepdims=True)
                                         / math.sqrt(n))
    assert np.all(np.abs(y - ref) <= bound + 1e-30)
    yy = oracle.hadamard_n(y.astype(np.float32)).astype(np.float64)
    assert np.max(np.abs(yy - x) / np.abs(x).max(axis=1, keepdims=True)) < 2e-5


@pytest.mark.parametrize("mode,n", [(oracle.ROT_HADAMARD64, 64), (oracle.ROT_HADAMARD128, 128)])
def test_larger_block_modes_rotate_groups_then_quantise_per_32(mode, n):
    xb, _ = synth.activation_bf16(2, 6, 512, 0.02, 20.0)
    x32 = synth.bf16_bits_to_f32(xb)
    q, s = oracle.rotate_quantize(xb, mode)
    y = oracle.hadamard_n(x32.reshape(-1, n)).reshape(-1, 32)
    codes, sc = oracle.quantize_blocks(y)
    assert np.array_equal(oracle.unpack_codes(q).reshape(-1, 32), codes)
    assert np.array_equal(s.reshape(-1), sc)
    # weights rotated the same way: the layer's dot products are preserved (H_n orthonormal)
    w = synth.weight_f32(2, 4, 512, 3)
    yw = oracle.hadamard_n(w.reshape(-1, n)).reshape(4, 512).astype(np.float64)
    ref = x32.astype(np.float64) @ w.astype(np.float64).T
    got = oracle.hadamard_n(x32.reshape(-1, n)).reshape(6, 512).astype(np.float64) @ yw.T
    assert np.max(np.abs(got - ref)) < 1e-4 * np.abs(ref).max()
