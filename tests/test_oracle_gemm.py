"""Pins for the oracle's block-scaled contraction.

Brute force: dequantise both operands to double with a decode written here
from the E2M1 value set and the E8M0 definition (2^(b-127)), then a plain
triple loop / numpy matmul on tiny shapes. Special cases: one nonzero pair,
all-zero operands, scale handling across blocks.
"""
import numpy as np

import oracle
import synth

_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _decode(q, s):
    rows, K = q.shape[0], q.shape[1] * 2
    codes = np.empty((rows, K), np.int64)
    codes[:, 0::2] = q & 15
    codes[:, 1::2] = q >> 4
    vals = np.where(codes & 8, -1.0, 1.0) * _GRID[codes & 7]
    return vals * np.repeat(2.0 ** (s.astype(np.float64) - 127.0), 32, axis=1)


def _rand_operands(seed, rows, K, lo=110, hi=140, tid=0):
    q = synth.uniform_u8(seed, synth.TID_CODES + tid, (rows, K // 2), 0, 255)
    s = synth.uniform_u8(seed, synth.TID_SCALES + tid, (rows, K // 32), lo, hi)
    return q, s


def test_brute_force_tiny_shapes():
    for K in (32, 64, 96):
        for M, N in ((1, 1), (3, 5), (8, 8)):
            aq, as_ = _rand_operands(K, M, K, tid=0)
            bq, bs = _rand_operands(K, N, K, tid=1)
            A = _decode(aq, as_)
            B = _decode(bq, bs)
            ref, S = oracle.gemm(aq, as_, bq, bs)
            for m in range(M):
                for n in range(N):
                    tot = 0.0
                    mag = 0.0
                    for k in range(K):
                        tot += A[m, k] * B[n, k]
                        mag += abs(A[m, k] * B[n, k])
                    assert abs(ref[m, n] - tot) <= 1e-12 * mag + 1e-300
                    assert abs(S[m, n] - mag) <= 1e-12 * mag + 1e-300


def test_matches_dequantised_matmul_medium():
    aq, as_ = _rand_operands(7, 40, 512, 100, 150, tid=2)
    bq, bs = _rand_operands(7, 24, 512, 100, 150, tid=3)
    ref, S = oracle.gemm(aq, as_, bq, bs)
    A, B = _decode(aq, as_), _decode(bq, bs)
    full = A @ B.T
    assert np.all(np.abs(ref - full) <= 1e-12 * (np.abs(A) @ np.abs(B).T))
    assert np.allclose(S, np.abs(A) @ np.abs(B).T, rtol=1e-12)


def test_single_nonzero_pair_exact():
    K = 128
    aq = np.zeros((1, K // 2), np.uint8)
    bq = np.zeros((1, K // 2), np.uint8)
    as_ = np.full((1, K // 32), 127, np.uint8)
    bs = np.full((1, K // 32), 127, np.uint8)
    # element 70 (block 2, high nibble of byte 35): a = -3 (code 13), b = 1.5 (code 3)
    aq[0, 35] = 13 << 4
    bq[0, 35] = 3 << 4
    as_[0, 2] = 130   # 2^3
    bs[0, 2] = 120    # 2^-7
    ref, S = oracle.gemm(aq, as_, bq, bs)
    assert ref[0, 0] == -3 * 1.5 * 2.0 ** (3 - 7)
    assert S[0, 0] == 3 * 1.5 * 2.0 ** (3 - 7)


def test_all_zero_operands():
    aq = np.zeros((4, 64), np.uint8)
    as_ = synth.uniform_u8(0, 77, (4, 4), 0, 254)
    bq, bs = _rand_operands(1, 5, 128)
    ref, S = oracle.gemm(aq, as_, bq, bs)
    assert not ref.any() and not S.any()


def test_pairs_equal_full():
    aq, as_ = _rand_operands(3, 17, 256, tid=4)
    bq, bs = _rand_operands(3, 9, 256, tid=5)
    ref, S = oracle.gemm(aq, as_, bq, bs)
    mi = np.array([0, 16, 5, 5, 16])
    ni = np.array([0, 8, 3, 0, 0])
    r2, S2 = oracle.gemm_pairs(aq, as_, bq, bs, mi, ni)
    assert np.array_equal(r2, ref[mi, ni]) and np.array_equal(S2, S[mi, ni])


def test_linear_equals_rotated_float_product_up_to_quantisation():
    """End-to-end oracle linear vs the unquantised product x.w in double: the
    MXFP4 error must be of the size the 4-bit grid allows (a loose sanity pin
    that the rotation is applied to X and W consistently)."""
    wl = synth.WORKLOADS["tiny"].linears[0]
    xb, _ = synth.activation_bf16(0, wl.M, wl.K, wl.outlier_frac, wl.outlier_factor)
    w = synth.weight_f32(0, wl.N, wl.K)
    wq, ws = oracle.prepare_weight(w, oracle.ROT_HADAMARD32)
    ref, S, _, _ = oracle.linear(xb, wq, ws, oracle.ROT_HADAMARD32)
    exact = synth.bf16_bits_to_f32(xb).astype(np.float64) @ w.astype(np.float64).T
    rel = np.linalg.norm(ref - exact) / np.linalg.norm(exact)
    assert rel < 0.2, rel
    # without the rotation the error is larger on outlier-heavy activations
    wq0, ws0 = oracle.prepare_weight(w, oracle.ROT_NONE)
    ref0, _, _, _ = oracle.linear(xb, wq0, ws0, oracle.ROT_NONE)
    rel0 = np.linalg.norm(ref0 - exact) / np.linalg.norm(exact)
    assert rel < rel0, (rel, rel0)
