"""Pins for the oracle's NVFP4 path (row f2): unsigned E4M3 group scales, 16-element
groups, an fp32 tensor scale, and the exact group-scaled product.

Checked against format facts of E4M3 (bias 7, 3 mantissa bits, no infinities, largest
finite 448, smallest subnormal 2^-9), round trips and ties, closed-form groups whose
codes are known, the quantisation error bound of the E2M1 grid, and a brute-force
dequantised matrix product."""
import numpy as np
import pytest

import oracle
import synth


def test_e4m3_value_set():
    v = np.array([oracle.e4m3_value(c) for c in range(127)])
    assert v[0] == 0.0 and v[1] == 2.0 ** -9 and v[7] == 7 * 2.0 ** -9  # subnormals
    assert v[8] == 2.0 ** -6                                             # smallest normal
    assert v[0x38] == 1.0 and v[0x3F] == 1.875 and v[0x40] == 2.0
    assert v[126] == 448.0                                               # largest finite
    assert np.all(np.diff(v) > 0)                                        # strictly increasing
    # every normal binade holds 8 values spaced 2^(e-10)
    for e in range(1, 16):
        seg = v[8 * e: 8 * e + 8] if 8 * e + 8 <= 127 else v[8 * e: 127]
        assert np.allclose(np.diff(seg), 2.0 ** (e - 10))


def test_e4m3_round_trip_ties_and_saturation():
    for c in range(127):
        assert oracle.e4m3_code(oracle.e4m3_value(c)) == c
    for c in range(126):
        mid = (oracle.e4m3_value(c) + oracle.e4m3_value(c + 1)) / 2
        want = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_code(mid) == want
        assert oracle.e4m3_code(np.nextafter(mid, 0)) == c
        assert oracle.e4m3_code(np.nextafter(mid, 1e9)) == c + 1
    assert oracle.e4m3_code(448.0) == 126 and oracle.e4m3_code(1e9) == 126


def test_group_on_the_grid_is_exact():
    """st = 1, group = E2M1 grid values * 2: amax 12, g = 12 / 6 = 2 = E4M3 0x40, S = 2, and
    the codes are the grid's codes (ties are not involved)."""
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    y = np.concatenate([grid, -grid]) * np.float32(2.0)
    codes, sb = oracle.nvfp4_quantize_group(y, 1.0)
    assert sb == 0x40
    want = np.array([oracle.e2m1_code(v / 2.0) for v in y], np.uint8)
    assert np.array_equal(codes, want)


def test_group_edge_cases():
    z, sb = oracle.nvfp4_quantize_group(np.zeros(16, np.float32), 0.5)
    assert sb == 0 and not z.any()                      # all-zero group
    y = np.linspace(-3, 3, 16).astype(np.float32)
    z, sb = oracle.nvfp4_quantize_group(y, 0.0)         # all-zero tensor: st = 0
    assert sb == 0 and not z.any()
    y = np.full(16, 1e-30, np.float32)                  # g underflows to E4M3 0: codes 0
    z, sb = oracle.nvfp4_quantize_group(y, 1.0)
    assert sb == 0 and not z.any()
    y = np.full(16, 2688.0, np.float32)                 # g = 448 exactly
    z, sb = oracle.nvfp4_quantize_group(y, 1.0)
    assert sb == 126 and np.all(z == 7)                 # 2688 / 448 = 6 -> code 7


def test_tensor_quantisation_error_bound():
    """Every element of a quantised tensor is within one E2M1 step (at most 2 units of the
    element scale S in [4, 6], 1 in [2, 4], 0.5 below) of its input, in units of S, and
    the tensor scale makes every group byte finite and at most 448."""
    x, _ = synth.activation_bf16(3, 20, 512, 0.02, 40.0)
    for mode in (oracle.ROT_NONE, oracle.ROT_HADAMARD32):
        st = oracle.nvfp4_tensor_scale(x, mode)
        q, s = oracle.nvfp4_rotate_quantize(x, mode, st)
        assert s.max() <= 126
        xf = synth.bf16_bits_to_f32(x)
        if mode == oracle.ROT_HADAMARD32:
            xf = oracle.rotate_blocks(xf.reshape(-1, 32), mode).reshape(xf.shape)
        deq = oracle.nvfp4_dequantize(q, s, st)
        S = np.repeat(np.vectorize(oracle.e4m3_value)(s.astype(np.int64)), 16, axis=1) * float(st)
        u = np.abs(xf.astype(np.float64)) / np.where(S > 0, S, 1)
        step = np.where(u <= 2, 0.5, np.where(u <= 4, 1.0, 2.0))
        err = np.abs(xf - deq) / np.where(S > 0, S, 1)
        assert np.all(err <= step / 2 + 1e-6 + np.maximum(u - 6, 0))  # saturation beyond 6


def test_nvfp4_gemm_matches_dequantised_product():
    rng = np.random.default_rng(4)
    M, N, K = 5, 7, 96
    aq = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    bq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    as_ = rng.integers(20, 90, (M, K // 16), dtype=np.uint8)
    bs = rng.integers(20, 90, (N, K // 16), dtype=np.uint8)
    ref, S = oracle.nvfp4_gemm(aq, as_, bq, bs, 0.375)
    A = oracle.nvfp4_dequantize(aq, as_, 1.0)
    B = oracle.nvfp4_dequantize(bq, bs, 1.0)
    assert np.allclose(ref, 0.375 * (A @ B.T), rtol=1e-12, atol=0)
    assert np.allclose(S, 0.375 * (np.abs(A) @ np.abs(B).T), rtol=1e-12, atol=0)


def test_nvfp4_scale_layout_is_the_atom_map_with_16_element_groups():
    K = 96
    s = np.arange(3 * (K // 16), dtype=np.uint8).reshape(3, K // 16) + 1
    phys = oracle.nvfp4_sf_to_physical(s, K)
    assert phys.size == oracle.nvfp4_sf_bytes(3, K) == 2 * 512   # ceil(6 / 4) atoms
    for r in range(3):
        for g in range(K // 16):
            off = (g // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + g % 4
            assert phys[off] == s[r, g]


def _f32_inv_sqrt32():
    """fp32 nearest 1/sqrt(32), from 60-digit decimals (independent of the oracle)."""
    from decimal import Decimal, getcontext
    getcontext().prec = 60
    return np.float32(float(Decimal(1) / Decimal(32).sqrt()))


def _bf16(v):
    return synth.f32_to_bf16_bits(np.asarray(v, np.float32))


def test_tensor_scale_closed_form_unrotated():
    """No rotation: st = amax / (6 * 448) in one fp32 rounding. With amax = 2688 * 2^k
    (a bf16 value) st is exactly 2^k, wherever the largest magnitude sits and whatever
    its sign; a wrong divisor (448 or 6 alone) or a signed maximum fails."""
    for k in (-20, -3, 0, 5):
        x = np.zeros((7, 96), np.float32)
        x[0, :] = 0.25 * 2688 * 2.0 ** k          # smaller entries everywhere in row 0
        x[6, 95] = -2688 * 2.0 ** k                # the largest magnitude: last element, negative
        st = oracle.nvfp4_tensor_scale(_bf16(x), oracle.ROT_NONE)
        assert st == np.float32(2.0 ** k)
    # a value that is not a power of two: one fp32 division
    x = np.zeros((2, 32), np.float32)
    x[1, 7] = 3.0
    st = oracle.nvfp4_tensor_scale(_bf16(x), oracle.ROT_NONE)
    assert st == np.float32(np.float32(3.0) / np.float32(2688.0))


def test_tensor_scale_closed_form_after_hadamard():
    """Hadamard mode: the amax is taken after the rotation. A block c * e_0 rotates to 32
    equal values fl(c * fl(1/sqrt(32))) (the butterfly only adds zeros), so st is that value
    / 2688 in one fp32 rounding. A second block with a larger raw maximum b e_0 + ... but a
    smaller rotated one shows that the maximum is not taken before the rotation."""
    c32 = _f32_inv_sqrt32()
    for c in (1.0, 3.0, 448.0, 1.5 * 2.0 ** -10):
        x = np.zeros((3, 128), np.float32)
        x[2, 64] = c                               # block 2 of row 2 is c * e_0
        st = oracle.nvfp4_tensor_scale(_bf16(x), oracle.ROT_HADAMARD32)
        assert st == np.float32(np.float32(np.float32(c) * c32) / np.float32(2688.0))
    # block A = a (e_0 + e_1): rotated even entries fl(2a * c32), odd ones 0;
    # block B = 1.5 a e_0: raw maximum 1.5 a > a, rotated maximum fl(1.5 a * c32) < 2a c32
    a = 8.0
    x = np.zeros((1, 64), np.float32)
    x[0, 0] = x[0, 1] = a
    x[0, 32] = 1.5 * a
    st = oracle.nvfp4_tensor_scale(_bf16(x), oracle.ROT_HADAMARD32)
    want = np.float32(np.float32(np.float32(2 * a) * c32) / np.float32(2688.0))
    assert st == want
    assert st != np.float32(np.float32(1.5 * a) / np.float32(2688.0))
