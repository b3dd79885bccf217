"""GPU parity of the GEMM epilogues beyond plain bf16 / fp32 output: a bias, and an MXFP4
output that is the next layer's activation operand.

The expected side comes from the oracle alone. The epilogue takes its decisions (one fp32
bias add, then the rotation, the scale and the codes of every 32-column block) from the
kernel's fp32 accumulator, so the operands of the bit-exact tests are built to make that
accumulator exact: every scale byte of an operand lies within 2 of the others and
K <= 4096, so every product is a whole multiple of the smallest product's quantum and the
largest possible sum stays below 2^24 of those quanta. Any partial sum, in any order, is
then exact in fp32, so the GPU's accumulator equals the oracle's exact product; the
oracle rounds it to fp32 (exact), adds the bias in fp32, and rotates and quantises it.
Codes and scale bytes must match bit for bit.

A second test uses realistic layer inputs, whose fp32 accumulation is not exact: a block
whose decisions all lie farther than the GEMM tolerance (1e-5 * sum |a_i b_i|, spread
through the rotation) from a scale or rounding boundary must match bit for bit; the
others may differ by one step, and their count is reported.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import check_gemm_values, to_dev

pytestmark = pytest.mark.gpu

# few-row kernel (M <= 128, K split over 1-8 CTAs of a cluster) and CTA-pair kernel
# (M > 128; every pair-kernel shape here runs its only round as 256 x 128 column-half
# units, (129, 416, 512) with a last half of 32 columns); N % 128 != 0 included.
SHAPES = [(1, 416, 1024), (5, 128, 4096), (17, 12288, 1024), (128, 4096, 2048),
          (129, 416, 512), (300, 1024, 768), (512, 512, 4096)]


def _operands(M, N, K, seed):
    """Random codes; scale bytes in [125, 127] (A) and [126, 128] (B). The smallest
    nonzero product is 0.25 * 2^(125 + 126 - 254), the largest 36 * 2^(127 + 128 - 254):
    2304 quanta, so K <= 4096 terms stay below 2^24 quanta whatever the order."""
    assert K <= 4096
    aq = synth.uniform_u8(seed, synth.TID_CODES + 20, (M, K // 2), 0, 255)
    as_ = synth.uniform_u8(seed, synth.TID_SCALES + 20, (M, K // 32), 125, 127)
    bq = synth.uniform_u8(seed, synth.TID_CODES + 21, (N, K // 2), 0, 255)
    bs = synth.uniform_u8(seed, synth.TID_SCALES + 21, (N, K // 32), 126, 128)
    return aq, as_, bq, bs


def _exact_product(aq, as_, bq, bs):
    """The oracle's exact product, checked to be an fp32 value (it is, by construction)."""
    ref, _ = oracle.gemm(aq, as_, bq, bs)
    r32 = ref.astype(np.float32)
    assert np.array_equal(r32.astype(np.float64), ref)
    return r32


def _dev(aq, as_, bq, bs, K):
    return (to_dev(aq), to_dev(oracle.sf_to_physical(as_, K)), to_dev(bq),
            to_dev(oracle.sf_to_physical(bs, K)))


def _bias(N, seed):
    return (synth.weight_f32(seed, 1, N, 40)[0] * np.float32(50.0)).astype(np.float32)


def _fp32_gemm(d, M, N, K):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    y = mx.gemm(*d, M, N, K, out_dtype=torch.float32)
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_bias_is_one_fp32_add(M, N, K):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    aq, as_, bq, bs = _operands(M, N, K, M + N)
    d = _dev(aq, as_, bq, bs, K)
    ref = _exact_product(aq, as_, bq, bs)
    assert np.array_equal(_fp32_gemm(d, M, N, K), ref)  # the accumulator is exact
    b = _bias(N, K)
    yb = mx.gemm_bias(*d, M, N, K, to_dev(b), out_dtype=torch.float32)
    yb16 = mx.gemm_bias(*d, M, N, K, to_dev(b))
    torch.cuda.synchronize()
    want = (ref + b[None, :]).astype(np.float32)  # one fp32 rounding
    assert np.array_equal(yb.cpu().numpy().view(np.uint32), want.view(np.uint32))
    got16 = yb16.view(torch.int16).cpu().numpy().view(np.uint16)
    want16 = (oracle.bf16_round(want.astype(np.float64)).astype(np.float32)
              .view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(got16, want16)


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("mode", [0, 1, 2])
def test_mxfp4_output_matches_oracle_quantisation(M, N, K, mode):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    aq, as_, bq, bs = _operands(M, N, K, 7 * M + N)
    d = _dev(aq, as_, bq, bs, K)
    ref = _exact_product(aq, as_, bq, bs)
    A = B = None
    if mode == 2:
        A, B = synth.kron_factors(3)
    for bias in (None, _bias(N, 3)):
        yq, ysf = mx.gemm_quantize(*d, M, N, K, bias=to_dev(bias) if bias is not None else None,
                                   mode=mode, kron_a=A, kron_b=B)
        torch.cuda.synchronize()
        q_ref, s_ref = oracle.quantize_output(ref, bias, mode, A, B)
        got_q = yq.cpu().numpy()
        assert np.array_equal(got_q, q_ref), f"codes {M}x{N}x{K} mode {mode}"
        assert np.array_equal(ysf.cpu().numpy(), oracle.sf_to_physical(s_ref, N)), \
            f"scales {M}x{N}x{K} mode {mode}"


def _open_blocks(ref, S, bias, mode, A=None, B=None):
    """Blocks of the MXFP4 output whose decisions the GEMM tolerance leaves open.

    v = fl(ref + bias) may be off by tau = 1e-5 * S (the accumulator's tolerance) plus
    one rounding; the rotation spreads that to |dr_j| <= sum_i |T_ji| dv_i, plus the
    rotation's own rounding (6 fp32 roundings for the Hadamard butterfly and its
    multiply, 12 for the Kronecker FMA chains) on both sides. A block is open when its
    amax can cross a power of two, or a scaled element |r_j| 2^-e can cross a rounding
    midpoint of the E2M1 grid, or r_j can change sign, within that margin."""
    M, N = ref.shape
    v = ref.astype(np.float32)
    if bias is not None:
        v = (v + bias[None, :]).astype(np.float32)
    vb = v.astype(np.float64).reshape(M, N // 32, 32)
    dv = (1e-5 * S + 2.0 ** -23 * np.abs(ref)).reshape(M, N // 32, 32) + \
        2.0 ** -23 * np.abs(vb)
    if mode == 1:
        T = np.full((32, 32), 1 / np.sqrt(32.0))
        rounds = 6
    elif mode == 2:
        T = np.abs(np.kron(A.astype(np.float64), B.astype(np.float64)))
        rounds = 12
    else:
        T = np.eye(32)
        rounds = 0
    r = oracle.rotate_blocks(v.reshape(-1, 32), mode, A, B).astype(np.float64)
    r = r.reshape(M, N // 32, 32)
    marg = dv @ T.T + 2 * rounds * 2.0 ** -24 * (np.abs(vb) @ T.T) + 2.0 ** -24 * np.abs(r)
    amax = np.abs(r).max(-1)
    mmax = marg.max(-1)
    with np.errstate(divide="ignore"):
        lo = np.floor(np.log2(np.maximum(amax - mmax, 0)))
        hi = np.floor(np.log2(amax + mmax))
    e = np.floor(np.log2(np.where(amax > 0, amax, 1))) - 2
    s = np.abs(r) * 2.0 ** -e[..., None]
    ms = marg * 2.0 ** -e[..., None]
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    near_mid = (np.min(np.abs(s[..., None] - mids), -1) <= ms).any(-1)
    near_zero = (np.abs(r) <= marg).any(-1)
    return (lo != hi) | near_mid | near_zero


def test_mxfp4_output_realistic_inputs():
    """A DiT-like layer (3072 -> 1024, activations with outlier channels, Hadamard-rotated
    MXFP4 on both sides), its output re-quantised with a bias for a Hadamard next layer.
    Blocks the tolerance decides are bit-exact; the open ones are within one step."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    M, N, K = 512, 1024, 3072
    x, _ = synth.activation_bf16(5, M, K, 0.01, 30.0)
    w = synth.weight_f32(5, N, K, 6)
    wq, ws = oracle.prepare_weight(w, oracle.ROT_HADAMARD32)
    xq, xs = oracle.rotate_quantize(x, oracle.ROT_HADAMARD32)
    ref, S = oracle.gemm(xq, xs, wq, ws)
    bias = (synth.weight_f32(5, 1, N, 7)[0] * np.float32(20.0)).astype(np.float32)
    d = _dev(xq, xs, wq, ws, K)
    yq, ysf = mx.gemm_quantize(*d, M, N, K, bias=to_dev(bias), mode=1)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quantize_output(ref, bias, 1)
    open_ = _open_blocks(ref, S, bias, 1)
    got_s = oracle.sf_from_physical(ysf.cpu().numpy(), M, N)
    gq = oracle.unpack_codes(yq.cpu().numpy()).reshape(M, N // 32, 32)
    eq = oracle.unpack_codes(q_ref).reshape(M, N // 32, 32)
    same = (gq == eq).all(-1) & (got_s == s_ref)
    assert same[~open_].all(), f"{(~same & ~open_).sum()} decided blocks differ"
    # open blocks: scale within one step; where the scale agrees, codes within one step
    ds = np.abs(got_s.astype(int) - s_ref.astype(int))
    assert (ds[open_] <= 1).all()
    mag = lambda c: (c & 7).astype(int)
    step_ok = (np.abs(mag(gq) - mag(eq)) <= 1).all(-1) | (ds != 0)
    assert step_ok[open_].all()
    print(f"MXFP4 output, realistic layer: {open_.sum()} of {open_.size} blocks open "
          f"({open_.mean():.1%}), {(~same).sum()} differ")


def test_mxfp4_output_feeds_the_next_layer():
    """Two layers with no bf16 in between: layer 1 writes MXFP4 (Hadamard-rotated), layer 2
    consumes it directly; layer 2's result is the exact product of the oracle's layer-1
    quantisation (from the exact layer-1 product) with W2, within the GEMM tolerance."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    M, K, N1, N2 = 384, 1024, 2048, 512
    aq, as_, bq, bs = _operands(M, N1, K, 11)
    d = _dev(aq, as_, bq, bs, K)
    y1 = _exact_product(aq, as_, bq, bs)
    b1 = _bias(N1, 5)
    yq, ysf = mx.gemm_quantize(*d, M, N1, K, bias=to_dev(b1), mode=1)
    w2 = synth.weight_f32(9, N2, N1, 41)
    w2q, w2s = oracle.prepare_weight(w2, 1)
    y2 = mx.gemm(yq, ysf, to_dev(w2q), to_dev(oracle.sf_to_physical(w2s, N1)), M, N2, N1,
                 out_dtype=torch.float32)
    torch.cuda.synchronize()
    q1, s1 = oracle.quantize_output(y1, b1, 1)
    assert np.array_equal(yq.cpu().numpy(), q1)
    ref, S = oracle.gemm(q1, s1, w2q, w2s)
    check_gemm_values(y2.cpu().numpy().astype(np.float64), ref, S, "f32", "layer 2")
