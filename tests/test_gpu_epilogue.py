"""GPU parity of the GEMM epilogues beyond plain bf16 / fp32 output: a bias, and an MXFP4
output that is the next layer's activation operand.

The quantised output is decided from the kernel's own fp32 accumulator, so the oracle
takes the same decisions from the same fp32 values: the fp32 output of the same GEMM
(the same MMAs and split order) is checked against the exact contraction first, then
oracle.quantize_output(that fp32 output, bias, mode) must match codes and scale bytes bit
for bit, padding included."""
import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import check_gemm_values, to_dev

pytestmark = pytest.mark.gpu

# few-row kernel (M <= 128, K split over 1-8 CTAs of a cluster) and CTA-pair kernel
# (M > 128; (512, 512, 4096) splits its only round along K); N % 128 != 0 included.
SHAPES = [(1, 416, 1024), (5, 128, 4096), (17, 12288, 1024), (128, 4096, 2048),
          (129, 416, 512), (300, 1024, 768), (512, 512, 4096)]


def _operands(M, N, K, seed):
    aq = synth.uniform_u8(seed, synth.TID_CODES + 20, (M, K // 2), 0, 255)
    as_ = synth.uniform_u8(seed, synth.TID_SCALES + 20, (M, K // 32), 112, 138)
    bq = synth.uniform_u8(seed, synth.TID_CODES + 21, (N, K // 2), 0, 255)
    bs = synth.uniform_u8(seed, synth.TID_SCALES + 21, (N, K // 32), 112, 138)
    return aq, as_, bq, bs


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
    y = _fp32_gemm(d, M, N, K)
    ref, S = oracle.gemm(aq, as_, bq, bs)
    check_gemm_values(y.astype(np.float64), ref, S, "f32", f"no bias {M}x{N}x{K}")
    b = _bias(N, K)
    yb = mx.gemm_bias(*d, M, N, K, to_dev(b), out_dtype=torch.float32)
    yb16 = mx.gemm_bias(*d, M, N, K, to_dev(b))
    torch.cuda.synchronize()
    want = (y + b[None, :]).astype(np.float32)
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
    y = _fp32_gemm(d, M, N, K)
    A = B = None
    if mode == 2:
        A, B = synth.kron_factors(3)
    for bias in (None, _bias(N, 3)):
        yq, ysf = mx.gemm_quantize(*d, M, N, K, bias=to_dev(bias) if bias is not None else None,
                                   mode=mode, kron_a=A, kron_b=B)
        torch.cuda.synchronize()
        q_ref, s_ref = oracle.quantize_output(y, bias, mode, A, B)
        got_q = yq.cpu().numpy()
        assert np.array_equal(got_q, q_ref), f"codes {M}x{N}x{K} mode {mode}"
        assert np.array_equal(ysf.cpu().numpy(), oracle.sf_to_physical(s_ref, N)), \
            f"scales {M}x{N}x{K} mode {mode}"


def test_mxfp4_output_feeds_the_next_layer():
    """Two layers with no bf16 in between: layer 1 writes MXFP4 (Hadamard-rotated), layer 2
    consumes it directly; layer 2's result is the exact product of the oracle's layer-1
    quantisation with W2, within the GEMM tolerance."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    M, K, N1, N2 = 384, 1024, 2048, 512
    aq, as_, bq, bs = _operands(M, N1, K, 11)
    d = _dev(aq, as_, bq, bs, K)
    y1 = _fp32_gemm(d, M, N1, K)
    b1 = _bias(N1, 5)
    yq, ysf = mx.gemm_quantize(*d, M, N1, K, bias=to_dev(b1), mode=1)
    w2 = synth.weight_f32(9, N2, N1, 41)
    w2q, w2s = oracle.prepare_weight(w2, 1)
    y2 = mx.gemm(yq, ysf, to_dev(w2q), to_dev(oracle.sf_to_physical(w2s, N1)), M, N2, N1,
                 out_dtype=torch.float32)
    torch.cuda.synchronize()
    q1, s1 = oracle.quantize_output(y1, b1, 1)
    ref, S = oracle.gemm(q1, s1, w2q, w2s)
    check_gemm_values(y2.cpu().numpy().astype(np.float64), ref, S, "f32", "layer 2")
