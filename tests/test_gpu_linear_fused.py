"""The layer for 1..8 activation rows runs as one kernel that rotates and quantises x
inside the GEMM's CTAs. Its output must equal, byte for byte, the two-step path (the
quantiser, then the few-row GEMM on the quantised operands: the same splits and the same
summation order), and match the oracle's layer."""
import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import bf16_dev_to_f64, check_gemm_values, to_dev, to_dev_bf16
from test_gpu_gemm import _sample_pairs

pytestmark = pytest.mark.gpu

MODES = [oracle.ROT_NONE, oracle.ROT_HADAMARD32, oracle.ROT_KRON_4x8]


def _weights(N, K, mode, seed):
    w = synth.weight_f32(seed, N, K, 1)
    A = B = None
    if mode == oracle.ROT_KRON_4x8:
        A, B = synth.kron_factors(seed)
    wq, ws = oracle.prepare_weight(w, mode, A, B)
    return wq, ws, A, B


def _both_paths(x, wq, ws, N, mode, A, B):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    M, K = x.shape
    xd = to_dev_bf16(x)
    wq_d, wsf_d = to_dev(wq), to_dev(oracle.sf_to_physical(ws, K))
    y = mx.linear(xd, wq_d, wsf_d, N, mode, A, B)
    xq_d, xsf_d = mx.rotate_quantize(xd, mode, A, B)
    y2 = mx.gemm(xq_d, xsf_d, wq_d, wsf_d, M, N, K)
    y3 = mx.linear_noalloc(xd, wq_d, wsf_d, N, mode, A, B)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16)), "fused != two-step"
    assert torch.equal(y.view(torch.int16), y3.view(torch.int16)), "fused != no-alloc"
    return bf16_dev_to_f64(y)


# (M, N, K): several W tiles and K splits, a K tail inside the last k-tile (K = 1056:
# 33 blocks), one row, the 8-row limit, and a split of 8 with 5 k-tiles per CTA.
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M,N,K", [(1, 128, 256), (3, 256, 1056), (8, 384, 2048),
                                   (7, 4096, 3072), (8, 1152, 8448)])
def test_fused_layer_matches_two_step_and_oracle(M, N, K, mode):
    import mxfp4_quantized_linear_block_b200 as mx
    assert mx.linear_kernel_count(M, N, K, mode) == 1
    x, _ = synth.activation_bf16(11 + M, M, K, 0.01, 30.0)
    wq, ws, A, B = _weights(N, K, mode, 5)
    y = _both_paths(x, wq, ws, N, mode, A, B)
    ref, S, _, _ = oracle.linear(x, wq, ws, mode, A, B)
    check_gemm_values(y, ref, S, "bf16", f"fused M{M} N{N} K{K} mode{mode}")


def test_beyond_fused_limits_falls_back():
    """More than 12 k-tiles per CTA (150 W tiles: one split of 14 k-tiles), 9 rows and 17
    rows take the two-kernel path; results as before."""
    import mxfp4_quantized_linear_block_b200 as mx
    for M, N, K in [(5, 150 * 128, 3584), (9, 256, 1024), (17, 256, 1024)]:
        assert mx.linear_kernel_count(M, N, K, oracle.ROT_HADAMARD32) == 2
        x, _ = synth.activation_bf16(3, M, K, 0.01, 30.0)
        wq, ws, A, B = _weights(N, K, oracle.ROT_HADAMARD32, 6)
        y = _both_paths(x, wq, ws, N, oracle.ROT_HADAMARD32, A, B)
        xq, xs = oracle.rotate_quantize(x, oracle.ROT_HADAMARD32)
        mi, ni = _sample_pairs(M, N, n_random=2048, seed=M)
        ref, S = oracle.gemm_pairs(xq, xs, wq, ws, mi, ni)
        check_gemm_values(y[mi, ni], ref, S, "bf16", f"fallback M{M} N{N} K{K}")


def test_fused_layer_repeatable_and_status_clear():
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    M, N, K = 6, 640, 1536
    x, _ = synth.activation_bf16(2, M, K, 0.01, 30.0)
    wq, ws, A, B = _weights(N, K, oracle.ROT_HADAMARD32, 7)
    xd = to_dev_bf16(x)
    wq_d, wsf_d = to_dev(wq), to_dev(oracle.sf_to_physical(ws, K))
    wsp = mx.new_workspace(mx.workspace_bytes(mx.OP_LINEAR, M, N, K))
    ys = [mx.linear(xd, wq_d, wsf_d, N, oracle.ROT_HADAMARD32, ws=wsp) for _ in range(3)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(ys[0].view(torch.int16), y.view(torch.int16))
    assert mx.poll_status(wsp) == mx.OK
