"""GPU parity of the norm prologue (row f3): the kernel's row statistics against exact
arithmetic, and codes / scale bytes bit for bit against the oracle's normalise-rotate-
quantise run with those fp32 statistics; then the layer."""
import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import bf16_dev_to_f64, check_gemm_values, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


def _vec(seed, K, mean, std):
    return (mean + std * synth.normal_f32(seed, 77, (1, K))[0]).astype(np.float32)


@pytest.mark.parametrize("kind", [oracle.NORM_LAYER, oracle.NORM_RMS])
# K <= 51168 takes the one-pass kernel (groups of 16 / 8 / 4 / 2 / 1 rows per CTA for
# K = 3072 / 6144 / 12288 / 24576 / 51168, with a partial last group); K = 51200 the
# statistics kernel + norm quantiser.
@pytest.mark.parametrize("rows,K", [(1, 64), (5, 3072), (129, 1024), (17, 6144),
                                    (300, 12288), (7, 24576), (3, 51168), (3, 51200)])
@pytest.mark.parametrize("affine", [False, True])
def test_norm_rotate_quantize(kind, rows, K, affine):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    x, _ = synth.activation_bf16(rows + K + kind, rows, K, 0.01, 30.0)
    xb = synth.bf16_bits_to_f32(x)
    x = synth.f32_to_bf16_bits(xb * np.float32(3.0) + np.float32(1.5))  # non-zero mean
    g = _vec(1, K, 1.0, 0.2) if affine else None
    b = _vec(2, K, 0.0, 0.5) if affine else None
    A, B = synth.kron_factors(0)
    for mode in (oracle.ROT_NONE, oracle.ROT_HADAMARD32, oracle.ROT_KRON_4x8):
        q, sf, st = mx.norm_rotate_quantize(
            to_dev_bf16(x), kind, 1e-6, to_dev(g) if affine else None,
            to_dev(b) if affine else None, mode, A if mode == 2 else None,
            B if mode == 2 else None)
        torch.cuda.synchronize()
        st = st.cpu().numpy()
        mu, rstd = oracle.row_stats(x, kind, 1e-6)
        # fp32 summation of K terms: |error| <= K u sum|x_i| (u = 2^-24), twice for safety;
        # the variance inherits the same relative bound
        u = 2.0 ** -24
        mean_abs = np.abs(synth.bf16_bits_to_f32(x).astype(np.float64)).mean(axis=1)
        assert np.all(np.abs(st[:, 0] - mu) <= 2 * K * u * mean_abs + 1e-30)
        assert np.all(np.abs(st[:, 1] - rstd) <= (2 * K * u + 1e-6) * rstd)
        q_ref, s_ref = oracle.norm_rotate_quantize(x, st[:, 0], st[:, 1], g, b, mode,
                                                   A if mode == 2 else None,
                                                   B if mode == 2 else None)
        assert np.array_equal(q.cpu().numpy(), q_ref), f"codes mode {mode}"
        assert np.array_equal(sf.cpu().numpy()[: oracle.sf_bytes(rows, K)],
                              oracle.sf_to_physical(s_ref, K)), f"scales mode {mode}"


@pytest.mark.parametrize("kind", [oracle.NORM_LAYER, oracle.NORM_RMS])
@pytest.mark.parametrize("M", [16, 384])
def test_norm_linear(kind, M):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    K, N = 3072, 1024
    x, _ = synth.activation_bf16(M + 5, M, K, 0.01, 30.0)
    g = _vec(3, K, 1.0, 0.1)
    b = _vec(4, K, 0.0, 0.3)
    w = synth.weight_f32(4, N, K, 7)
    wq, ws = oracle.prepare_weight(w, oracle.ROT_HADAMARD32)
    y = mx.norm_linear(to_dev_bf16(x), to_dev(wq), to_dev(oracle.sf_to_physical(ws, K)), N, kind,
                       1e-6, to_dev(g), to_dev(b), oracle.ROT_HADAMARD32)
    # the layer's statistics are the standalone call's (same kernel, same inputs)
    _, _, st = mx.norm_rotate_quantize(to_dev_bf16(x), kind, 1e-6, to_dev(g), to_dev(b),
                                       oracle.ROT_HADAMARD32)
    torch.cuda.synchronize()
    st = st.cpu().numpy()
    xq, xs = oracle.norm_rotate_quantize(x, st[:, 0], st[:, 1], g, b, oracle.ROT_HADAMARD32)
    ref, S = oracle.gemm(xq, xs, wq, ws)
    check_gemm_values(bf16_dev_to_f64(y), ref, S, "bf16", f"norm linear kind {kind} M{M}")
