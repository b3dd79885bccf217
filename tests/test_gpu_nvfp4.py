"""GPU parity of the NVFP4 path (row f2) against the oracle: tensor scale and E4M3 group
bytes and codes bit for bit, the tcgen05 kind::mxf4nvf4 GEMM within the GEMM tolerance,
and the whole NVFP4 layer."""
import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import bf16_dev_to_f64, check_gemm_values, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

MODES = [oracle.ROT_NONE, oracle.ROT_HADAMARD32]


def _dev_x(x):
    return to_dev_bf16(x) if x.dtype == np.uint16 else to_dev(x)


def _quantize(x, mode, ld_pad=0):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    rows, K = x.shape
    if ld_pad:
        big = np.zeros((rows, K + ld_pad), x.dtype)
        big[:, :K] = x
        d = _dev_x(big)[:, :K]
    else:
        d = _dev_x(x)
    sc = mx.nvfp4_tensor_scale(d, mode)
    q, sf = mx.nvfp4_quantize(d, sc, mode)
    torch.cuda.synchronize()
    return sc.cpu().numpy()[0], q.cpu().numpy(), sf.cpu().numpy()[: oracle.nvfp4_sf_bytes(rows, K)]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rows,K", [(1, 32), (5, 96), (127, 160), (129, 512), (300, 3072)])
def test_nvfp4_quantize_bit_exact(mode, dtype, rows, K):
    x, _ = synth.activation_bf16(rows * 3 + K, rows, K, 0.02, 40.0)
    if dtype == "f32":
        x = synth.bf16_bits_to_f32(x) * np.float32(1.37)
    st, q, sf = _quantize(x, mode)
    st_ref = oracle.nvfp4_tensor_scale(x, mode)
    assert np.float32(st) == st_ref
    q_ref, s_ref = oracle.nvfp4_rotate_quantize(x, mode, st_ref)
    assert np.array_equal(q, q_ref)
    assert np.array_equal(sf, oracle.nvfp4_sf_to_physical(s_ref, K))


def test_nvfp4_quantize_edges_and_strides():
    """Groups whose g lands on E4M3 ties and at 448, zero groups, an all-zero tensor,
    subnormal-scale groups; rows read with a padded stride."""
    rng = np.random.default_rng(9)
    rows, K = 40, 256
    x = rng.standard_normal((rows, K)).astype(np.float32)
    x[0, :16] = 0.0                                    # zero group
    x[1, :16] = 2688.0 * np.linspace(-1, 1, 16)        # amax = tensor amax: g = 448
    x[2, 16:32] = 1e-6                                 # g far below E4M3's range
    for r in range(3, 12):                             # g on E4M3 midpoints (st fixed below)
        x[r, :16] *= 0.0
        x[r, 0] = 6.0 * (oracle.e4m3_value(r) + oracle.e4m3_value(r + 1)) / 2 * 2688.0 / 2688.0
    st, q, sf = _quantize(x, oracle.ROT_NONE, ld_pad=32)
    q_ref, s_ref = oracle.nvfp4_rotate_quantize(x, oracle.ROT_NONE, np.float32(st))
    assert np.float32(st) == oracle.nvfp4_tensor_scale(x, oracle.ROT_NONE)
    assert np.array_equal(q, q_ref)
    assert np.array_equal(sf, oracle.nvfp4_sf_to_physical(s_ref, K))
    z = np.zeros((7, 64), np.float32)                  # all-zero tensor: st = 0
    st0, q0, sf0 = _quantize(z, oracle.ROT_HADAMARD32)
    assert st0 == 0.0 and not q0.any() and not sf0.any()


def _nv_operands(M, N, K, seed):
    aq = synth.uniform_u8(seed, synth.TID_CODES + 30, (M, K // 2), 0, 255)
    bq = synth.uniform_u8(seed, synth.TID_CODES + 31, (N, K // 2), 0, 255)
    as_ = synth.uniform_u8(seed, synth.TID_SCALES + 30, (M, K // 16), 24, 80)
    bs = synth.uniform_u8(seed, synth.TID_SCALES + 31, (N, K // 16), 24, 80)
    return aq, as_, bq, bs


# few-row kernel (M <= 128; clusters of 1-8 K splits) and CTA-pair kernel (M > 128;
# every pair-kernel shape here runs its last round as 256 x 128 column-half units: N = 144
# ends in a half of 16 columns, N = 384 in a half wholly past N); K tails at 32 / 96 of 64
NV_SHAPES = [(1, 16, 64), (5, 400, 2080), (16, 256, 8192), (128, 4096, 2048), (129, 144, 96),
             (300, 384, 1056), (512, 512, 4096), (768, 1024, 8192)]


@pytest.mark.parametrize("M,N,K", NV_SHAPES)
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_nvfp4_gemm(M, N, K, out):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    aq, as_, bq, bs = _nv_operands(M, N, K, M + N + K)
    sa = torch.tensor([0.75, 0.0], dtype=torch.float32, device="cuda")
    sb = torch.tensor([1.0 / 3.0, 0.0], dtype=torch.float32, device="cuda")
    y = mx.nvfp4_gemm(to_dev(aq), to_dev(oracle.nvfp4_sf_to_physical(as_, K)), sa, to_dev(bq),
                      to_dev(oracle.nvfp4_sf_to_physical(bs, K)), sb, M, N, K,
                      out_dtype=torch.float32 if out == "f32" else torch.bfloat16)
    torch.cuda.synchronize()
    alpha = float(np.float32(np.float32(0.75) * np.float32(1.0 / 3.0)))
    ref, S = oracle.nvfp4_gemm(aq, as_, bq, bs, alpha)
    got = y.cpu().numpy().astype(np.float64) if out == "f32" else bf16_dev_to_f64(y)
    check_gemm_values(got, ref, S, out, f"nvfp4 gemm {M}x{N}x{K} {out}")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M", [16, 384])
def test_nvfp4_linear(mode, M):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    K, N = 1024, 512
    x, _ = synth.activation_bf16(M + 1, M, K, 0.01, 30.0)
    w = synth.weight_f32(3, N, K, 6)
    w_d = torch.from_numpy(w).cuda()
    w_sc = mx.nvfp4_tensor_scale(w_d, mode)
    wq, wsf = mx.nvfp4_quantize(w_d, w_sc, mode)
    y = mx.nvfp4_linear(to_dev_bf16(x), wq, wsf, w_sc, N, mode)
    torch.cuda.synchronize()
    st_w = oracle.nvfp4_tensor_scale(w, mode)
    wq_r, ws_r = oracle.nvfp4_rotate_quantize(w, mode, st_w)
    assert np.array_equal(wq.cpu().numpy(), wq_r)
    st_x = oracle.nvfp4_tensor_scale(x, mode)
    xq_r, xs_r = oracle.nvfp4_rotate_quantize(x, mode, st_x)
    alpha = float(np.float32(st_x) * np.float32(st_w))
    ref, S = oracle.nvfp4_gemm(xq_r, xs_r, wq_r, ws_r, alpha)
    check_gemm_values(bf16_dev_to_f64(y), ref, S, "bf16", f"nvfp4 linear M{M} mode {mode}")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M", [16, 300])
@pytest.mark.parametrize("factor", [0.25, 1.0, 4.0])
def test_nvfp4_linear_static_scale(mode, M, factor):
    """The NVFP4 layer with a static activation tensor scale: the dynamic scale of x times
    `factor` (0.25: many groups saturate at group scale 448; 4: finer groups), given on
    the device; against the oracle's quantisation with that same scale."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    K, N = 1024, 512
    x, _ = synth.activation_bf16(M + 2, M, K, 0.01, 30.0)
    w = synth.weight_f32(4, N, K, 6)
    w_d = torch.from_numpy(w).cuda()
    w_sc = mx.nvfp4_tensor_scale(w_d, mode)
    wq, wsf = mx.nvfp4_quantize(w_d, w_sc, mode)
    st_x = np.float32(np.float32(oracle.nvfp4_tensor_scale(x, mode)) * np.float32(factor))
    x_sc = torch.tensor([float(st_x), 0.0], dtype=torch.float32, device="cuda")
    y = mx.nvfp4_linear_static(to_dev_bf16(x), x_sc, wq, wsf, w_sc, N, mode)
    torch.cuda.synchronize()
    st_w = oracle.nvfp4_tensor_scale(w, mode)
    wq_r, ws_r = oracle.nvfp4_rotate_quantize(w, mode, st_w)
    xq_r, xs_r = oracle.nvfp4_rotate_quantize(x, mode, st_x)
    alpha = float(np.float32(st_x) * np.float32(st_w))
    ref, S = oracle.nvfp4_gemm(xq_r, xs_r, wq_r, ws_r, alpha)
    check_gemm_values(bf16_dev_to_f64(y), ref, S, "bf16",
                      f"nvfp4 static-scale linear M{M} mode {mode} x{factor}")


def test_nvfp4_linear_static_zero_scale():
    """A static activation scale of 0 gives zero codes, so a zero output."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    M, K, N = 40, 256, 128
    x, _ = synth.activation_bf16(5, M, K, 0.01, 30.0)
    w_d = torch.from_numpy(synth.weight_f32(5, N, K, 6)).cuda()
    w_sc = mx.nvfp4_tensor_scale(w_d, oracle.ROT_NONE)
    wq, wsf = mx.nvfp4_quantize(w_d, w_sc, oracle.ROT_NONE)
    x_sc = torch.zeros(2, dtype=torch.float32, device="cuda")
    y = mx.nvfp4_linear_static(to_dev_bf16(x), x_sc, wq, wsf, w_sc, N, oracle.ROT_NONE)
    torch.cuda.synchronize()
    assert not bool(y.float().abs().max() > 0)


def test_nvfp4_tensor_scale_of_empty_and_zero_tensors():
    """amax of no elements, or of zeros only, is 0, so the tensor scale is 0 (written over
    whatever the 2-float buffer held, by the pass's one block when there are no rows)."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    for rows in (0, 3):
        for mode in (oracle.ROT_NONE, oracle.ROT_HADAMARD32):
            for dt in (torch.bfloat16, torch.float32):
                x = torch.zeros((rows, 96), dtype=dt, device="cuda")
                sc = torch.full((2,), 7.5, dtype=torch.float32, device="cuda")
                mx.nvfp4_tensor_scale(x, mode, scale2=sc)
                torch.cuda.synchronize()
                assert float(sc[0]) == 0.0, (rows, mode, dt)


def test_nvfp4_linear_repeated_on_one_workspace():
    """The layer's tensor-scale pass keeps its running maximum and block counter in the
    workspace and leaves them zero: a call whose x has a smaller amax than the one before
    on the same workspace gets its own scale (a leftover maximum would inflate it)."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    M, K, N, mode = 300, 1024, 512, oracle.ROT_HADAMARD32
    w = synth.weight_f32(4, N, K, 6)
    w_d = torch.from_numpy(w).cuda()
    w_sc = mx.nvfp4_tensor_scale(w_d, mode)
    wq, wsf = mx.nvfp4_quantize(w_d, w_sc, mode)
    st_w = oracle.nvfp4_tensor_scale(w, mode)
    wq_r, ws_r = oracle.nvfp4_rotate_quantize(w, mode, st_w)
    ws = mx.new_workspace(mx.workspace_bytes(mx.OP_NVFP4_LINEAR, M, N, K))
    big, _ = synth.activation_bf16(7, M, K, 0.01, 30.0)
    small = synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(big) * np.float32(0.125))
    for x in (big, small, big):
        y = mx.nvfp4_linear(to_dev_bf16(x), wq, wsf, w_sc, N, mode, ws=ws)
        torch.cuda.synchronize()
        st_x = oracle.nvfp4_tensor_scale(x, mode)
        xq_r, xs_r = oracle.nvfp4_rotate_quantize(x, mode, st_x)
        alpha = float(np.float32(st_x) * np.float32(st_w))
        ref, S = oracle.nvfp4_gemm(xq_r, xs_r, wq_r, ws_r, alpha)
        check_gemm_values(bf16_dev_to_f64(y), ref, S, "bf16", "nvfp4 linear, shared workspace")
    assert mx.poll_status(ws) == mx.OK
