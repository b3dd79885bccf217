"""GPU parity of the whole layer (rotate + quantise + block-scaled GEMM, bf16 out)
on the workload recipes, with pre-quantised weights prepared by the oracle."""
import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import bf16_dev_to_f64, check_gemm_values, to_dev, to_dev_bf16
from test_gpu_gemm import _sample_pairs

pytestmark = pytest.mark.gpu


def _layer_inputs(wl, lin):
    x, _ = synth.activation_bf16(wl.seed, lin.M, lin.K, lin.outlier_frac, lin.outlier_factor,
                                 lin.x_tensor)
    w = synth.weight_f32(wl.seed, lin.N, lin.K, lin.layer)
    A = B = None
    if wl.rotation == oracle.ROT_KRON_4x8:
        A, B = synth.kron_factors(wl.seed)
    wq, ws = oracle.prepare_weight(w, wl.rotation, A, B)
    return x, wq, ws, A, B


def _run_linear(x, wq, ws, N, mode, A, B, workspace=None):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    K = x.shape[1]
    y = mx.linear(to_dev_bf16(x), to_dev(wq), to_dev(oracle.sf_to_physical(ws, K)), N, mode, A, B,
                  ws=workspace)
    torch.cuda.synchronize()
    return bf16_dev_to_f64(y)


@pytest.mark.parametrize("name", ["tiny"])
def test_linear_full_compare(name):
    wl = synth.WORKLOADS[name]
    for lin in wl.linears:
        x, wq, ws, A, B = _layer_inputs(wl, lin)
        y = _run_linear(x, wq, ws, lin.N, wl.rotation, A, B)
        ref, S, _, _ = oracle.linear(x, wq, ws, wl.rotation, A, B)
        check_gemm_values(y, ref, S, "bf16", f"{name}/{lin.name}")


@pytest.mark.parametrize("name", ["dit_b1", "kron", "llm_small_m1", "llm_small_m16",
                                  "llm_small_m128"])
def test_linear_workloads_sampled(name):
    wl = synth.WORKLOADS[name]
    for lin in wl.linears:
        x, wq, ws, A, B = _layer_inputs(wl, lin)
        y = _run_linear(x, wq, ws, lin.N, wl.rotation, A, B)
        xq, xs = oracle.rotate_quantize(x, wl.rotation, A, B)
        mi, ni = _sample_pairs(lin.M, lin.N, n_random=4096, seed=lin.layer)
        ref, S = oracle.gemm_pairs(xq, xs, wq, ws, mi, ni)
        check_gemm_values(y[mi, ni], ref, S, "bf16", f"{name}/{lin.name}")


@pytest.mark.parametrize("j", [0, 1])
def test_linear_batch16_sampled(j):
    """Both layers of the batch-16 DiT MLP at full size (57344 tokens): 3072 -> 12288 and
    12288 -> 3072, each one kernel (quantiser warps beside the CTA-pair GEMM). Every code
    and scale byte the quantiser warps leave in the workspace against the oracle's, and
    sampled outputs (first and last tiles, edge rows and columns, 8192 random) against the
    oracle's exact products of its own quantisation."""
    import mxfp4_quantized_linear_block_b200 as mx
    wl = synth.WORKLOADS["dit_b16"]
    lin = wl.linears[j]
    assert mx.linear_kernel_count(lin.M, lin.N, lin.K, wl.rotation) == 1
    x, wq, ws, A, B = _layer_inputs(wl, lin)
    wsd = mx.new_workspace(mx.workspace_bytes(mx.OP_LINEAR, lin.M, lin.N, lin.K))
    y = _run_linear(x, wq, ws, lin.N, wl.rotation, A, B, workspace=wsd)
    xq, xs = oracle.rotate_quantize(x, wl.rotation)
    # workspace: 256-byte status region, the codes, then the scales at the next 256 bytes
    h = wsd.cpu().numpy()
    M, K = lin.M, lin.K
    sf_off = -(-(256 + M * K // 2) // 256) * 256
    assert np.array_equal(h[256:256 + M * K // 2].reshape(M, K // 2), xq), "codes differ"
    assert np.array_equal(h[sf_off:sf_off + oracle.sf_bytes(M, K)],
                          oracle.sf_to_physical(xs, K)), "scale bytes differ"
    mi, ni = _sample_pairs(lin.M, lin.N, n_random=8192, seed=3 + j)
    ref, S = oracle.gemm_pairs(xq, xs, wq, ws, mi, ni)
    check_gemm_values(y[mi, ni], ref, S, "bf16", f"dit_b16/{lin.name}")


def test_linear_repeatable():
    """Two runs give identical bytes (no races between the paired kernels)."""
    wl = synth.WORKLOADS["dit_b1"]
    lin = wl.linears[0]
    x, wq, ws, A, B = _layer_inputs(wl, lin)
    y1 = _run_linear(x, wq, ws, lin.N, wl.rotation, A, B)
    y2 = _run_linear(x, wq, ws, lin.N, wl.rotation, A, B)
    assert np.array_equal(y1, y2)


def test_status_word_clear_after_runs():
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    wl = synth.WORKLOADS["tiny"]
    lin = wl.linears[0]
    x, wq, ws, A, B = _layer_inputs(wl, lin)
    wsp = mx.new_workspace(mx.workspace_bytes(mx.OP_LINEAR, lin.M, lin.N, lin.K))
    mx.linear(to_dev_bf16(x), to_dev(wq), to_dev(oracle.sf_to_physical(ws, lin.K)), lin.N,
              wl.rotation, ws=wsp)
    torch.cuda.synchronize()
    assert mx.poll_status(wsp) == mx.OK


@pytest.mark.parametrize("mode", [oracle.ROT_HADAMARD64, oracle.ROT_HADAMARD128])
@pytest.mark.parametrize("M", [16, 300])
def test_linear_wide_hadamard(mode, M):
    """The layer with a larger rotation group: weights rotated by the same H_n on the GPU
    (fp32 input), activations online; compared with the oracle's layer."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    K, N = 1024, 768
    x, _ = synth.activation_bf16(M, M, K, 0.01, 30.0)
    w = synth.weight_f32(2, N, K, 5)
    wq_d, wsf_d = mx.rotate_quantize(torch.from_numpy(w).cuda(), mode)
    y = mx.linear(to_dev_bf16(x), wq_d, wsf_d, N, mode)
    torch.cuda.synchronize()
    wq, ws = oracle.prepare_weight(w, mode)
    assert np.array_equal(wq_d.cpu().numpy(), wq)
    ref, S, _, _ = oracle.linear(x, wq, ws, mode)
    check_gemm_values(bf16_dev_to_f64(y), ref, S, "bf16", f"H{oracle.rotation_span(mode)} M{M}")
