"""The layer for more than 128 rows as one kernel: quantiser warps beside the CTA-pair GEMM
rotate and quantise x into the workspace while the other warps multiply, and each CTA's
TMA producer waits per 128-row group for the rows to be published.

Checked against the oracle: the codes and scale bytes the quantiser warps leave in the
workspace, bit for bit (K padding of each real row included), and the output; and
against the two-kernel form of the same layer, byte for byte (the same GEMM on the same
codes). The one-kernel form is forced for small and ragged problems
(mxfp4_set_linear_form); the larger cases take it by size.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import bf16_dev_to_f64, check_gemm_values, to_dev, to_dev_bf16
from test_gpu_gemm import _sample_pairs

pytestmark = pytest.mark.gpu

MODES = [oracle.ROT_NONE, oracle.ROT_HADAMARD32, oracle.ROT_KRON_4x8]


@pytest.fixture
def form():
    """Set the layer's form for one test; the size rule is restored afterwards."""
    import mxfp4_quantized_linear_block_b200 as mx
    yield mx.set_linear_form
    mx.set_linear_form(mx.LINEAR_AUTO)


def _weights(N, K, mode, seed):
    w = synth.weight_f32(seed, N, K, 2)
    A = B = None
    if mode == oracle.ROT_KRON_4x8:
        A, B = synth.kron_factors(seed)
    wq, ws = oracle.prepare_weight(w, mode, A, B)
    return wq, ws, A, B


def _workspace_operand(ws, M, K):
    """The activation codes [M, K/2] and the physical scale bytes the layer left in its
    workspace (status region of 256 bytes, codes, then scales at the next 256 bytes)."""
    import mxfp4_quantized_linear_block_b200 as mx
    sf_off = -(-(256 + M * K // 2) // 256) * 256
    h = ws.cpu().numpy()
    return h[256:256 + M * K // 2].reshape(M, K // 2), h[sf_off:sf_off + mx.sf_bytes(M, K)]


def _check_operand(q, phys, x, mode, A, B, what):
    """Codes and scales bit for bit against the oracle's rotate_quantize, for the real
    rows; the K-padding scale bytes of real rows are 0."""
    M, K = x.shape
    xq, xs = oracle.rotate_quantize(x, mode, A, B)
    assert np.array_equal(q, xq), f"{what}: codes differ in {int((q != xq).sum())} bytes"
    exp = oracle.sf_to_physical(xs, K)
    katoms = -(-K // 128)
    # bytes of real rows: every (row, block) of the 4 * katoms blocks a row's atoms hold
    rows = np.arange(M)
    kbs = np.arange(4 * katoms)
    r, kb = np.meshgrid(rows, kbs, indexing="ij")
    off = ((r // 128) * katoms + kb // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + kb % 4
    got, want = phys[off], exp[off]
    assert np.array_equal(got, want), \
        f"{what}: {int((got != want).sum())} scale bytes of real rows differ"


def _run(x, wq, ws, N, mode, A, B, forms):
    """y of each form (bf16 bits as int16) and the one-kernel form's workspace."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    M, K = x.shape
    xd = to_dev_bf16(x)
    wq_d, wsf_d = to_dev(wq), to_dev(oracle.sf_to_physical(ws, K))
    out = {}
    wsd = None
    for f in forms:
        mx.set_linear_form(f)
        wsd = mx.new_workspace(mx.workspace_bytes(mx.OP_LINEAR, M, N, K))
        wsd[256:] = 0x5A  # junk past the status region: every byte read must be written
        y = mx.linear(xd, wq_d, wsf_d, N, mode, A, B, ws=wsd)
        torch.cuda.synchronize()
        assert mx.poll_status(wsd) == mx.OK
        out[f] = (y, wsd)
    mx.set_linear_form(mx.LINEAR_AUTO)
    return out


# Ragged rows (groups of 128 cut short, a 256-row tile with one live CTA), K with a tail
# inside its last 128 (33 and 35 blocks: scale padding), several work-item sizes.
SHAPES = [(129, 16, 64), (300, 272, 1056), (255, 784, 1120), (1000, 1040, 3072),
          (2560, 2048, 6144)]
CASES = ([(M, N, K, mode) for M, N, K in SHAPES for mode in MODES] +
         [(4100, 528, 12288, oracle.ROT_HADAMARD32)])


@pytest.mark.parametrize("M,N,K,mode", CASES)
def test_one_kernel_layer_codes_and_output(M, N, K, mode, form):
    import mxfp4_quantized_linear_block_b200 as mx
    x, _ = synth.activation_bf16(M + 7 * K, M, K, 0.01, 30.0)
    wq, ws, A, B = _weights(N, K, mode, 3)
    out = _run(x, wq, ws, N, mode, A, B, [mx.LINEAR_ONE_KERNEL, mx.LINEAR_TWO_KERNELS])
    y1, ws1 = out[mx.LINEAR_ONE_KERNEL]
    y2, _ = out[mx.LINEAR_TWO_KERNELS]
    import torch
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), "one kernel != two kernels"
    q, phys = _workspace_operand(ws1, M, K)
    _check_operand(q, phys, x, mode, A, B, f"one-kernel M{M} K{K} mode{mode}")
    y = bf16_dev_to_f64(y1)
    if M * N <= 300_000:
        ref, S, _, _ = oracle.linear(x, wq, ws, mode, A, B)
        check_gemm_values(y, ref, S, "bf16", f"one-kernel layer M{M} N{N} K{K}")
    else:
        xq, xs = oracle.rotate_quantize(x, mode, A, B)
        mi, ni = _sample_pairs(M, N, n_random=4096, seed=M)
        ref, S = oracle.gemm_pairs(xq, xs, wq, ws, mi, ni)
        check_gemm_values(y[mi, ni], ref, S, "bf16", f"one-kernel layer M{M} N{N} K{K}")


def test_size_rule_takes_one_kernel_and_matches_oracle():
    """A problem the size rule gives one kernel (8000 x 2624 -> 5008: 640 tiles of
    256 x 256, 40.04 MiB of x; K = 82 blocks, so scale padding): codes bit for bit,
    output sampled."""
    import mxfp4_quantized_linear_block_b200 as mx
    M, K, N = 8000, 2624, 5008
    assert mx.linear_kernel_count(M, N, K, mx.ROT_HADAMARD32) == 1
    x, _ = synth.activation_bf16(41, M, K, 0.01, 30.0)
    wq, ws, A, B = _weights(N, K, oracle.ROT_HADAMARD32, 4)
    out = _run(x, wq, ws, N, oracle.ROT_HADAMARD32, None, None, [mx.LINEAR_AUTO])
    y, wsd = out[mx.LINEAR_AUTO]
    q, phys = _workspace_operand(wsd, M, K)
    _check_operand(q, phys, x, oracle.ROT_HADAMARD32, None, None, "size-rule layer")
    xq, xs = oracle.rotate_quantize(x, oracle.ROT_HADAMARD32)
    mi, ni = _sample_pairs(M, N, n_random=4096, seed=5)
    ref, S = oracle.gemm_pairs(xq, xs, wq, ws, mi, ni)
    check_gemm_values(bf16_dev_to_f64(y)[mi, ni], ref, S, "bf16", "size-rule layer")


def test_one_workspace_across_shapes_and_forms(form):
    """One workspace serves one-kernel calls of different sizes in a row (each call clears
    its own row counters), interleaved with two-kernel calls; every result equals a call
    on a fresh workspace."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    shapes = [(2560, 2048, 6144), (300, 272, 1056), (1000, 1040, 3072), (300, 272, 1056)]
    ws = mx.new_workspace(max(mx.workspace_bytes(mx.OP_LINEAR, M, N, K) for M, N, K in shapes))
    for i, (M, N, K) in enumerate(shapes * 2):
        x, _ = synth.activation_bf16(100 + i, M, K, 0.01, 30.0)
        wq, wsc, _, _ = _weights(N, K, oracle.ROT_HADAMARD32, 7)
        xd = to_dev_bf16(x)
        wq_d, wsf_d = to_dev(wq), to_dev(oracle.sf_to_physical(wsc, K))
        form(mx.LINEAR_ONE_KERNEL if i % 3 != 2 else mx.LINEAR_TWO_KERNELS)
        y = mx.linear(xd, wq_d, wsf_d, N, mx.ROT_HADAMARD32, ws=ws)
        form(mx.LINEAR_TWO_KERNELS)
        y_ref = mx.linear(xd, wq_d, wsf_d, N, mx.ROT_HADAMARD32)
        torch.cuda.synchronize()
        assert mx.poll_status(ws) == mx.OK
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), f"call {i} {M}x{K}"


def test_noalloc_one_kernel_matches_linear(form):
    """The allocation-free layer takes the same one-kernel form (its row counters follow
    the scales in the library's array) with the same bytes as mxfp4_linear."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    for M, N, K in [(3000, 1040, 2048), (129, 16, 64), (2560, 2048, 6144)]:
        x, _ = synth.activation_bf16(M, M, K, 0.01, 30.0)
        wq, wsc, _, _ = _weights(N, K, oracle.ROT_HADAMARD32, 8)
        xd = to_dev_bf16(x)
        wq_d, wsf_d = to_dev(wq), to_dev(oracle.sf_to_physical(wsc, K))
        form(mx.LINEAR_ONE_KERNEL)
        status = torch.zeros(4, dtype=torch.int32, device="cuda")
        y = mx.linear_noalloc(xd, wq_d, wsf_d, N, mx.ROT_HADAMARD32, status=status)
        y2 = mx.linear(xd, wq_d, wsf_d, N, mx.ROT_HADAMARD32)
        torch.cuda.synchronize()
        assert int(status[0]) == 0
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16)), f"noalloc {M}x{K}"
