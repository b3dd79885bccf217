"""A bounded device wait that runs out: the kernel records MXFP4_ERR_TIMEOUT in the
status word and returns; nothing faults or hangs.

The library's test hook (mxfp4_test_set_fault) makes the first CTA pair of the CTA-pair
GEMM never signal that its first accumulator is complete, and shortens its epilogue's
wait for that signal to 1 ms. That wait then expires on purpose: the epilogue records the
timeout and stops, the pair's MMA and copy roles see the stop at their next bounded wait,
drain, release tensor memory and return. The test checks that the call returns, that the
status word reads MXFP4_ERR_TIMEOUT, that the other pairs' tiles are right, and that the
next call is right.
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import check_gemm_values, to_dev
from test_gpu_gemm import _operand, _sample_pairs

pytestmark = pytest.mark.gpu

# 10 x 8 = 80 tiles on 74 pairs: pair 0 owns tile 0 (rows 0..255, columns 0..255) and the
# first column-half unit of the last round; the test hook stops it at tile 0.
M, K, N = 2560, 6144, 2048


def test_accumulator_wait_expires_reports_timeout_and_returns():
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    aq, as_ = _operand(77, M, K, 30)
    bq, bs = _operand(77, N, K, 31)
    args = (to_dev(aq), to_dev(oracle.sf_to_physical(as_, K)), to_dev(bq),
            to_dev(oracle.sf_to_physical(bs, K)), M, N, K)
    ws = mx.new_workspace(mx.workspace_bytes(mx.OP_GEMM, M, N, K))
    mx.test_set_fault(mx.TEST_FAULT_WITHHOLD_ACCUMULATOR)
    try:
        y_bad = mx.gemm(*args, out_dtype=torch.float32, ws=ws)
    finally:
        mx.test_set_fault(mx.TEST_FAULT_NONE)
    torch.cuda.synchronize()  # the kernel returned
    assert mx.poll_status(ws) == mx.ERR_TIMEOUT
    assert mx.poll_status(ws) == mx.OK  # polling clears the word
    # the other pairs' tiles are right: rows 0..255 against columns 256.. (tiles 1..7)
    rows = np.arange(256)
    cols = np.arange(256, N, 29)
    mi, ni = np.repeat(rows, cols.size), np.tile(cols, rows.size)
    ref, S = oracle.gemm_pairs(aq, as_, bq, bs, mi, ni)
    # (only these elements are converted: pair 0's tile holds whatever was in memory)
    check_gemm_values(y_bad.cpu().numpy()[mi, ni].astype(np.float64), ref, S, "f32",
                      "tiles of the pairs that were not stopped")
    # the next call on the same workspace is right, tile 0 and the last round included
    y = mx.gemm(*args, out_dtype=torch.float32, ws=ws)
    torch.cuda.synchronize()
    assert mx.poll_status(ws) == mx.OK
    mi, ni = _sample_pairs(M, N, n_random=4096, seed=5)
    ref, S = oracle.gemm_pairs(aq, as_, bq, bs, mi, ni)
    check_gemm_values(y.cpu().numpy().astype(np.float64)[mi, ni], ref, S, "f32",
                      "after a timeout, on the same workspace")


def test_one_kernel_layer_wait_expires_reports_timeout_and_returns():
    """The same expired wait inside the one-kernel layer (quantiser warps beside the GEMM,
    forced at this size): the quantiser warps finish their rows beside the stopped pair,
    the call returns with MXFP4_ERR_TIMEOUT in the status word, every other pair's tiles
    are right, and the next call on the same workspace is right."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    import synth
    from gpu_helpers import bf16_dev_to_f64, to_dev_bf16
    x, _ = synth.activation_bf16(78, M, K, 0.01, 30.0)
    bq, bs = _operand(78, N, K, 32)
    xd, wq, wsf = to_dev_bf16(x), to_dev(bq), to_dev(oracle.sf_to_physical(bs, K))
    ws = mx.new_workspace(mx.workspace_bytes(mx.OP_LINEAR, M, N, K))
    xq, xs = oracle.rotate_quantize(x, oracle.ROT_HADAMARD32)
    mx.set_linear_form(mx.LINEAR_ONE_KERNEL)
    try:
        mx.test_set_fault(mx.TEST_FAULT_WITHHOLD_ACCUMULATOR)
        try:
            y_bad = mx.linear(xd, wq, wsf, N, mx.ROT_HADAMARD32, ws=ws)
        finally:
            mx.test_set_fault(mx.TEST_FAULT_NONE)
        torch.cuda.synchronize()  # the kernel returned
        assert mx.poll_status(ws) == mx.ERR_TIMEOUT
        assert mx.poll_status(ws) == mx.OK
        rows = np.arange(256)
        cols = np.arange(256, N, 29)
        mi, ni = np.repeat(rows, cols.size), np.tile(cols, rows.size)
        ref, S = oracle.gemm_pairs(xq, xs, bq, bs, mi, ni)
        # (only these elements are converted: pair 0's tile holds whatever was in memory)
        sel = y_bad[torch.as_tensor(mi, device=y_bad.device), torch.as_tensor(ni, device=y_bad.device)]
        check_gemm_values(bf16_dev_to_f64(sel), ref, S, "bf16",
                          "one-kernel layer: tiles of the pairs that were not stopped")
        y = mx.linear(xd, wq, wsf, N, mx.ROT_HADAMARD32, ws=ws)
        torch.cuda.synchronize()
        assert mx.poll_status(ws) == mx.OK
    finally:
        mx.set_linear_form(mx.LINEAR_AUTO)
    mi, ni = _sample_pairs(M, N, n_random=4096, seed=6)
    ref, S = oracle.gemm_pairs(xq, xs, bq, bs, mi, ni)
    check_gemm_values(bf16_dev_to_f64(y)[mi, ni], ref, S, "bf16",
                      "one-kernel layer after a timeout, on the same workspace")
