"""A bounded device wait that runs out: the kernel records MXFP4_ERR_TIMEOUT in the
status word and returns; nothing faults or hangs.

The library's test hook (mxfp4_test_set_fault) makes chunk 1 of every K-split tile of
the CTA-pair GEMM store its partial without publishing it, and shortens the owning
chunk's wait for it to 1 ms. That wait then expires on purpose: the owner records the
timeout and finishes its tile without waiting any longer (what it reads of that partial
then depends on timing, so those tiles are not checked). The test checks that the call
returns, that the status word reads MXFP4_ERR_TIMEOUT, and that the next call on the
re-zeroed workspace is right.
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import check_gemm_values, to_dev
from test_gpu_gemm import _operand
from test_gpu_workspace_reuse import SPLIT, _split_tile_pairs

pytestmark = pytest.mark.gpu


def test_split_wait_expires_reports_timeout_and_returns():
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    M, K, N = SPLIT
    aq, as_ = _operand(77, M, K, 30)
    bq, bs = _operand(77, N, K, 31)
    args = (to_dev(aq), to_dev(oracle.sf_to_physical(as_, K)), to_dev(bq),
            to_dev(oracle.sf_to_physical(bs, K)), M, N, K)
    ws = mx.new_workspace(mx.workspace_bytes(mx.OP_GEMM, M, N, K))
    mx.test_set_fault(mx.TEST_FAULT_SKIP_SPLIT_PUBLISH)
    try:
        y_bad = mx.gemm(*args, out_dtype=torch.float32, ws=ws)
    finally:
        mx.test_set_fault(mx.TEST_FAULT_NONE)
    torch.cuda.synchronize()  # the kernel returned
    assert mx.poll_status(ws) == mx.ERR_TIMEOUT
    assert mx.poll_status(ws) == mx.OK  # polling clears the word
    # tiles outside the split last round were not affected: rows 0..255 are whole tiles
    rows = np.arange(256)
    cols = np.arange(0, N, 37)
    mi, ni = np.repeat(rows, cols.size), np.tile(cols, rows.size)
    ref, S = oracle.gemm_pairs(aq, as_, bq, bs, mi, ni)
    check_gemm_values(y_bad.cpu().numpy().astype(np.float64)[mi, ni], ref, S, "f32",
                      "whole tiles next to a timed-out split tile")
    # the next call on the re-zeroed workspace is right, split tiles included
    ws.zero_()
    y = mx.gemm(*args, out_dtype=torch.float32, ws=ws)
    torch.cuda.synchronize()
    assert mx.poll_status(ws) == mx.OK
    mi, ni = _split_tile_pairs(M, N, seed=5)
    ref, S = oracle.gemm_pairs(aq, as_, bq, bs, mi, ni)
    check_gemm_values(y.cpu().numpy().astype(np.float64)[mi, ni], ref, S, "f32",
                      "after a timeout, on a re-zeroed workspace")
