"""mxfp4_linear_noalloc -- the layer for callers that cannot allocate device memory
at call time (a fixed start-up memory plan, a plugin inside another framework's
enqueue step, latency-critical code avoiding cudaMalloc's implicit synchronisation).
Its scratch is a fixed array inside the library; the output must match the
workspace-taking entry point, call after call, whatever the previous call left in
the shared array.

This file is collected last on purpose, so a run that stops at the first failure
has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import bf16_dev_to_f64, bf16_ulp, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


def _problem(seed, M, K, N, mode):
    x, _ = synth.activation_bf16(seed, M, K, 0.01, 30.0)
    w = synth.weight_f32(seed, N, K, layer=seed)
    A = B = None
    if mode == oracle.ROT_KRON_4x8:
        A, B = synth.kron_factors(seed)
        wq, ws = oracle.prepare_weight(w, mode, A, B)
    else:
        wq, ws = oracle.prepare_weight(w, mode)
    return x, wq, oracle.sf_to_physical(ws, K), A, B


def _call_noalloc(mx, xd, wqd, wsfd, M, K, N, yd, status, mode, A=None, B=None):
    import torch
    a = np.ascontiguousarray(A, np.float32) if A is not None else None
    b = np.ascontiguousarray(B, np.float32) if B is not None else None
    return mx.lib.mxfp4_linear_noalloc(
        xd.data_ptr(), M, K, mode, a.ctypes.data if a is not None else None,
        b.ctypes.data if b is not None else None, wqd.data_ptr(), wsfd.data_ptr(), N,
        yd.data_ptr(), status.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _same_within_tolerance(y_na, y_ref, what):
    a, b = bf16_dev_to_f64(y_na), bf16_dev_to_f64(y_ref)
    assert np.all(np.abs(a - b) <= bf16_ulp(b)), f"{what}: outputs differ"


# (seed, (M, K, N), mode, what the shape exercises)
CASES = [
    (1, (4096, 8192, 2048), oracle.ROT_HADAMARD32, "pair GEMM, 16 MiB of codes"),
    (2, (2560, 6144, 2048), oracle.ROT_HADAMARD32, "pair GEMM, last round split along K"),
    (3, (4, 2048, 1024), oracle.ROT_HADAMARD32, "one-kernel layer (1..8 rows)"),
    (4, (100, 7168, 1024), oracle.ROT_HADAMARD32, "few-row GEMM, K splits summed through L2"),
    (5, (300, 1024, 512), oracle.ROT_KRON_4x8, "Kronecker rotation"),
    (6, (129, 512, 256), oracle.ROT_NONE, "no rotation, one row past a tile"),
]


def test_noalloc_matches_linear_on_two_calls_in_a_row():
    """Each case is run twice in a row, after the previous (often larger) case, and
    compared with mxfp4_linear on a fresh workspace."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for seed, (M, K, N), mode, what in CASES:
        x, wq, wsf, A, B = _problem(seed, M, K, N, mode)
        xd, wqd, wsfd = to_dev_bf16(x), to_dev(wq), to_dev(wsf)
        y_ref = mx.linear(xd, wqd, wsfd, N, mode, A, B)
        for call in range(2):
            y_na = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
            assert _call_noalloc(mx, xd, wqd, wsfd, M, K, N, y_na, status, mode, A, B) == mx.OK
            torch.cuda.synchronize()
            _same_within_tolerance(y_na, y_ref, f"{what}, call {call + 1}")
            assert int(status.item()) == mx.OK


def test_noalloc_call_after_a_timeout_needs_no_reset():
    """A call whose accumulator wait ran out (the library's test hook) leaves the timeout
    in the caller's status word and part of Y unwritten; the next calls on the shared
    array need no reset and are right."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx

    M, K, N = 2560, 6144, 2048
    x, wq, wsf, _, _ = _problem(2, M, K, N, oracle.ROT_HADAMARD32)
    xd, wqd, wsfd = to_dev_bf16(x), to_dev(wq), to_dev(wsf)
    y_ref = mx.linear(xd, wqd, wsfd, N, mx.ROT_HADAMARD32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y_na = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    mx.test_set_fault(mx.TEST_FAULT_WITHHOLD_ACCUMULATOR)
    try:
        st = _call_noalloc(mx, xd, wqd, wsfd, M, K, N, y_na, status, mx.ROT_HADAMARD32)
    finally:
        mx.test_set_fault(mx.TEST_FAULT_NONE)
    assert st == mx.OK
    torch.cuda.synchronize()
    assert int(status.item()) == mx.ERR_TIMEOUT
    status.zero_()
    for call in range(2):
        assert _call_noalloc(mx, xd, wqd, wsfd, M, K, N, y_na, status,
                             mx.ROT_HADAMARD32) == mx.OK
        torch.cuda.synchronize()
        assert int(status.item()) == mx.OK
        _same_within_tolerance(y_na, y_ref, f"call {call + 1} after a timeout")


def test_noalloc_rejects_what_linear_rejects():
    import torch
    import mxfp4_quantized_linear_block_b200 as mx

    fake = torch.empty(16, dtype=torch.uint8, device="cuda")
    P = fake.data_ptr()
    # 8192 x 8192 activations need 32 MiB of codes alone: over the fixed capacity
    st = mx.lib.mxfp4_linear_noalloc(P, 8192, 8192, mx.ROT_HADAMARD32, None, None, P, P, 256,
                                     P, None, ctypes.c_void_p(0))
    assert st == mx.ERR_WORKSPACE
    # weights beyond the kernels' index range are rejected as by mxfp4_linear
    for args in ((P, 4, 1 << 21, mx.ROT_HADAMARD32, None, None, P, P, 65536, P),
                 (P, 4, 96, mx.ROT_HADAMARD64, None, None, P, P, 256, P),
                 (P, 4, 256, mx.ROT_KRON_4x8, None, None, P, P, 256, P)):
        st = mx.lib.mxfp4_linear_noalloc(*args, None, ctypes.c_void_p(0))
        ws = mx.lib.mxfp4_linear(*args, P, 1 << 40, ctypes.c_void_p(0))
        assert st == ws != mx.OK
