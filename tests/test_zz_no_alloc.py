"""mxfp4_linear_noalloc -- the layer for callers that cannot allocate device
memory at call time (a fixed start-up memory plan, a plugin inside another
framework's enqueue step, latency-critical code avoiding cudaMalloc's implicit
synchronisation). Its scratch is a fixed array inside the library; the output
must match the workspace-taking entry point, call after call.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import bf16_dev_to_f64, bf16_ulp, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


def _problem(seed, M, K, N):
    x, _ = synth.activation_bf16(seed, M, K, 0.01, 30.0)
    w = synth.weight_f32(seed, N, K, layer=seed)
    wq, ws = oracle.prepare_weight(w, oracle.ROT_HADAMARD32)
    return x, wq, oracle.sf_to_physical(ws, K)


def _call_noalloc(mx, xd, wqd, wsfd, M, K, N, yd, status):
    torch = pytest.importorskip("torch")
    return mx.lib.mxfp4_linear_noalloc(
        xd.data_ptr(), M, K, mx.ROT_HADAMARD32, None, None, wqd.data_ptr(), wsfd.data_ptr(), N,
        yd.data_ptr(), status.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_linear_on_two_calls_in_a_row():
    import torch
    import mxfp4_quantized_linear_block_b200 as mx

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # a larger problem first, then a smaller one: the second call must not see the
    # first call's leftovers in the shared array
    for seed, (M, K, N) in ((1, (1000, 3072, 1024)), (2, (129, 512, 256))):
        x, wq, wsf = _problem(seed, M, K, N)
        xd, wqd, wsfd = to_dev_bf16(x), to_dev(wq), to_dev(wsf)
        y_ref = mx.linear(xd, wqd, wsfd, N, mx.ROT_HADAMARD32)
        y_na = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(mx, xd, wqd, wsfd, M, K, N, y_na, status) == mx.OK
        torch.cuda.synchronize()
        a, b = bf16_dev_to_f64(y_na), bf16_dev_to_f64(y_ref)
        assert np.all(np.abs(a - b) <= bf16_ulp(b)), f"call {seed}: outputs differ"
        assert int(status.item()) == mx.OK


def test_noalloc_rejects_problems_beyond_its_scratch():
    import torch
    import mxfp4_quantized_linear_block_b200 as mx

    # 8192 x 8192 activations need 32 MiB of codes alone: over the fixed capacity
    M = K = 8192
    fake = torch.empty(16, dtype=torch.uint8, device="cuda")
    st = mx.lib.mxfp4_linear_noalloc(fake.data_ptr(), M, K, mx.ROT_HADAMARD32, None, None,
                                     fake.data_ptr(), fake.data_ptr(), 256, fake.data_ptr(),
                                     None, ctypes.c_void_p(0))
    assert st == mx.ERR_WORKSPACE
