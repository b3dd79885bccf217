"""One workspace serving layer calls of different sizes.

Every part of a layer workspace past its status region is written before it is read, so
what an earlier call with other sizes left there never reaches a later call. The sequence
below checks that: a large call fills the workspace with codes and scales, then a call
whose last round runs in column halves (2560 x 6144 -> 2048: 80 tiles of 256 x 256 on 74
CTA pairs, the last 6 tiles as twelve 256 x 128 units) runs on the same workspace, and
both again. Its outputs, the tiles of the last round included, are checked against the
oracle's exact products, and repeated calls give the same bits.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import bf16_dev_to_f64, check_gemm_values, to_dev, to_dev_bf16
from test_gpu_gemm import _sample_pairs

pytestmark = pytest.mark.gpu

LARGE = (4096, 8192, 2048)  # M, K, N: 128 tiles: a full round, then 54 whole tiles
SPLIT = (2560, 6144, 2048)  # 80 tiles: the last 6 (rows 2304.., columns 512..) in halves


def _problem(seed, M, K, N):
    x, _ = synth.activation_bf16(seed, M, K, 0.01, 30.0)
    w = synth.weight_f32(seed, N, K, layer=seed)
    wq, ws = oracle.prepare_weight(w, oracle.ROT_HADAMARD32)
    return x, wq, ws


def _split_tile_pairs(M, N, seed):
    """Every (m, n) of 64 random columns of the last round's tiles (the last row tile of
    256, columns 512..N-1), plus the usual edge and random samples."""
    rng = np.random.default_rng(seed)
    rows = np.arange(M - 256, M)
    cols = rng.choice(np.arange(512, N), 64, replace=False)
    mi, ni = _sample_pairs(M, N, n_random=4096, seed=seed)
    return (np.r_[mi, np.repeat(rows, cols.size)].astype(np.int64),
            np.r_[ni, np.tile(cols, rows.size)].astype(np.int64))


def _check(y, x, wq, ws, what, seed):
    M, N = y.shape
    xq, xs = oracle.rotate_quantize(x, oracle.ROT_HADAMARD32)
    mi, ni = _split_tile_pairs(M, N, seed)
    ref, S = oracle.gemm_pairs(xq, xs, wq, ws, mi, ni)
    check_gemm_values(y[mi, ni], ref, S, "bf16", what)


def test_workspace_sizes_of_the_two_calls():
    """The layer workspace is the status region, the codes, the scales and the row
    counters of the one-launch layer (no GEMM scratch for more than 128 rows)."""
    import mxfp4_quantized_linear_block_b200 as mx
    for M, K, N in (LARGE, SPLIT):
        assert mx.workspace_bytes(mx.OP_GEMM, M, N, K) == 256
        assert mx.workspace_bytes(mx.OP_LINEAR, M, N, K) == (
            256 + M * K // 2 + mx.sf_bytes(M, K) + -(-4 * (-(-M // 128) + 1) // 256) * 256)


def test_linear_workspace_large_then_split_call():
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    ws = mx.new_workspace(max(mx.workspace_bytes(mx.OP_LINEAR, M, N, K) for M, K, N in
                              (LARGE, SPLIT)))
    results = []
    for rep in range(2):
        for seed, (M, K, N) in ((41, LARGE), (42, SPLIT)):
            x, wq, wsc = _problem(seed, M, K, N)
            y = mx.linear(to_dev_bf16(x), to_dev(wq), to_dev(oracle.sf_to_physical(wsc, K)), N,
                          mx.ROT_HADAMARD32, ws=ws)
            torch.cuda.synchronize()
            assert mx.poll_status(ws) == mx.OK
            got = bf16_dev_to_f64(y)
            if rep == 0:
                _check(got, x, wq, wsc, f"linear {M}x{K}->{N} after a larger call", seed)
            results.append(got)
    # the same calls again on the same workspace give the same bits
    assert np.array_equal(results[0], results[2])
    assert np.array_equal(results[1], results[3])
