"""The C-ABI library on a machine without a GPU: it loads, exports every symbol
the header declares, its host helpers agree with the oracle's own layout map,
and argument errors are reported before anything is launched."""
import os
import re

import numpy as np
import pytest

import oracle
import mxfp4_quantized_linear_block_b200 as mx

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "mxfp4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mxfp4_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(mx.lib, n), n
    assert set(names) == set(mx.EXPORTS)


def test_sf_layout_matches_oracle_map():
    for rows, K in ((1, 32), (127, 96), (300, 640), (3584, 3072), (16, 14336)):
        assert mx.sf_bytes(rows, K) == oracle.sf_bytes(rows, K)
        rng = np.random.default_rng(rows + K)
        for r, b in zip(rng.integers(0, rows, 200), rng.integers(0, K // 32, 200)):
            assert mx.sf_offset(int(r), int(b), K) == oracle.sf_offset(int(r), int(b), K)
    assert mx.sf_offset(0, 3, 64) == -1          # block beyond K
    assert mx.sf_bytes(10, 33) == 0


def test_status_strings():
    for s in range(8):
        assert isinstance(mx.status_string(s), str) and mx.status_string(s)
    assert mx.status_string(99) == "unknown status"


def test_workspace_sizes():
    assert mx.workspace_bytes(mx.OP_QUANTIZE, 10, 16, 64) == 0
    assert mx.workspace_bytes(mx.OP_GEMM, 10, 16, 64) == 256
    M, K = 3584, 3072
    ws = mx.workspace_bytes(mx.OP_LINEAR, M, 9216, K)
    # status, codes, scales, and the one-launch layer's row counters (4 bytes per 128 rows)
    assert ws == 256 + M * K // 2 + mx.sf_bytes(M, K) + 256


# Fake device addresses: validation rejects these calls on the host, so nothing is dereferenced.
P = 1 << 20


def test_quantize_argument_errors():
    L = mx.lib
    assert L.mxfp4_rotate_quantize(None, 0, 4, 64, 64, 1, None, None, P, P, None) == mx.ERR_INVALID_ARG
    assert L.mxfp4_rotate_quantize(P, 0, 4, 64, 64, 1, None, None, None, P, None) == mx.ERR_INVALID_ARG
    assert L.mxfp4_rotate_quantize(P, 0, 4, 48, 64, 1, None, None, P, P, None) == mx.ERR_SHAPE
    assert L.mxfp4_rotate_quantize(P, 0, 4, 64, 32, 1, None, None, P, P, None) == mx.ERR_SHAPE
    assert L.mxfp4_rotate_quantize(P, 0, -1, 64, 64, 1, None, None, P, P, None) == mx.ERR_SHAPE
    assert L.mxfp4_rotate_quantize(P + 8, 0, 4, 64, 64, 1, None, None, P, P, None) == mx.ERR_ALIGN
    assert L.mxfp4_rotate_quantize(P, 0, 4, 64, 68, 1, None, None, P, P, None) == mx.ERR_ALIGN
    assert L.mxfp4_rotate_quantize(P, 2, 4, 64, 64, 1, None, None, P, P, None) == mx.ERR_UNSUPPORTED
    assert L.mxfp4_rotate_quantize(P, 0, 4, 64, 64, 7, None, None, P, P, None) == mx.ERR_UNSUPPORTED
    # Kronecker mode needs both host factors
    assert L.mxfp4_rotate_quantize(P, 0, 4, 64, 64, 2, None, None, P, P, None) == mx.ERR_INVALID_ARG
    # empty input: valid, launches nothing
    assert L.mxfp4_rotate_quantize(P, 0, 0, 64, 64, 1, None, None, P, P, None) == mx.OK
    assert L.mxfp4_quantize(P, 1, 0, 64, 64, P, P, None) == mx.OK


def test_gemm_argument_errors():
    L = mx.lib
    ok = dict(aq=P, asf=P, bq=P, bsf=P, M=4, N=16, K=64, y=P, ydt=0, ldy=16, ws=P, wsb=256)

    def call(**kw):
        a = {**ok, **kw}
        return L.mxfp4_gemm(a["aq"], a["asf"], a["bq"], a["bsf"], a["M"], a["N"], a["K"], a["y"],
                            a["ydt"], a["ldy"], a["ws"], a["wsb"], None)

    assert call(aq=None) == mx.ERR_INVALID_ARG
    assert call(ws=None) == mx.ERR_INVALID_ARG
    assert call(N=24) == mx.ERR_SHAPE
    assert call(K=48) == mx.ERR_SHAPE
    assert call(ldy=8) == mx.ERR_SHAPE
    assert call(y=P + 4) == mx.ERR_ALIGN
    assert call(ldy=20) == mx.ERR_ALIGN
    assert call(ydt=5) == mx.ERR_UNSUPPORTED
    assert call(wsb=16) == mx.ERR_WORKSPACE
    assert call(M=0) == mx.OK


def test_linear_argument_errors():
    L = mx.lib
    need = mx.workspace_bytes(mx.OP_LINEAR, 8, 32, 64)
    assert L.mxfp4_linear(P, 8, 64, 1, None, None, P, P, 32, P, P, need - 1, None) == mx.ERR_WORKSPACE
    assert L.mxfp4_linear(P, 8, 64, 1, None, None, P, P, 24, P, P, need, None) == mx.ERR_SHAPE
    assert L.mxfp4_linear(P, 8, 64, 9, None, None, P, P, 32, P, P, need, None) == mx.ERR_UNSUPPORTED
    assert L.mxfp4_linear(P, 8, 64, 2, None, None, P, P, 32, P, P, need, None) == mx.ERR_INVALID_ARG
    assert L.mxfp4_linear(None, 8, 64, 1, None, None, P, P, 32, P, P, need, None) == mx.ERR_INVALID_ARG
    assert L.mxfp4_linear(P, 0, 64, 1, None, None, P, P, 32, P, P, need, None) == mx.OK


def test_poll_status_null():
    import ctypes
    out = ctypes.c_int(0)
    assert mx.lib.mxfp4_poll_status(None, ctypes.byref(out)) == mx.ERR_INVALID_ARG


def test_gemm_bias_and_quantize_argument_errors():
    L = mx.lib
    assert L.mxfp4_gemm_bias(P, P, P, P, 4, 16, 64, None, P, 0, 16, P, 256, None) == \
        mx.ERR_INVALID_ARG  # bias is required
    assert L.mxfp4_gemm_bias(P, P, P, P, 4, 16, 64, P + 4, P, 0, 16, P, 256, None) == mx.ERR_ALIGN
    assert L.mxfp4_gemm_bias(P, P, P, P, 4, 24, 64, P, P, 0, 24, P, 256, None) == mx.ERR_SHAPE
    assert L.mxfp4_gemm_bias(P, P, P, P, 0, 16, 64, P, P, 0, 16, P, 256, None) == mx.OK
    ok = dict(M=4, N=64, K=64, bias=None, mode=1, a=None, b=None, yq=P, ysf=P, ws=P, wsb=256)

    def q(**kw):
        a = {**ok, **kw}
        return L.mxfp4_gemm_quantize(P, P, P, P, a["M"], a["N"], a["K"], a["bias"], a["mode"],
                                     a["a"], a["b"], a["yq"], a["ysf"], a["ws"], a["wsb"], None)

    assert q(yq=None) == mx.ERR_INVALID_ARG
    assert q(ysf=None) == mx.ERR_INVALID_ARG
    assert q(N=48) == mx.ERR_SHAPE            # N % 32 != 0 (the output's 32-blocks)
    assert q(mode=7) == mx.ERR_UNSUPPORTED
    assert q(mode=2) == mx.ERR_INVALID_ARG    # Kronecker needs both factors
    assert q(bias=P + 8) == mx.ERR_ALIGN
    assert q(ysf=P + 1) == mx.ERR_ALIGN
    assert q(wsb=16) == mx.ERR_WORKSPACE
    assert q(M=0) == mx.OK


def test_empty_calls_accept_null_row_operands():
    """With no rows, x / the activation codes and scales / y may be NULL (frameworks hand out
    NULL for empty tensors); the weight operands and the workspace stay required."""
    L = mx.lib
    assert L.mxfp4_rotate_quantize(None, 0, 0, 64, 64, 1, None, None, None, None, None) == mx.OK
    assert L.mxfp4_gemm(None, None, P, P, 0, 16, 64, None, 0, 16, P, 256, None) == mx.OK
    assert L.mxfp4_gemm(None, None, None, P, 0, 16, 64, None, 0, 16, P, 256, None) == \
        mx.ERR_INVALID_ARG
    assert L.mxfp4_gemm(None, P, P, P, 4, 16, 64, P, 0, 16, P, 256, None) == mx.ERR_INVALID_ARG
    need = mx.workspace_bytes(mx.OP_LINEAR, 0, 32, 64)
    assert L.mxfp4_linear(None, 0, 64, 1, None, None, P, P, 32, None, P, need, None) == mx.OK
    assert L.mxfp4_linear(None, 0, 64, 1, None, None, P, P, 32, None, None, need, None) == \
        mx.ERR_INVALID_ARG
    assert L.mxfp4_linear(P, 4, 64, 1, None, None, P, P, 32, None, P, 1 << 20, None) == \
        mx.ERR_INVALID_ARG
    assert L.mxfp4_linear_noalloc(None, 0, 64, 1, None, None, P, P, 32, None, None, None) == mx.OK


def test_linear_kernel_count():
    """One kernel for 1..8 rows with rotation 0/1/2 and short K splits, and for large
    problems (8 rounds of 256 x 256 tiles on 74 CTA pairs, x of 40 MiB or more); two
    otherwise."""
    kc = mx.linear_kernel_count
    assert kc(57344, 12288, 3072, mx.ROT_HADAMARD32) == 1   # 10752 tiles, 336 MiB of x
    assert kc(57344, 3072, 12288, mx.ROT_KRON_4x8) == 1
    assert kc(7168, 12288, 3072, mx.ROT_NONE) == 1          # 1344 tiles, 42 MiB
    assert kc(7168, 3072, 12288, mx.ROT_HADAMARD32) == 2    # 336 tiles: under 8 rounds
    assert kc(3584, 12288, 3072, mx.ROT_HADAMARD32) == 2    # 21 MiB of x
    assert kc(57344, 3072, 12288, mx.ROT_HADAMARD64) == 2   # wide groups: two kernels
    assert kc(1, 14336, 4096, mx.ROT_HADAMARD32) == 1
    assert kc(8, 4096, 14336, mx.ROT_KRON_4x8) == 1
    assert kc(4, 128, 256, mx.ROT_NONE) == 1
    assert kc(9, 4096, 14336, mx.ROT_HADAMARD32) == 2
    assert kc(128, 4096, 14336, mx.ROT_HADAMARD32) == 2
    assert kc(1, 4096, 4096, mx.ROT_HADAMARD64) == 2
    assert kc(5, 150 * 128, 3584, mx.ROT_HADAMARD32) == 2  # one split of 14 k-tiles
    assert kc(0, 128, 256, mx.ROT_HADAMARD32) == 0
    assert kc(1, 128, 48, mx.ROT_HADAMARD32) == -1
    assert kc(1, 24, 256, mx.ROT_HADAMARD32) == -1
    assert kc(1, 128, 256, 9) == -1


def test_norm_linear_kernel_count():
    """The norm prologue is one kernel while two row buffers fit one SM (K <= 51168)."""
    kc = mx.norm_linear_kernel_count
    assert kc(3584, 9216, 3072, mx.ROT_HADAMARD32) == 2
    assert kc(3584, 3072, 12288, mx.ROT_HADAMARD32) == 2
    assert kc(3, 256, 51168, mx.ROT_KRON_4x8) == 2
    assert kc(3, 256, 51200, mx.ROT_HADAMARD32) == 3
    assert kc(0, 256, 1024, mx.ROT_NONE) == 0
    assert kc(4, 256, 1024, mx.ROT_HADAMARD64) == -1
    assert kc(4, 24, 1024, mx.ROT_HADAMARD32) == -1


def test_gemm_scratch_for_few_rows():
    """Every workspace starts with the 256-byte status region. The few-row GEMM's K-split
    partials follow it for 33..128 rows split 4 or more ways: units x rows x 128 columns
    x 4 bytes; fewer splits or rows need nothing past the head."""
    def gemm_ws(M, N, K):
        return mx.workspace_bytes(mx.OP_GEMM, M, N, K)
    # 4096 -> 14336 weights transposed, 128 rows (one CTA per SM): 32 W tiles x 4 splits
    # = 128 units
    assert gemm_ws(128, 4096, 14336) == 256 + 128 * 128 * 128 * 4
    # 100 rows, 8 W tiles x 7 splits (28 k-tiles in splits of 4)
    assert gemm_ws(100, 1024, 7168) == 256 + 56 * 100 * 128 * 4
    assert gemm_ws(128, 14336, 4096) == 256  # 112 W tiles, one split: no sum
    assert gemm_ws(32, 4096, 14336) == 256   # 32 rows: on-chip sum
    assert gemm_ws(1, 14336, 4096) == 256


def test_pair_gemm_needs_no_scratch():
    """The CTA-pair GEMM (more than 128 rows) exchanges nothing between pairs, whatever
    its last round looks like: its workspace is the status region alone, and the layer's
    adds the activation codes and scales, one row counter per 128-row group of them and
    the one-kernel form's work-item counter."""
    r256 = lambda v: -(-v // 256) * 256
    for M, N, K in [(2560, 2048, 6144), (4096, 2048, 8192), (57344, 12288, 3072),
                    (3584, 3072, 3072), (129, 16, 64)]:
        assert mx.workspace_bytes(mx.OP_GEMM, M, N, K) == 256
        assert mx.workspace_bytes(mx.OP_LINEAR, M, N, K) == (
            256 + r256(M * K // 2) + r256(mx.sf_bytes(M, K)) + r256(4 * (-(-M // 128) + 1)))


def test_kron_weight_factors_match_oracle():
    """mxfp4_kron_weight_factors (the library's own double Gauss-Jordan) against the
    oracle's: within 1 fp32 ulp everywhere, and identical on the seeded workload factors,
    so weights prepared through the library and through the oracle are the same bytes."""
    import synth
    for seed in range(12):
        A, B = synth.kron_factors(seed)
        At, Bt = mx.kron_weight_factors(A, B)
        oAt, oBt = oracle.kron_weight_factors(A, B)
        for got, exp in ((At, oAt), (Bt, oBt)):
            ulp = np.spacing(np.abs(exp).astype(np.float32))
            assert np.all(np.abs(got.astype(np.float64) - exp) <= ulp)
        # inverse and transpose: A^T At = I (A^-T = (A^T)^-1)
        assert np.allclose(A.astype(np.float64).T @ At.astype(np.float64), np.eye(4), atol=1e-6)
        assert np.allclose(B.astype(np.float64).T @ Bt.astype(np.float64), np.eye(8), atol=1e-6)
    A, B = synth.kron_factors(0)
    At, Bt = mx.kron_weight_factors(A, B)
    oAt, oBt = oracle.kron_weight_factors(A, B)
    assert np.array_equal(At, oAt) and np.array_equal(Bt, oBt)
    w = synth.weight_f32(0, 64, 256, 3)
    assert all(np.array_equal(p, q) for p, q in zip(
        oracle.rotate_quantize(w, oracle.ROT_KRON_4x8, At, Bt),
        oracle.rotate_quantize(w, oracle.ROT_KRON_4x8, oAt, oBt)))


def test_kron_weight_factors_closed_forms_and_errors():
    # a permutation with scaling: inverse known exactly (powers of two)
    A = np.zeros((4, 4), np.float32)
    for i, j, v in ((0, 2, 2.0), (1, 0, -0.5), (2, 3, 4.0), (3, 1, 0.25)):
        A[i, j] = v
    B = np.diag(np.arange(1, 9, dtype=np.float32) * 2.0)
    At, Bt = mx.kron_weight_factors(A, B)
    assert np.array_equal(At, np.linalg.inv(A.astype(np.float64)).T.astype(np.float32))
    assert np.array_equal(np.diag(Bt), (1.0 / (np.arange(1, 9) * 2.0)).astype(np.float32))
    L = mx.lib
    buf4 = np.zeros((4, 4), np.float32)
    buf8 = np.zeros((8, 8), np.float32)
    eye4, eye8 = np.eye(4, dtype=np.float32), np.eye(8, dtype=np.float32)
    assert L.mxfp4_kron_weight_factors(None, eye8.ctypes.data, buf4.ctypes.data,
                                       buf8.ctypes.data) == mx.ERR_INVALID_ARG
    sing = eye4.copy()
    sing[2] = sing[1]
    assert L.mxfp4_kron_weight_factors(sing.ctypes.data, eye8.ctypes.data, buf4.ctypes.data,
                                       buf8.ctypes.data) == mx.ERR_INVALID_ARG
    nan8 = eye8.copy()
    nan8[3, 3] = np.nan
    assert L.mxfp4_kron_weight_factors(eye4.ctypes.data, nan8.ctypes.data, buf4.ctypes.data,
                                       buf8.ctypes.data) == mx.ERR_INVALID_ARG


def test_test_fault_hook_arguments():
    assert mx.lib.mxfp4_test_set_fault(7) == mx.ERR_UNSUPPORTED
    assert mx.lib.mxfp4_test_set_fault(mx.TEST_FAULT_NONE) == mx.OK


def test_linear_form_control():
    """mxfp4_set_linear_form overrides the choice by size (host only), and the default is
    restored."""
    kc, H = mx.linear_kernel_count, mx.ROT_HADAMARD32
    try:
        mx.set_linear_form(mx.LINEAR_ONE_KERNEL)
        assert kc(129, 16, 64, H) == 1 and kc(3584, 9216, 3072, mx.ROT_KRON_4x8) == 1
        assert kc(9, 4096, 14336, H) == 2                  # 9..128 rows: no one-kernel form
        assert kc(57344, 3072, 12288, mx.ROT_HADAMARD128) == 2
        assert kc(4, 128, 256, mx.ROT_NONE) == 1
        mx.set_linear_form(mx.LINEAR_TWO_KERNELS)
        assert kc(57344, 12288, 3072, H) == 2 and kc(4, 128, 256, mx.ROT_NONE) == 2
    finally:
        mx.set_linear_form(mx.LINEAR_AUTO)
    assert kc(57344, 12288, 3072, H) == 1 and kc(4, 128, 256, mx.ROT_NONE) == 1
    assert mx.lib.mxfp4_set_linear_form(3) == mx.ERR_UNSUPPORTED
    assert mx.lib.mxfp4_set_linear_form(-1) == mx.ERR_UNSUPPORTED


def test_one_kernel_size_rule_boundaries():
    """The large-problem one-kernel form needs at least 8 x 74 = 592 output tiles of
    256 x 256 and at least 40 MiB of bf16 x (M K >= 20971520): both edges exactly."""
    kc, H = mx.linear_kernel_count, mx.ROT_HADAMARD32
    assert kc(4096, 9472, 5120, H) == 1   # 16 x 37 = 592 tiles, M K = 20971520
    assert kc(4096, 9472, 5088, H) == 2   # M K one 32-block column short
    assert kc(4096, 9216, 5120, H) == 2   # 16 x 36 = 576 tiles
    assert kc(4096, 9472, 5120, mx.ROT_HADAMARD64) == 2  # wide groups: two kernels


def test_nvfp4_static_scale_argument_errors():
    """mxfp4_nvfp4_linear_static: the static activation scale must be given and 4-byte
    aligned; the rest is checked as for mxfp4_nvfp4_linear (all on the host, nothing
    launched); an empty call is valid."""
    L = mx.lib
    ws = mx.workspace_bytes(mx.OP_NVFP4_LINEAR, 4, 32, 64)
    assert L.mxfp4_nvfp4_linear_static(P, 4, 64, 0, None, P, P, P, 32, P, P, ws, None) == \
        mx.ERR_INVALID_ARG
    assert L.mxfp4_nvfp4_linear_static(P, 4, 64, 0, P + 2, P, P, P, 32, P, P, ws, None) == \
        mx.ERR_ALIGN
    assert L.mxfp4_nvfp4_linear_static(P, 4, 64, 2, P, P, P, P, 32, P, P, ws, None) == \
        mx.ERR_UNSUPPORTED
    assert L.mxfp4_nvfp4_linear_static(P, 4, 48, 0, P, P, P, P, 32, P, P, ws, None) == \
        mx.ERR_SHAPE
    assert L.mxfp4_nvfp4_linear_static(P, 4, 64, 0, P, P, P, P, 32, P, P, ws - 16, None) == \
        mx.ERR_WORKSPACE
    assert L.mxfp4_nvfp4_linear_static(P, 4, 64, 0, P, P, P, None, 32, P, P, ws, None) == \
        mx.ERR_INVALID_ARG
    assert L.mxfp4_nvfp4_linear_static(None, 0, 64, 1, P, P, P, P, 32, None, P, ws, None) == \
        mx.OK


def test_empty_calls_of_the_epilogue_norm_and_nvfp4_layers():
    """With no rows the remaining entry points validate their arguments and return OK
    without launching anything (so no device is touched here); the row operands may be
    NULL, the weight operands, scales and workspace stay required."""
    L = mx.lib
    ws = mx.workspace_bytes(mx.OP_GEMM, 0, 32, 64)
    assert L.mxfp4_gemm_bias(None, None, P, P, 0, 32, 64, P, None, 0, 32, P, ws, None) == mx.OK
    assert L.mxfp4_gemm_bias(None, None, P, P, 0, 32, 64, None, None, 0, 32, P, ws, None) == \
        mx.ERR_INVALID_ARG  # the bias stays required
    assert L.mxfp4_gemm_quantize(None, None, P, P, 0, 32, 64, None, 1, None, None, None, None, P,
                                 ws, None) == mx.OK
    assert L.mxfp4_gemm_quantize(None, None, None, P, 0, 32, 64, None, 1, None, None, None, None,
                                 P, ws, None) == mx.ERR_INVALID_ARG
    assert L.mxfp4_norm_rotate_quantize(None, 0, 64, 64, mx.NORM_LAYER, 1e-6, None, None, 1, None,
                                        None, None, None, P, None) == mx.OK
    assert L.mxfp4_norm_rotate_quantize(None, 0, 64, 64, mx.NORM_LAYER, 1e-6, None, None, 1, None,
                                        None, None, None, None, None) == mx.ERR_INVALID_ARG
    wsn = mx.workspace_bytes(mx.OP_NORM_LINEAR, 0, 32, 64)
    assert L.mxfp4_norm_linear(None, 0, 64, mx.NORM_RMS, 1e-6, None, None, 1, None, None, P, P,
                               32, None, P, wsn, None) == mx.OK
    assert L.mxfp4_nvfp4_quantize(None, 0, 0, 64, 64, 1, P, None, None, None) == mx.OK
    assert L.mxfp4_nvfp4_quantize(None, 0, 0, 64, 64, 1, None, None, None, None) == \
        mx.ERR_INVALID_ARG  # the tensor scale stays required
    assert L.mxfp4_nvfp4_gemm(None, None, P, P, P, P, 0, 32, 64, None, 0, 32, P, ws,
                              None) == mx.OK
    wsv = mx.workspace_bytes(mx.OP_NVFP4_LINEAR, 0, 32, 64)
    assert L.mxfp4_nvfp4_linear(None, 0, 64, 1, P, P, P, 32, None, P, wsv, None) == mx.OK
    assert L.mxfp4_nvfp4_linear_static(None, 0, 64, 1, P, P, P, P, 32, None, P, wsv,
                                       None) == mx.OK
    assert L.mxfp4_nvfp4_linear_static(None, 0, 64, 1, None, P, P, P, 32, None, P, wsv,
                                       None) == mx.ERR_INVALID_ARG
