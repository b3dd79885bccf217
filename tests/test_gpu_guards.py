"""Out-of-bounds writes and races, looked for without compute-sanitizer.

Every buffer a call writes (its outputs and its workspace) is cut from a larger allocation
whose bytes around it hold a seeded random pattern, and the call runs twice:
  - the bytes before and after each buffer must come back unchanged (a store past the end
    of a row, a tile or the buffer lands there); so must the bytes between the rows of an
    output with a leading dimension wider than its row;
  - each run starts from a different random pattern inside the outputs, and the two runs
    must give the same output bytes: an element no thread writes keeps its pattern and
    differs, and a race that changes a result differs too;
  - the workspace past its 256-byte status region starts as random bytes (the library
    writes every part of it before reading it), and the status word is still 0 after;
  - the inputs must be unchanged.
The shapes are small and ragged: row counts that fill no tile, columns that leave partial
tiles, K of one or a few 32-blocks, and each path of the GEMM (one or several CTAs per
output tile for few rows, the CTA-pair kernel, its last round in column halves). The
values themselves are checked against the oracle by the parity tests.
"""
import numpy as np
import pytest

import guards
import oracle
import synth

pytestmark = pytest.mark.gpu


def run_twice(what, inputs, call):
    import mxfp4_quantized_linear_block_b200 as mx
    guards.run_twice(what, inputs, call, "cuda", mx.poll_status)


def _dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _x_bf16(seed, rows, K, ld=None):
    """Seeded bf16 activations [rows, K] on the device, optionally inside a wider row."""
    import torch
    x, _ = synth.activation_bf16(seed, rows, K, 0.01, 30.0)
    if ld is None:
        return _dev(x.view(np.int16)).view(torch.bfloat16)
    big = np.zeros((rows, ld), np.uint16)
    big[:, :K] = x
    return _dev(big.view(np.int16)).view(torch.bfloat16)[:, :K]


def _mx_operand(seed, rows, K, tid):
    q = synth.uniform_u8(seed, synth.TID_CODES + tid, (rows, K // 2), 0, 255)
    s = synth.uniform_u8(seed, synth.TID_SCALES + tid, (rows, K // 32), 112, 138)
    return _dev(q), _dev(oracle.sf_to_physical(s, K))


def _kron(seed):
    A, B = synth.kron_factors(seed)
    return np.asarray(A, np.float32), np.asarray(B, np.float32)


# ---------------------------------------------------------------- quantisers

QUANT_CASES = [  # rows, K, ld (None: dense), dtype, mode
    (1, 32, None, "bf16", oracle.ROT_NONE),
    (131, 96, 128, "bf16", oracle.ROT_NONE),
    (300, 1056, None, "f32", oracle.ROT_NONE),
    (257, 160, 192, "bf16", oracle.ROT_HADAMARD32),
    (129, 64, None, "f32", oracle.ROT_KRON_4x8),
    (3, 4096, None, "bf16", oracle.ROT_HADAMARD32),
]


@pytest.mark.parametrize("rows,K,ld,dt,mode", QUANT_CASES)
def test_rotate_quantize_guards(rows, K, ld, dt, mode):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    x = _x_bf16(rows + K, rows, K, ld)
    if dt == "f32":
        x = x.float() * 1.37
    A, B = _kron(5) if mode == oracle.ROT_KRON_4x8 else (None, None)

    def call(ar):
        q = ar.out("q", rows, K // 2, torch.uint8)
        sf = ar.flat("sf", mx.sf_bytes(rows, K), torch.uint8)
        mx.rotate_quantize(x, mode, A, B, q=q, sf=sf)

    run_twice(f"rotate_quantize {rows}x{K} ld={ld} {dt} mode {mode}", [x], call)


@pytest.mark.parametrize("rows,K,kind,gb", [(77, 224, 0, True), (5, 96, 1, False),
                                            (130, 12288, 0, True), (3, 53248, 1, False)])
def test_norm_rotate_quantize_guards(rows, K, kind, gb):
    """One-pass (K up to 51168) and two-pass row statistics."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    x = _x_bf16(rows * 7 + K, rows, K)
    g = _dev(synth.normal_f32(3, 50, (K,), 0.2) + 1.0) if gb else None
    b = _dev(synth.normal_f32(3, 51, (K,), 0.1)) if gb else None
    kinds = (mx.NORM_LAYER, mx.NORM_RMS)

    def call(ar):
        q = ar.out("q", rows, K // 2, torch.uint8)
        sf = ar.flat("sf", mx.sf_bytes(rows, K), torch.uint8)
        st = ar.out("stats", rows, 2, torch.float32)
        mx.norm_rotate_quantize(x, kinds[kind], 1e-6, g, b, mx.ROT_HADAMARD32, q=q, sf=sf,
                                stats=st)

    run_twice(f"norm_rotate_quantize {rows}x{K} kind {kind}",
               [x] + ([g, b] if gb else []), call)


@pytest.mark.parametrize("rows,K,mode", [(1, 32, oracle.ROT_NONE), (131, 96, oracle.ROT_NONE),
                                         (257, 1056, oracle.ROT_HADAMARD32)])
def test_nvfp4_quantize_guards(rows, K, mode):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    x = _x_bf16(rows * 5 + K, rows, K)

    def call(ar):
        sc = ar.flat("scale2", 8, torch.float32)
        sc.zero_()
        mx.nvfp4_tensor_scale(x, mode, scale2=sc)
        q = ar.out("q", rows, K // 2, torch.uint8)
        sf = ar.flat("sf", mx.nvfp4_sf_bytes(rows, K), torch.uint8)
        mx.nvfp4_quantize(x, sc, mode, q=q, sf=sf)

    run_twice(f"nvfp4 quantize {rows}x{K} mode {mode}", [x], call)


# ---------------------------------------------------------------- GEMMs

GEMM_CASES = [  # M, N, K, out, ld pad (elements)
    (1, 16, 32, "bf16", 0),
    (17, 48, 96, "f32", 16),
    (32, 4096, 2048, "bf16", 0),     # few rows, on-chip cluster sum
    (77, 4096, 2048, "bf16", 8),     # few rows, partial sums through the workspace
    (77, 4096, 2048, "f32", 4),
    (128, 8192, 1024, "bf16", 0),    # few rows, one CTA per SM with deep staging
    (129, 272, 288, "f32", 0),       # CTA pairs, ragged rows and columns
    (300, 384, 512, "bf16", 24),
    (700, 2496, 160, "bf16", 0),     # CTA pairs, last round in column halves, ragged
    (700, 784, 6176, "f32", 16),
]


@pytest.mark.parametrize("M,N,K,out,pad", GEMM_CASES)
def test_gemm_guards(M, N, K, out, pad):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    aq, asf = _mx_operand(M + N + K, M, K, 1)
    bq, bsf = _mx_operand(M + N + K, N, K, 2)
    dt = torch.float32 if out == "f32" else torch.bfloat16

    def call(ar):
        y = ar.out("y", M, N, dt, ld=N + pad)
        ws = ar.workspace(mx.workspace_bytes(mx.OP_GEMM, M, N, K))
        mx.gemm(aq, asf, bq, bsf, M, N, K, y=y, ws=ws)

    run_twice(f"gemm {M}x{N}x{K} {out} ld+{pad}", [aq, asf, bq, bsf], call)


def test_gemm_guard_cases_reach_every_path():
    """The few-row cases above include one with workspace partials; the pair cases none."""
    import mxfp4_quantized_linear_block_b200 as mx
    assert mx.workspace_bytes(mx.OP_GEMM, 77, 4096, 2048) > 256
    assert mx.workspace_bytes(mx.OP_GEMM, 32, 4096, 2048) == 256
    assert mx.workspace_bytes(mx.OP_GEMM, 700, 2496, 160) == 256
    tiles = -(-700 // 256) * -(-2496 // 256)
    assert 0 < tiles % 74 <= 37  # the last round runs in column halves


@pytest.mark.parametrize("M,N,K", [(33, 512, 256), (300, 384, 512)])
def test_gemm_bias_guards(M, N, K):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    aq, asf = _mx_operand(M * 3 + K, M, K, 3)
    bq, bsf = _mx_operand(M * 3 + K, N, K, 4)
    bias = _dev(synth.normal_f32(M, 52, (N,), 0.5))

    def call(ar):
        y = ar.out("y", M, N, torch.bfloat16, ld=N + 8)
        ws = ar.workspace(mx.workspace_bytes(mx.OP_GEMM, M, N, K))
        mx.gemm_bias(aq, asf, bq, bsf, M, N, K, bias, y=y, ws=ws)

    run_twice(f"gemm_bias {M}x{N}x{K}", [aq, asf, bq, bsf, bias], call)


@pytest.mark.parametrize("M,N,K,mode", [(20, 256, 128, oracle.ROT_HADAMARD32),
                                        (300, 384, 512, oracle.ROT_HADAMARD32),
                                        (129, 256, 64, oracle.ROT_KRON_4x8),
                                        (700, 2496, 160, oracle.ROT_NONE)])
def test_gemm_quantize_guards(M, N, K, mode):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    aq, asf = _mx_operand(M * 5 + K, M, K, 5)
    bq, bsf = _mx_operand(M * 5 + K, N, K, 6)
    bias = _dev(synth.normal_f32(M, 53, (N,), 0.5))
    A, B = _kron(6) if mode == oracle.ROT_KRON_4x8 else (None, None)

    def call(ar):
        yq = ar.out("yq", M, N // 2, torch.uint8)
        ysf = ar.flat("ysf", mx.sf_bytes(M, N), torch.uint8)
        ws = ar.workspace(mx.workspace_bytes(mx.OP_GEMM, M, N, K))
        mx.gemm_quantize(aq, asf, bq, bsf, M, N, K, bias, mode, A, B, yq=yq, ysf=ysf, ws=ws)

    run_twice(f"gemm_quantize {M}x{N}x{K} mode {mode}", [aq, asf, bq, bsf, bias], call)


@pytest.mark.parametrize("M,N,K,out", [(5, 64, 64, "bf16"), (300, 384, 512, "f32"),
                                       (700, 2496, 160, "bf16")])
def test_nvfp4_gemm_guards(M, N, K, out):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    aq = _dev(synth.uniform_u8(M + K, synth.TID_CODES + 40, (M, K // 2), 0, 255))
    bq = _dev(synth.uniform_u8(M + K, synth.TID_CODES + 41, (N, K // 2), 0, 255))
    asf = _dev(oracle.nvfp4_sf_to_physical(
        synth.uniform_u8(M + K, synth.TID_SCALES + 40, (M, K // 16), 24, 80), K))
    bsf = _dev(oracle.nvfp4_sf_to_physical(
        synth.uniform_u8(M + K, synth.TID_SCALES + 41, (N, K // 16), 24, 80), K))
    sa = torch.tensor([0.75, 0.0], dtype=torch.float32, device="cuda")
    sb = torch.tensor([1.25, 0.0], dtype=torch.float32, device="cuda")
    dt = torch.float32 if out == "f32" else torch.bfloat16

    def call(ar):
        y = ar.out("y", M, N, dt, ld=N + 16)
        ws = ar.workspace(mx.workspace_bytes(mx.OP_GEMM, M, N, K))
        mx.nvfp4_gemm(aq, asf, sa, bq, bsf, sb, M, N, K, y=y, ws=ws)

    run_twice(f"nvfp4_gemm {M}x{N}x{K} {out}", [aq, asf, bq, bsf, sa, sb], call)


# ---------------------------------------------------------------- layers

LINEAR_CASES = [  # M, K, N, mode
    (1, 4096, 4096, oracle.ROT_HADAMARD32),
    (5, 512, 256, oracle.ROT_HADAMARD32),
    (77, 2048, 4096, oracle.ROT_KRON_4x8),
    (300, 1024, 384, oracle.ROT_HADAMARD32),
    (700, 160, 2496, oracle.ROT_HADAMARD32),
    (2560, 6144, 2048, oracle.ROT_HADAMARD32),
]


@pytest.mark.parametrize("M,K,N,mode", LINEAR_CASES)
def test_linear_guards(M, K, N, mode):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    x = _x_bf16(M + 2 * K, M, K)
    wq, wsf = _mx_operand(M + 2 * K, N, K, 7)
    A, B = _kron(7) if mode == oracle.ROT_KRON_4x8 else (None, None)

    def call(ar):
        y = ar.out("y", M, N, torch.bfloat16)
        ws = ar.workspace(mx.workspace_bytes(mx.OP_LINEAR, M, N, K))
        mx.linear(x, wq, wsf, N, mode, A, B, y=y, ws=ws)

    run_twice(f"linear {M}x{K}->{N} mode {mode}", [x, wq, wsf], call)


def test_linear_guard_cases_reach_both_launch_forms():
    """Among the cases above, some quantise x inside the GEMM's CTAs (one kernel) and some
    run the quantiser first (two kernels)."""
    import mxfp4_quantized_linear_block_b200 as mx
    counts = {mx.linear_kernel_count(M, N, K, mode) for M, K, N, mode in LINEAR_CASES}
    assert counts == {1, 2}, counts


@pytest.mark.parametrize("M,K,N,mode", [(129, 64, 16, oracle.ROT_NONE),
                                        (300, 1024, 384, oracle.ROT_HADAMARD32),
                                        (700, 160, 2496, oracle.ROT_KRON_4x8),
                                        (2560, 6144, 2048, oracle.ROT_HADAMARD32)])
def test_linear_one_kernel_guards(M, K, N, mode):
    """The layer for more than 128 rows as one kernel (forced here for small sizes): its
    row counters past the scales and everything around its buffers."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    x = _x_bf16(M + 5 * K, M, K)
    wq, wsf = _mx_operand(M + 5 * K, N, K, 10)
    A, B = _kron(8) if mode == oracle.ROT_KRON_4x8 else (None, None)

    def call(ar):
        y = ar.out("y", M, N, torch.bfloat16)
        ws = ar.workspace(mx.workspace_bytes(mx.OP_LINEAR, M, N, K))
        mx.linear(x, wq, wsf, N, mode, A, B, y=y, ws=ws)

    mx.set_linear_form(mx.LINEAR_ONE_KERNEL)
    try:
        run_twice(f"one-kernel linear {M}x{K}->{N} mode {mode}", [x, wq, wsf], call)
    finally:
        mx.set_linear_form(mx.LINEAR_AUTO)


@pytest.mark.parametrize("M,K,N,kind", [(77, 224, 256, 0), (300, 1024, 384, 1),
                                        (3, 53248, 64, 1)])
def test_norm_linear_guards(M, K, N, kind):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    x = _x_bf16(M * 11 + K, M, K)
    g = _dev(synth.normal_f32(4, 50, (K,), 0.2) + 1.0)
    b = _dev(synth.normal_f32(4, 51, (K,), 0.1)) if kind == 0 else None
    wq, wsf = _mx_operand(M + K, N, K, 8)
    kinds = (mx.NORM_LAYER, mx.NORM_RMS)

    def call(ar):
        y = ar.out("y", M, N, torch.bfloat16)
        ws = ar.workspace(mx.workspace_bytes(mx.OP_NORM_LINEAR, M, N, K))
        mx.norm_linear(x, wq, wsf, N, kinds[kind], 1e-6, g, b, mx.ROT_HADAMARD32, y=y, ws=ws)

    run_twice(f"norm_linear {M}x{K}->{N} kind {kind}",
               [x, g, wq, wsf] + ([b] if b is not None else []), call)


@pytest.mark.parametrize("M,K,N", [(5, 256, 128), (131, 256, 128), (300, 1024, 384)])
def test_nvfp4_linear_guards(M, K, N):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    x = _x_bf16(M * 13 + K, M, K)
    wq = _dev(synth.uniform_u8(M + K, synth.TID_CODES + 42, (N, K // 2), 0, 255))
    wsf = _dev(oracle.nvfp4_sf_to_physical(
        synth.uniform_u8(M + K, synth.TID_SCALES + 42, (N, K // 16), 24, 80), K))
    wsc = torch.tensor([0.5, 0.0], dtype=torch.float32, device="cuda")

    def call(ar):
        y = ar.out("y", M, N, torch.bfloat16)
        ws = ar.workspace(mx.workspace_bytes(mx.OP_NVFP4_LINEAR, M, N, K))
        mx.nvfp4_linear(x, wq, wsf, wsc, N, mx.ROT_HADAMARD32, y=y, ws=ws)

    run_twice(f"nvfp4_linear {M}x{K}->{N}", [x, wq, wsf, wsc], call)


@pytest.mark.parametrize("M,K,N", [(5, 256, 128), (300, 1024, 384)])
def test_nvfp4_linear_static_guards(M, K, N):
    """The NVFP4 layer with a static activation scale (two kernels)."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    x = _x_bf16(M * 19 + K, M, K)
    wq = _dev(synth.uniform_u8(M + K, synth.TID_CODES + 43, (N, K // 2), 0, 255))
    wsf = _dev(oracle.nvfp4_sf_to_physical(
        synth.uniform_u8(M + K, synth.TID_SCALES + 43, (N, K // 16), 24, 80), K))
    wsc = torch.tensor([0.5, 0.0], dtype=torch.float32, device="cuda")
    xsc = torch.tensor([0.125, 0.0], dtype=torch.float32, device="cuda")

    def call(ar):
        y = ar.out("y", M, N, torch.bfloat16)
        ws = ar.workspace(mx.workspace_bytes(mx.OP_NVFP4_LINEAR, M, N, K))
        mx.nvfp4_linear_static(x, xsc, wq, wsf, wsc, N, mx.ROT_HADAMARD32, y=y, ws=ws)

    run_twice(f"nvfp4_linear_static {M}x{K}->{N}", [x, wq, wsf, wsc, xsc], call)


@pytest.mark.parametrize("M,K,N", [(5, 512, 256), (300, 1024, 384)])
def test_linear_noalloc_guards(M, K, N):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    x = _x_bf16(M * 17 + K, M, K)
    wq, wsf = _mx_operand(M + 3 * K, N, K, 9)

    def call(ar):
        y = ar.out("y", M, N, torch.bfloat16)
        status = ar.flat("status", 16, torch.int32)
        status.zero_()
        mx.linear_noalloc(x, wq, wsf, N, mx.ROT_HADAMARD32, y=y, status=status)
        torch.cuda.synchronize()
        assert int(status[0]) == 0

    run_twice(f"linear_noalloc {M}x{K}->{N}", [x, wq, wsf], call)
