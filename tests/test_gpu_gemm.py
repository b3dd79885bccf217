"""GPU parity of the tcgen05 block-scaled GEMM against the oracle's exact contraction."""
import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import bf16_dev_to_f64, check_gemm_values, to_dev

pytestmark = pytest.mark.gpu


def _operand(seed, rows, K, tid, lo=112, hi=138):
    q = synth.uniform_u8(seed, synth.TID_CODES + tid, (rows, K // 2), 0, 255)
    s = synth.uniform_u8(seed, synth.TID_SCALES + tid, (rows, K // 32), lo, hi)
    return q, s


def _run(aq, as_, bq, bs, out):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    M, K = aq.shape[0], aq.shape[1] * 2
    N = bq.shape[0]
    y = mx.gemm(to_dev(aq), to_dev(oracle.sf_to_physical(as_, K)), to_dev(bq),
                to_dev(oracle.sf_to_physical(bs, K)), M, N, K,
                out_dtype=torch.float32 if out == "f32" else torch.bfloat16)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64) if out == "f32" else bf16_dev_to_f64(y)


SHAPES = [
    (1, 16, 32), (2, 16, 64), (64, 128, 256), (127, 144, 96), (128, 256, 256), (129, 272, 288),
    (300, 384, 512), (256, 512, 1024), (200, 400, 3072), (130, 128, 320),
]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_gemm_shapes(M, N, K, out):
    aq, as_ = _operand(M * 31 + N * 7 + K, M, K, 0)
    bq, bs = _operand(M * 31 + N * 7 + K, N, K, 1)
    y = _run(aq, as_, bq, bs, out)
    ref, S = oracle.gemm(aq, as_, bq, bs)
    check_gemm_values(y, ref, S, out, f"gemm {M}x{N}x{K} {out}")


def test_gemm_zero_and_single_pair():
    K = 512
    aq = np.zeros((130, K // 2), np.uint8)
    bq = np.zeros((144, K // 2), np.uint8)
    as_ = synth.uniform_u8(1, 90, (130, K // 32), 100, 150)
    bs = synth.uniform_u8(1, 91, (144, K // 32), 100, 150)
    y = _run(aq, as_, bq, bs, "f32")
    assert not y.any()
    aq[129, 200] = 13 << 4   # element 401 = -3
    bq[143, 200] = 3 << 4    # element 401 = 1.5
    y = _run(aq, as_, bq, bs, "f32")
    expect = -3 * 1.5 * 2.0 ** (int(as_[129, 401 // 32]) + int(bs[143, 401 // 32]) - 254)
    assert y[129, 143] == expect
    y[129, 143] = 0
    assert not y.any()


# Few activation rows (M <= 128): the weight-streaming kernel splits K over the
# CTAs of a thread-block cluster (two CTAs per SM, one for 65..128 rows) and adds the
# partials through distributed shared memory (up to 32 rows, or fewer than 4 splits) or
# through L2 (33..128 rows split 4 or more ways, with the workspace's scratch).
# (M, N, K) -> W tiles x K splits: (1,16,4096) 1x8; (5,400,2080) 4x5 with a 32-element
# K tail; (16,256,8192) 2x8; (17,12288,1024) 96x2; (33,9216,1536) 72x3; (64,2048,3104)
# 16x7 with a K tail (L2); (100,1024,7168) 8x7 (L2); (65,14336,4096) 112x1 (no sum);
# (128,4096,14336) 32x4 (L2).
SMALLM_SHAPES = [
    (1, 16, 4096), (5, 400, 2080), (16, 256, 8192), (17, 12288, 1024), (33, 9216, 1536),
    (64, 2048, 3104), (100, 1024, 7168), (65, 14336, 4096), (128, 4096, 14336),
]


@pytest.mark.parametrize("M,N,K", SMALLM_SHAPES)
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_gemm_few_rows_split_k(M, N, K, out):
    aq, as_ = _operand(M * 17 + N + K, M, K, 6)
    bq, bs = _operand(M * 17 + N + K, N, K, 7)
    y = _run(aq, as_, bq, bs, out)
    ref, S = oracle.gemm(aq, as_, bq, bs)
    check_gemm_values(y, ref, S, out, f"few-row gemm {M}x{N}x{K} {out}")


def test_gemm_few_rows_single_pair_in_last_split():
    """One nonzero product in the K tail, which only the last split of the cluster
    holds: the cross-CTA sum must carry it to exactly one output, unchanged."""
    M, N, K = 3, 400, 2080
    aq = np.zeros((M, K // 2), np.uint8)
    bq = np.zeros((N, K // 2), np.uint8)
    as_ = synth.uniform_u8(2, 92, (M, K // 32), 100, 150)
    bs = synth.uniform_u8(2, 93, (N, K // 32), 100, 150)
    aq[2, K // 2 - 1] = 7 << 4    # element K-1 = 6
    bq[399, K // 2 - 1] = 12 << 4  # element K-1 = -2
    y = _run(aq, as_, bq, bs, "f32")
    expect = 6 * -2 * 2.0 ** (int(as_[2, K // 32 - 1]) + int(bs[399, K // 32 - 1]) - 254)
    assert y[2, 399] == expect
    y[2, 399] = 0
    assert not y.any()


# Large-M shapes whose last round of 256x256 tiles leaves at least half of the 74 CTA
# pairs of a B200 idle, so that its tiles run as two 256 x 128 units each (N = 128 MMAs,
# the scale group of the column half): tiles -> units. (512,512,4096) 4 -> 8;
# (768,1024,8192) 12 -> 24; (700,784,6176) 12 ragged tiles -> 24, a 32-element K tail,
# and a last column tile of 16 columns (its second half lies wholly past N).
HALF_SHAPES = [(512, 512, 4096), (768, 1024, 8192), (700, 784, 6176)]


@pytest.mark.parametrize("M,N,K", HALF_SHAPES)
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_gemm_last_round_in_column_halves(M, N, K, out):
    aq, as_ = _operand(M + 3 * N + K, M, K, 8)
    bq, bs = _operand(M + 3 * N + K, N, K, 9)
    y = _run(aq, as_, bq, bs, out)
    ref, S = oracle.gemm(aq, as_, bq, bs)
    check_gemm_values(y, ref, S, out, f"column-half gemm {M}x{N}x{K} {out}")


def test_gemm_full_rounds_then_column_halves():
    """80 tiles on 74 pairs: one round of whole tiles, then 6 tiles as 12 column-half
    units. Every element of the last 256-row band (which holds the 6 tiles of the last
    round) is checked, plus sampled pairs elsewhere."""
    M, N, K = 2560, 2048, 6144
    aq, as_ = _operand(5, M, K, 10)
    bq, bs = _operand(5, N, K, 11)
    y = _run(aq, as_, bq, bs, "f32")
    ref, S = oracle.gemm(aq[M - 256:], as_[M - 256:], bq, bs)
    check_gemm_values(y[M - 256:], ref, S, "f32", "last band")
    mi, ni = _sample_pairs(M, N, n_random=2048, seed=3)
    ref, S = oracle.gemm_pairs(aq, as_, bq, bs, mi, ni)
    check_gemm_values(y[mi, ni], ref, S, "f32", "sampled")


def test_gemm_column_halves_repeat():
    """Back-to-back launches on different inputs through one workspace (the status
    region alone): each result is right and repeated inputs give identical bits."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    M, N, K = 768, 1024, 8192
    ws = mx.new_workspace(mx.workspace_bytes(mx.OP_GEMM, M, N, K))
    assert ws.numel() == 256
    outs = []
    for seed in (21, 22, 21):
        aq, as_ = _operand(seed, M, K, 12)
        bq, bs = _operand(seed, N, K, 13)
        y = mx.gemm(to_dev(aq), to_dev(oracle.sf_to_physical(as_, K)), to_dev(bq),
                    to_dev(oracle.sf_to_physical(bs, K)), M, N, K,
                    out_dtype=torch.float32, ws=ws)
        torch.cuda.synchronize()
        outs.append(y.cpu().numpy())
        ref, S = oracle.gemm(aq, as_, bq, bs)
        check_gemm_values(outs[-1].astype(np.float64), ref, S, "f32", f"seed {seed}")
    assert np.array_equal(outs[0].view(np.uint32), outs[2].view(np.uint32))
    assert mx.poll_status(ws) == mx.OK


def test_gemm_wide_scale_range_fp32():
    """Scales spread over most of the E8M0 range in fp32 output."""
    M, N, K = 256, 256, 1024
    aq, as_ = _operand(11, M, K, 2, 70, 180)
    bq, bs = _operand(11, N, K, 3, 70, 180)
    y = _run(aq, as_, bq, bs, "f32")
    ref, S = oracle.gemm(aq, as_, bq, bs)
    check_gemm_values(y, ref, S, "f32", "wide scales")


def _sample_pairs(M, N, BN=256, n_random=4096, seed=0):
    """(m, n) pairs the oracle computes one by one: the first and last row tile
    against the first and last column tile, 8 edge rows x every column, every
    row x 4 edge columns, and n_random seeded random pairs."""
    rows = np.unique(np.r_[np.arange(min(128, M)), np.arange(max(0, M - 128), M)])
    cols = np.unique(np.r_[np.arange(min(BN, N)), np.arange(max(0, N - BN), N)])
    edge_rows = np.unique(np.r_[rows[:4], rows[-4:]])
    edge_cols = np.unique(np.r_[cols[:2], cols[-2:]])
    rng = np.random.default_rng(seed)
    mi = [np.repeat(rows, cols.size), np.repeat(edge_rows, N), np.tile(np.arange(M), edge_cols.size),
          rng.integers(0, M, n_random)]
    ni = [np.tile(cols, rows.size), np.tile(np.arange(N), edge_rows.size),
          np.repeat(edge_cols, M), rng.integers(0, N, n_random)]
    return np.concatenate(mi).astype(np.int64), np.concatenate(ni).astype(np.int64)


@pytest.mark.parametrize("M,N,K", [(3584, 9216, 3072), (3584, 3072, 12288)])
def test_gemm_full_size_sampled(M, N, K):
    aq, as_ = _operand(K, M, K, 4)
    bq, bs = _operand(K, N, K, 5)
    y = _run(aq, as_, bq, bs, "bf16")
    mi, ni = _sample_pairs(M, N)
    ref, S = oracle.gemm_pairs(aq, as_, bq, bs, mi, ni)
    check_gemm_values(y[mi, ni], ref, S, "bf16", f"gemm {M}x{N}x{K} sampled")


@pytest.mark.parametrize("M,N,K", [(5, 144, 512), (300, 272, 768)])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_gemm_padded_output_rows(M, N, K, out):
    """y with a row stride larger than N (both kernels): the N columns of every row are
    the product, the padding between rows is never written."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    aq, as_ = _operand(M + N, M, K, 14)
    bq, bs = _operand(M + N, N, K, 15)
    dt = torch.float32 if out == "f32" else torch.bfloat16
    pad = 24 if out == "bf16" else 12  # row stride stays a multiple of 16 bytes
    big = torch.full((M, N + pad), 7.0, dtype=dt, device="cuda")
    y = big[:, :N]
    mx.gemm(to_dev(aq), to_dev(oracle.sf_to_physical(as_, K)), to_dev(bq),
            to_dev(oracle.sf_to_physical(bs, K)), M, N, K, y=y)
    torch.cuda.synchronize()
    assert torch.all(big[:, N:] == 7.0)
    got = y.float().cpu().numpy().astype(np.float64)
    ref, S = oracle.gemm(aq, as_, bq, bs)
    check_gemm_values(got, ref, S, out, f"padded rows {M}x{N}x{K} {out}")


def test_gemm_and_linear_with_no_rows_write_nothing():
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    K, N = 256, 128
    y = torch.full((1, N), 3.0, dtype=torch.bfloat16, device="cuda")
    x = torch.zeros((1, K), dtype=torch.bfloat16, device="cuda")[:0]  # M = 0, non-null
    wq = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    wsf = torch.zeros(mx.sf_bytes(N, K), dtype=torch.uint8, device="cuda")
    mx.gemm(torch.zeros((1, K // 2), dtype=torch.uint8, device="cuda"),
            torch.zeros(mx.sf_bytes(1, K), dtype=torch.uint8, device="cuda"), wq, wsf, 0, N, K,
            y=y)
    mx.linear(x, wq, wsf, N, y=y[:0])
    torch.cuda.synchronize()
    assert torch.all(y == 3.0)


@pytest.mark.parametrize("M,N,K", [(33, 4608, 1536), (100, 1024, 7168), (128, 4096, 14336)])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_few_rows_l2_and_on_chip_sums_agree(M, N, K, out):
    """33..128 rows split 4 to 7 ways (36 W tiles x 6, 8 x 7, 32 x 4) sum their K splits
    through L2 when the workspace has room for the partials past its 256-byte head,
    and through distributed shared memory when it has only the status region: same order
    of additions, so the same bits; both match the oracle."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    aq, as_ = _operand(M + N + K, M, K, 12)
    bq, bs = _operand(M + N + K, N, K, 13)
    args = (to_dev(aq), to_dev(oracle.sf_to_physical(as_, K)), to_dev(bq),
            to_dev(oracle.sf_to_physical(bs, K)), M, N, K)
    dt = torch.float32 if out == "f32" else torch.bfloat16
    full = mx.new_workspace(mx.workspace_bytes(mx.OP_GEMM, M, N, K))
    assert full.numel() > 256  # this size uses the L2 form
    y_l2 = mx.gemm(*args, out_dtype=dt, ws=full)
    y_chip = mx.gemm(*args, out_dtype=dt, ws=mx.new_workspace(256))
    torch.cuda.synchronize()
    assert torch.equal(y_l2, y_chip)
    y = y_l2.cpu().numpy().astype(np.float64) if out == "f32" else bf16_dev_to_f64(y_l2)
    ref, S = oracle.gemm(aq, as_, bq, bs)
    check_gemm_values(y, ref, S, out, f"few-row L2 sum {M}x{N}x{K} {out}")
    assert mx.poll_status(full) == mx.OK


def test_workspace_shared_by_few_row_and_pair_kernels():
    """One workspace serves a 128-row call (its L2 partials past the status region),
    then a pair call whose last round runs in column halves, and again."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    shapes = [(128, 4096, 14336), (512, 512, 4096)]
    ws = mx.new_workspace(max(mx.workspace_bytes(mx.OP_GEMM, *sh) for sh in shapes))
    for rep in range(2):
        for (M, N, K) in shapes:
            aq, as_ = _operand(M + N, M, K, 14)
            bq, bs = _operand(M + N, N, K, 15)
            y = mx.gemm(to_dev(aq), to_dev(oracle.sf_to_physical(as_, K)), to_dev(bq),
                        to_dev(oracle.sf_to_physical(bs, K)), M, N, K, out_dtype=torch.float32,
                        ws=ws)
            torch.cuda.synchronize()
            ref, S = oracle.gemm(aq, as_, bq, bs)
            check_gemm_values(y.cpu().numpy().astype(np.float64), ref, S, "f32",
                              f"shared workspace {M}x{N}x{K} pass {rep}")
            assert mx.poll_status(ws) == mx.OK
