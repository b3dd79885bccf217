"""GPU parity of the norm prologue (LayerNorm / RMSNorm, + adaLN-style g and b, before the
rotation and quantisation). The expected side comes from the oracle alone: its row
statistics are exact (double), rounded once to fp32, and its normalise-rotate-quantise
uses those.

Bit-exact tests use rows built so that every fp32 sum the statistics take is exact in any
order: elements are multiples of 1/16 (|x| <= 4, exact in bf16), a LayerNorm row is
mu0 + d with the deviations d in +/- pairs (so the mean is exactly mu0), |d| <= 2 (or
<= 1/2 for K = 65536) so that sum d^2 stays below 2^24 quanta of 1/256, and K is a power
of two (exact divisions). eps is 0 or 2^-12 (exact in fp32 and double). The kernel's
mean is then the oracle's exactly and its variance too; its rstd is a correctly rounded
1/sqrt of the same fp32 number, which is the oracle's rounded value unless the double
result lies on a rounding boundary (checked with 60-digit decimals). So statistics,
codes and scale bytes must all match bit for bit.

Realistic rows (N(0,1) with outlier channels, a non-zero mean) are checked too: the
kernel's statistics within the fp32 summation bound of the exact ones, and the codes
against the oracle's with the oracle's own statistics, every block whose decisions lie
farther than that bound (spread through the normalisation and rotation) from a boundary
bit for bit, the rest within one step, with their count reported.
"""
from decimal import Decimal, getcontext

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import bf16_dev_to_f64, check_gemm_values, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


def _vec(seed, K, mean, std):
    return (mean + std * synth.normal_f32(seed, 77, (1, K))[0]).astype(np.float32)


def _exact_rows(seed, rows, K, kind):
    """bf16 rows whose statistics are exact in fp32 whatever the summation order."""
    assert K & (K - 1) == 0 and K >= 64
    dmax16 = 32 if K <= 4096 else 8  # |d| <= 2 or 1/2, in sixteenths
    n = synth.uniform_u8(seed, 60, (rows, K // 2), 0, 2 * dmax16).astype(np.int64) - dmax16
    if kind == oracle.NORM_LAYER:
        d = np.concatenate([n, -n], axis=1)
        # spread the pairs over the row with a seeded permutation per row
        perm = np.argsort(synth.raw_u64(seed, 61, rows * K).reshape(rows, K), axis=1)
        d = np.take_along_axis(d, perm, axis=1)
        mu0 = synth.uniform_u8(seed, 62, (rows, 1), 0, 64).astype(np.int64) - 32
        x16 = mu0 + d                            # |x| <= 4 in sixteenths of 1
    else:
        x16 = synth.uniform_u8(seed, 63, (rows, K), 0, 2 * dmax16).astype(np.int64) - dmax16
    x = (x16.astype(np.float64) / 16.0).astype(np.float32)
    bits = synth.f32_to_bf16_bits(x)
    assert np.array_equal(synth.bf16_bits_to_f32(bits), x)
    return bits


def _rstd_f32_exact(x_bits, kind, eps):
    """1 / sqrt(var + eps) of each row to 60 digits, rounded to fp32 (for the rows above
    var + eps is an fp32 number, so this is what a correctly rounded rsqrt gives)."""
    getcontext().prec = 60
    x = synth.bf16_bits_to_f32(x_bits).astype(np.float64)
    out = []
    for row in x:
        K = row.size
        mu = Decimal(0) if kind == oracle.NORM_RMS else sum(Decimal(float(v)) for v in row) / K
        var = sum((Decimal(float(v)) - mu) ** 2 for v in row) / K + Decimal(eps)
        r = Decimal(1) / var.sqrt()
        out.append(np.float32(float(r)))  # float(): nearest double; then nearest fp32
        # the double is within half a double ulp of r; make sure no fp32 boundary lies between
        lo, hi = np.float32(float(r * (1 - Decimal(2) ** -52))), np.float32(float(r * (1 + Decimal(2) ** -52)))
        assert lo == hi == out[-1], "rstd on an fp32 rounding boundary: pick other rows"
    return np.array(out, np.float32)


def _oracle_stats_f32(x, kind, eps):
    mu, rstd = oracle.row_stats(x, kind, eps)
    return mu.astype(np.float32), rstd.astype(np.float32)


@pytest.mark.parametrize("kind", [oracle.NORM_LAYER, oracle.NORM_RMS])
# K <= 51168 takes the one-pass kernel (groups of 16 .. 1 rows per CTA, a partial last group
# included; 16384 and 32768: groups of 2 and 1 rows); K = 65536 the statistics kernel +
# norm quantiser.
@pytest.mark.parametrize("rows,K", [(1, 64), (5, 1024), (129, 1024), (17, 4096), (300, 2048),
                                    (9, 16384), (3, 32768), (3, 65536)])
@pytest.mark.parametrize("eps", [0.0, 2.0 ** -12])
def test_norm_rotate_quantize_exact_rows(kind, rows, K, eps):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    x = _exact_rows(rows * 7 + K + kind, rows, K, kind)
    mu, rstd = _oracle_stats_f32(x, kind, eps)
    assert np.array_equal(rstd, _rstd_f32_exact(x, kind, eps))
    g = _vec(1, K, 1.0, 0.2)
    b = _vec(2, K, 0.0, 0.5)
    A, B = synth.kron_factors(0)
    for mode in (oracle.ROT_NONE, oracle.ROT_HADAMARD32, oracle.ROT_KRON_4x8):
        for affine in (False, True):
            gg, bb = (g, b) if affine else (None, None)
            AA, BB = (A, B) if mode == oracle.ROT_KRON_4x8 else (None, None)
            q, sf, st = mx.norm_rotate_quantize(
                to_dev_bf16(x), kind, eps, to_dev(gg) if affine else None,
                to_dev(bb) if affine else None, mode, AA, BB)
            torch.cuda.synchronize()
            st = st.cpu().numpy()
            assert np.array_equal(st[:, 0], mu), "mean"
            assert np.array_equal(st[:, 1], rstd), "rstd"
            q_ref, s_ref = oracle.norm_rotate_quantize(x, mu, rstd, gg, bb, mode, AA, BB)
            assert np.array_equal(q.cpu().numpy(), q_ref), f"codes mode {mode} affine {affine}"
            assert np.array_equal(sf.cpu().numpy()[: oracle.sf_bytes(rows, K)],
                                  oracle.sf_to_physical(s_ref, K)), f"scales mode {mode}"


def _stat_bounds(x, kind, K):
    """fp32 summation of K terms: |error| <= K u sum |terms| (u = 2^-24), doubled."""
    u = 2.0 ** -24
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    dmu = 2 * K * u * np.abs(xf).mean(axis=1)
    drel = 2 * K * u + 1e-6
    return dmu, drel


def _norm_open_blocks(x, mu, rstd, dmu, drel, g, b, mode):
    """Blocks whose codes the statistics' error bound leaves open: v = ((x - mu) rstd) g + b
    moves by at most (dmu rstd + |x - mu| rstd drel) |g| + 4 ulp(v); the Hadamard rotation
    spreads that by 1/sqrt(32) per term and adds its own 6 roundings."""
    rows, K = x.shape
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    gg = np.ones(K) if g is None else g.astype(np.float64)
    bb = np.zeros(K) if b is None else b.astype(np.float64)
    v = ((xf - mu[:, None]) * rstd[:, None]) * gg + bb
    dv = (dmu[:, None] * rstd[:, None] + np.abs(xf - mu[:, None]) * rstd[:, None] * drel) * \
        np.abs(gg) + 4 * 2.0 ** -24 * np.abs(v)
    assert mode == oracle.ROT_HADAMARD32
    vb = v.reshape(rows, K // 32, 32)
    r = oracle.rotate_blocks(v.astype(np.float32).reshape(-1, 32), mode).astype(np.float64)
    r = r.reshape(rows, K // 32, 32)
    c = 1 / np.sqrt(32.0)
    marg = c * dv.reshape(rows, K // 32, 32).sum(-1, keepdims=True) + \
        12 * 2.0 ** -24 * c * np.abs(vb).sum(-1, keepdims=True) + 2.0 ** -24 * np.abs(r)
    amax = np.abs(r).max(-1)
    mmax = marg.max(-1)
    with np.errstate(divide="ignore"):
        lo = np.floor(np.log2(np.maximum(amax - mmax, 0)))
        hi = np.floor(np.log2(amax + mmax))
    e = np.floor(np.log2(np.where(amax > 0, amax, 1))) - 2
    s = np.abs(r) * 2.0 ** -e[..., None]
    ms = marg * 2.0 ** -e[..., None]
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    near_mid = (np.min(np.abs(s[..., None] - mids), -1) <= ms).any(-1)
    near_zero = (np.abs(r) <= marg).any(-1)
    return (lo != hi) | near_mid | near_zero


@pytest.mark.parametrize("kind", [oracle.NORM_LAYER, oracle.NORM_RMS])
@pytest.mark.parametrize("rows,K", [(5, 3072), (300, 12288), (7, 24576), (3, 51200)])
def test_norm_rotate_quantize_realistic_rows(kind, rows, K):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    x, _ = synth.activation_bf16(rows + K + kind, rows, K, 0.01, 30.0)
    xb = synth.bf16_bits_to_f32(x)
    x = synth.f32_to_bf16_bits(xb * np.float32(3.0) + np.float32(1.5))  # non-zero mean
    g = _vec(1, K, 1.0, 0.2)
    b = _vec(2, K, 0.0, 0.5)
    eps = 1e-6
    q, sf, st = mx.norm_rotate_quantize(to_dev_bf16(x), kind, eps, to_dev(g), to_dev(b),
                                        oracle.ROT_HADAMARD32)
    torch.cuda.synchronize()
    st = st.cpu().numpy()
    mu_x, rstd_x = oracle.row_stats(x, kind, eps)
    dmu, drel = _stat_bounds(x, kind, K)
    assert np.all(np.abs(st[:, 0] - mu_x) <= dmu + 1e-30)
    assert np.all(np.abs(st[:, 1] - rstd_x) <= drel * rstd_x)
    mu, rstd = mu_x.astype(np.float32), rstd_x.astype(np.float32)
    q_ref, s_ref = oracle.norm_rotate_quantize(x, mu, rstd, g, b, oracle.ROT_HADAMARD32)
    open_ = _norm_open_blocks(x, mu_x, rstd_x, dmu, drel, g, b, oracle.ROT_HADAMARD32)
    got_s = oracle.sf_from_physical(sf.cpu().numpy()[: oracle.sf_bytes(rows, K)], rows, K)
    gq = oracle.unpack_codes(q.cpu().numpy()).reshape(rows, K // 32, 32)
    eq = oracle.unpack_codes(q_ref).reshape(rows, K // 32, 32)
    same = (gq == eq).all(-1) & (got_s == s_ref)
    assert same[~open_].all(), f"{(~same & ~open_).sum()} decided blocks differ"
    ds = np.abs(got_s.astype(int) - s_ref.astype(int))
    assert (ds[open_] <= 1).all()
    mag = lambda c: (c & 7).astype(int)
    step_ok = (np.abs(mag(gq) - mag(eq)) <= 1).all(-1) | (ds != 0)
    assert step_ok[open_].all()
    print(f"norm kind {kind} {rows}x{K}: {open_.sum()} of {open_.size} blocks open "
          f"({open_.mean():.1%}), {(~same).sum()} differ")


@pytest.mark.parametrize("kind", [oracle.NORM_LAYER, oracle.NORM_RMS])
@pytest.mark.parametrize("M", [16, 384])
def test_norm_linear(kind, M):
    """The layer on exact rows against the oracle's layer built from its own statistics."""
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    K, N = 4096, 1024
    eps = 2.0 ** -12
    x = _exact_rows(M + 5, M, K, kind)
    g = _vec(3, K, 1.0, 0.1)
    b = _vec(4, K, 0.0, 0.3)
    w = synth.weight_f32(4, N, K, 7)
    wq, ws = oracle.prepare_weight(w, oracle.ROT_HADAMARD32)
    y = mx.norm_linear(to_dev_bf16(x), to_dev(wq), to_dev(oracle.sf_to_physical(ws, K)), N, kind,
                       eps, to_dev(g), to_dev(b), oracle.ROT_HADAMARD32)
    torch.cuda.synchronize()
    mu, rstd = _oracle_stats_f32(x, kind, eps)
    xq, xs = oracle.norm_rotate_quantize(x, mu, rstd, g, b, oracle.ROT_HADAMARD32)
    ref, S = oracle.gemm(xq, xs, wq, ws)
    check_gemm_values(bf16_dev_to_f64(y), ref, S, "bf16", f"norm linear kind {kind} M{M}")
