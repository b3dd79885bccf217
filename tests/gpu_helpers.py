"""Helpers for the GPU parity tests: device transfers, oracle comparisons and the
tolerance rules of the block-scaled GEMM.

Tolerances (fp32 accumulation of exact FP4 products):
  fp32 output: |y - ref| <= 1e-5 * S, S = sum_i |a_i b_i| (scales included);
  bf16 output: |y - bf16(ref)| <= 1 bf16 ulp of bf16(ref), or, for elements whose
  value cancels (1e-5 * S larger than that ulp), |y - ref| <= 1e-5 * S + ulp(y) / 2.
"""
from __future__ import annotations

import numpy as np

import oracle


def torch_mod():
    import torch
    return torch


def to_dev_bf16(bits: np.ndarray):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev(a: np.ndarray):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_dev_to_f64(t) -> np.ndarray:
    torch = torch_mod()
    return t.float().cpu().numpy().astype(np.float64)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |v| (8 significant bits; subnormal spacing 2^-133)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def check_gemm_values(y: np.ndarray, ref: np.ndarray, S: np.ndarray, out: str, what: str = ""):
    """Assert the tolerance rules; returns the number of elements that needed the
    cancellation clause (bf16 only)."""
    y = np.asarray(y, np.float64)
    assert y.shape == ref.shape
    finite = np.isfinite(ref)
    assert np.array_equal(np.isfinite(y), finite), f"{what}: non-finite pattern differs"
    y, ref, S = y[finite], ref[finite], S[finite]
    if out == "f32":
        err = np.abs(y - ref)
        bad = err > 1e-5 * S
        if bad.any():
            i = np.argmax(err - 1e-5 * S)
            raise AssertionError(f"{what}: {bad.sum()} fp32 elements out of tolerance; worst "
                                 f"y={y[i]!r} ref={ref[i]!r} S={S[i]!r}")
        return 0
    r16 = oracle.bf16_round(ref)
    ok1 = np.abs(y - r16) <= bf16_ulp(r16)
    ok2 = np.abs(y - ref) <= 1e-5 * S + 0.5 * bf16_ulp(y)
    bad = ~(ok1 | ok2)
    if bad.any():
        idx = np.flatnonzero(bad)[:5]
        raise AssertionError(f"{what}: {bad.sum()} bf16 elements out of tolerance, e.g. " +
                             ", ".join(f"y={y[i]!r} ref={ref[i]!r} S={S[i]!r}" for i in idx))
    return int((~ok1 & ok2).sum())


def describe_code_mismatch(xin: np.ndarray, got_q, exp_q, got_s, exp_s, K: int, limit=3) -> str:
    """Human-readable first mismatching blocks (for debugging a failed parity run)."""
    gq = oracle.unpack_codes(got_q).reshape(got_q.shape[0], K // 32, 32)
    eq = oracle.unpack_codes(exp_q).reshape(exp_q.shape[0], K // 32, 32)
    bad = np.argwhere((gq != eq).any(axis=2) | (got_s != exp_s))
    lines = [f"{len(bad)} mismatching blocks"]
    for r, b in bad[:limit]:
        lines.append(f" row {r} block {b}: scale got {got_s[r, b]} exp {exp_s[r, b]}; "
                     f"codes got {gq[r, b].tolist()} exp {eq[r, b].tolist()}; "
                     f"x {np.asarray(xin)[r, 32 * b:32 * b + 32].tolist()}")
    return "\n".join(lines)


def quantize_parity(x: np.ndarray, mode: int, A=None, B=None, ld_pad: int = 0):
    """Run the library's rotate_quantize on x (uint16 bf16 bits or float32) and
    compare codes and scale bytes (padding included) with the oracle, bit for bit."""
    import mxfp4_quantized_linear_block_b200 as mx
    torch = torch_mod()
    rows, K = x.shape
    if ld_pad:
        big = np.zeros((rows, K + ld_pad), dtype=x.dtype)
        big[:, :K] = x
        dev_big = to_dev_bf16(big) if x.dtype == np.uint16 else to_dev(big)
        dev = dev_big[:, :K]
    else:
        dev = to_dev_bf16(x) if x.dtype == np.uint16 else to_dev(x)
    q, sf = mx.rotate_quantize(dev, mode, A, B)
    torch.cuda.synchronize()
    got_q = q.cpu().numpy()
    got_phys = sf.cpu().numpy()[: oracle.sf_bytes(rows, K)]
    exp_q, exp_s = oracle.rotate_quantize(x, mode, A, B)
    exp_phys = oracle.sf_to_physical(exp_s, K)
    got_s = oracle.sf_from_physical(got_phys, rows, K)
    if not (np.array_equal(got_q, exp_q) and np.array_equal(got_phys, exp_phys)):
        xin = synth_view(x)
        raise AssertionError(describe_code_mismatch(xin, got_q, exp_q, got_s, exp_s, K) +
                             f"\n padding bytes equal: "
                             f"{np.array_equal(got_phys, exp_phys) or np.array_equal(got_s, exp_s)}")
    return exp_q, exp_s


def synth_view(x: np.ndarray) -> np.ndarray:
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32)
    return x
