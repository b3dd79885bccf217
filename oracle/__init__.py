"""CPU oracle for the MXFP4 W4A4 linear block (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It is plain C (``mxfp4_oracle.c``,
compiled with gcc, OpenMP over rows) behind numpy wrappers, and shares nothing
with the CUDA library: its own formats, rotations, scale rule, packing,
contraction and scale-factor layout map.

Pinned by ``tests/test_oracle_*.py`` against the E2M1 value set, all tie
cases, exact round trips, H.H^T = I, (A(x)B)(A^-1(x)B^-1) = I, explicit
matrix products and brute-force dequantised dot products.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_oracle.so")
_lib = None

ROT_NONE, ROT_HADAMARD32, ROT_KRON_4x8, ROT_HADAMARD64, ROT_HADAMARD128 = 0, 1, 2, 3, 4


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "mxfp4_oracle.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", src, "-o", _SO, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        vp, i64, i32, dbl, flt = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                  ctypes.c_double, ctypes.c_float)
        sig = {
            "oracle_e2m1_value": ([i32], dbl),
            "oracle_e8m0_value": ([i32], dbl),
            "oracle_e2m1_code": ([dbl], i32),
            "oracle_e2m1_code_array": ([vp, i64, vp], None),
            "oracle_floor_log2_f32": ([flt], i32),
            "oracle_scale_exponent": ([flt], i32),
            "oracle_quantize_block": ([vp, vp, vp], None),
            "oracle_inv_sqrt32": ([], flt),
            "oracle_fwht32_unnormalised": ([vp, vp], None),
            "oracle_hadamard32": ([vp, vp], None),
            "oracle_kron32": ([vp, vp, vp, vp], None),
            "oracle_rotate_blocks": ([vp, i64, i32, vp, vp, vp], None),
            "oracle_quantize_blocks": ([vp, i64, vp, vp], None),
            "oracle_rotate_quantize": ([vp, i32, i64, i64, i64, i32, vp, vp, vp, vp], None),
            "oracle_fwht_unnormalised": ([vp, i32, vp], None),
            "oracle_hadamard_n": ([vp, i32, vp], None),
            "oracle_rotation_span": ([i32], i32),
            "oracle_e4m3_value": ([i32], dbl),
            "oracle_e4m3_code": ([dbl], i32),
            "oracle_nvfp4_quantize_group": ([vp, ctypes.c_float, vp, vp], None),
            "oracle_nvfp4_tensor_scale": ([vp, i32, i64, i64, i64, i32], ctypes.c_float),
            "oracle_nvfp4_rotate_quantize": ([vp, i32, i64, i64, i64, i32, ctypes.c_float, vp,
                                              vp], None),
            "oracle_nvfp4_gemm": ([vp, vp, vp, vp, i64, i64, i64, dbl, vp, vp], None),
            "oracle_row_stats": ([vp, i32, i64, i64, i64, i32, dbl, vp, vp], None),
            "oracle_norm_rotate_quantize": ([vp, i32, i64, i64, i64, vp, vp, vp, vp, i32, vp,
                                             vp, vp, vp], None),
            "oracle_dequantize": ([vp, vp, i64, i64, vp], None),
            "oracle_gemm_pairs": ([vp, vp, vp, vp, i64, vp, vp, i64, vp, vp], None),
            "oracle_gemm": ([vp, vp, vp, vp, i64, i64, i64, vp, vp], None),
            "oracle_bf16_round": ([dbl], dbl),
            "oracle_bf16_round_array": ([vp, i64, vp], None),
            "oracle_inverse": ([vp, i32, vp], i32),
            "oracle_kron_weight_factors": ([vp, vp, vp, vp], i32),
            "oracle_sf_bytes": ([i64, i64], i64),
            "oracle_sf_offset": ([i64, i64, i64], i64),
            "oracle_sf_to_physical": ([vp, i64, i64, vp], None),
            "oracle_sf_from_physical": ([vp, i64, i64, vp], None),
        }
        for name, (args, res) in sig.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        _lib = lib
    return _lib


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- scalar formats

def e2m1_value(code: int) -> float:
    return _load().oracle_e2m1_value(int(code))


def e8m0_value(byte: int) -> float:
    return _load().oracle_e8m0_value(int(byte))


def e2m1_code(s: float) -> int:
    return _load().oracle_e2m1_code(float(s))


def e2m1_codes(s: np.ndarray) -> np.ndarray:
    s = _c(s, np.float64)
    out = np.empty(s.shape, dtype=np.uint8)
    _load().oracle_e2m1_code_array(_p(s), s.size, _p(out))
    return out


def floor_log2_f32(a: float) -> int:
    return _load().oracle_floor_log2_f32(float(np.float32(a)))


def scale_exponent(amax: float) -> int:
    return _load().oracle_scale_exponent(float(np.float32(amax)))


def inv_sqrt32() -> np.float32:
    return np.float32(_load().oracle_inv_sqrt32())


# ---------------------------------------------------------------- blocks

def quantize_blocks(y: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """y: (..., 32) fp32 -> (codes (..., 32) uint8 unpacked, scale bytes (...))."""
    y = _c(y, np.float32)
    assert y.shape[-1] == 32
    n = y.size // 32
    codes = np.empty(y.shape, dtype=np.uint8)
    scales = np.empty(y.shape[:-1], dtype=np.uint8)
    _load().oracle_quantize_blocks(_p(y), n, _p(codes), _p(scales))
    return codes, scales


def fwht32_unnormalised(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(32, dtype=np.float32)
    _load().oracle_fwht32_unnormalised(_p(x), _p(out))
    return out


def rotate_blocks(x: np.ndarray, mode: int, A=None, B=None) -> np.ndarray:
    """Rotate every 32-block (last axis 32) in fp32: mode 0 none, 1 Hadamard, 2 Kronecker."""
    x = _c(x, np.float32)
    assert x.shape[-1] == 32
    A = _c(A if A is not None else np.eye(4), np.float32)
    B = _c(B if B is not None else np.eye(8), np.float32)
    y = np.empty_like(x)
    _load().oracle_rotate_blocks(_p(x), x.size // 32, int(mode), _p(A), _p(B), _p(y))
    return y


# ---------------------------------------------------------------- matrices

def rotation_span(mode: int) -> int:
    """Elements per rotation group: 32, or 64 / 128 for the larger Hadamard modes."""
    return _load().oracle_rotation_span(int(mode))


def fwht_unnormalised(x: np.ndarray) -> np.ndarray:
    """Unnormalised fp32 Walsh-Hadamard butterfly over the last axis (n = 32, 64 or 128)."""
    x = _c(x, np.float32)
    n = x.shape[-1]
    flat = x.reshape(-1, n)
    out = np.empty_like(flat)
    for i in range(flat.shape[0]):
        _load().oracle_fwht_unnormalised(_p(flat[i]), n, _p(out[i]))
    return out.reshape(x.shape)


def hadamard_n(x: np.ndarray) -> np.ndarray:
    """Normalised Sylvester Hadamard H_n (n = 32, 64 or 128) of every row, in fp32."""
    x = _c(x, np.float32)
    n = x.shape[-1]
    flat = x.reshape(-1, n)
    out = np.empty_like(flat)
    for i in range(flat.shape[0]):
        _load().oracle_hadamard_n(_p(flat[i]), n, _p(out[i]))
    return out.reshape(x.shape)


def rotate_quantize(x: np.ndarray, mode: int, A=None, B=None, bf16: bool | None = None):
    """x[rows, K] (uint16 bf16 bits or float32) -> (q[rows, K/2], s[rows, K/32]) logical layout."""
    if bf16 is None:
        bf16 = x.dtype == np.uint16
    x = _c(x, np.uint16 if bf16 else np.float32)
    rows, K = x.shape
    assert K % rotation_span(mode) == 0
    A = _c(A if A is not None else np.eye(4), np.float32)
    B = _c(B if B is not None else np.eye(8), np.float32)
    q = np.empty((rows, K // 2), dtype=np.uint8)
    s = np.empty((rows, K // 32), dtype=np.uint8)
    _load().oracle_rotate_quantize(_p(x), 0 if bf16 else 1, rows, K, K, int(mode), _p(A), _p(B),
                                   _p(q), _p(s))
    return q, s


def dequantize(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    q = _c(q, np.uint8)
    s = _c(s, np.uint8)
    rows, K = q.shape[0], q.shape[1] * 2
    out = np.empty((rows, K), dtype=np.float64)
    _load().oracle_dequantize(_p(q), _p(s), rows, K, _p(out))
    return out


def gemm_pairs(aq, as_, bq, bs, m_idx, n_idx):
    """Exact block-scaled dot products for (m, n) pairs -> (ref, S) float64."""
    aq, as_, bq, bs = (_c(t, np.uint8) for t in (aq, as_, bq, bs))
    K = aq.shape[1] * 2
    assert bq.shape[1] * 2 == K
    m_idx = _c(m_idx, np.int64)
    n_idx = _c(n_idx, np.int64)
    ref = np.empty(m_idx.size, dtype=np.float64)
    S = np.empty(m_idx.size, dtype=np.float64)
    _load().oracle_gemm_pairs(_p(aq), _p(as_), _p(bq), _p(bs), K, _p(m_idx), _p(n_idx),
                              m_idx.size, _p(ref), _p(S))
    return ref, S


def gemm(aq, as_, bq, bs):
    """Full exact product ref[M, N] and magnitude S[M, N]."""
    aq, as_, bq, bs = (_c(t, np.uint8) for t in (aq, as_, bq, bs))
    M, N, K = aq.shape[0], bq.shape[0], aq.shape[1] * 2
    ref = np.empty((M, N), dtype=np.float64)
    S = np.empty((M, N), dtype=np.float64)
    _load().oracle_gemm(_p(aq), _p(as_), _p(bq), _p(bs), M, N, K, _p(ref), _p(S))
    return ref, S


def linear(x_bf16: np.ndarray, wq, ws, mode: int, A=None, B=None):
    """The whole layer: rotate+quantise X, then the exact block-scaled product with W."""
    xq, xs = rotate_quantize(x_bf16, mode, A, B, bf16=True)
    ref, S = gemm(xq, xs, wq, ws)
    return ref, S, xq, xs


def quantize_output(y_f32: np.ndarray, bias, mode: int, A=None, B=None):
    """MXFP4 output of a layer (no bf16 round trip between layers, "AMD Quark delivers
    MXFP4 quantization for FLUX.1-dev on Instinct MI350 with 1.92x speedup", opening
    section): y + bias in fp32 (one rounding), then each 32-column block of every row
    rotated and quantised exactly like activations. y_f32 is the fp32 accumulator the
    quantisation decisions are taken from."""
    y = _c(y_f32, np.float32)
    if bias is not None:
        y = (y + _c(bias, np.float32)[None, :]).astype(np.float32)
    return rotate_quantize(y, mode, A, B, bf16=False)


def prepare_weight(w_f32: np.ndarray, mode: int, A=None, B=None):
    """Offline weight preparation: rotate each 32-block of W (H, or T^-T for Kronecker), quantise."""
    if mode == ROT_KRON_4x8:
        At, Bt = kron_weight_factors(A, B)
        return rotate_quantize(w_f32, mode, At, Bt, bf16=False)
    return rotate_quantize(w_f32, mode, None, None, bf16=False)


# ---------------------------------------------------------------- norm prologue

NORM_LAYER, NORM_RMS = 0, 1


def row_stats(x: np.ndarray, kind: int, eps: float, bf16: bool | None = None):
    """Exact-arithmetic row statistics in double: (mu, rstd) per row (LayerNorm: mean and
    1 / sqrt(var + eps); RMSNorm: 0 and 1 / sqrt(mean(x^2) + eps))."""
    if bf16 is None:
        bf16 = x.dtype == np.uint16
    x = _c(x, np.uint16 if bf16 else np.float32)
    rows, K = x.shape
    mu = np.empty(rows, np.float64)
    rstd = np.empty(rows, np.float64)
    _load().oracle_row_stats(_p(x), 0 if bf16 else 1, rows, K, K, int(kind), float(eps), _p(mu),
                             _p(rstd))
    return mu, rstd


def norm_rotate_quantize(x: np.ndarray, mu_f32, rstd_f32, g, b, mode: int, A=None, B=None,
                         bf16: bool | None = None):
    """v = ((x - mu) * rstd) * g + b in fp32 with the given fp32 statistics, then
    rotate-quantise like rotate_quantize (modes 0, 1, 2)."""
    if bf16 is None:
        bf16 = x.dtype == np.uint16
    x = _c(x, np.uint16 if bf16 else np.float32)
    rows, K = x.shape
    mu = _c(mu_f32, np.float32)
    rs = _c(rstd_f32, np.float32)
    gg = _c(g, np.float32) if g is not None else None
    bb = _c(b, np.float32) if b is not None else None
    A = _c(A if A is not None else np.eye(4), np.float32)
    B = _c(B if B is not None else np.eye(8), np.float32)
    q = np.empty((rows, K // 2), np.uint8)
    s = np.empty((rows, K // 32), np.uint8)
    _load().oracle_norm_rotate_quantize(_p(x), 0 if bf16 else 1, rows, K, K, _p(mu), _p(rs),
                                        _p(gg) if gg is not None else None,
                                        _p(bb) if bb is not None else None, int(mode), _p(A),
                                        _p(B), _p(q), _p(s))
    return q, s


# ---------------------------------------------------------------- NVFP4

def e4m3_value(byte: int) -> float:
    """Unsigned E4M3 group-scale byte (0..126) -> value."""
    return _load().oracle_e4m3_value(int(byte))


def e4m3_code(v: float) -> int:
    """Nearest finite E4M3 code to v >= 0 (ties to even, above 448 -> 448)."""
    return _load().oracle_e4m3_code(float(v))


def nvfp4_quantize_group(y: np.ndarray, st: float):
    """16 fp32 values, fp32 tensor scale -> (16 unpacked codes, E4M3 group byte)."""
    y = _c(y, np.float32)
    assert y.shape == (16,)
    codes = np.empty(16, np.uint8)
    sb = np.empty(1, np.uint8)
    _load().oracle_nvfp4_quantize_group(_p(y), float(np.float32(st)), _p(codes), _p(sb))
    return codes, int(sb[0])


def nvfp4_tensor_scale(x: np.ndarray, mode: int, bf16: bool | None = None) -> np.float32:
    """amax of x rotated by mode (0 or 1) / (6 * 448), fp32."""
    if bf16 is None:
        bf16 = x.dtype == np.uint16
    x = _c(x, np.uint16 if bf16 else np.float32)
    rows, K = x.shape
    return np.float32(_load().oracle_nvfp4_tensor_scale(_p(x), 0 if bf16 else 1, rows, K, K,
                                                        int(mode)))


def nvfp4_rotate_quantize(x: np.ndarray, mode: int, st, bf16: bool | None = None):
    """x[rows, K] -> (q[rows, K/2] packed codes, s[rows, K/16] E4M3 group bytes)."""
    if bf16 is None:
        bf16 = x.dtype == np.uint16
    x = _c(x, np.uint16 if bf16 else np.float32)
    rows, K = x.shape
    assert K % 32 == 0 and mode in (ROT_NONE, ROT_HADAMARD32)
    q = np.empty((rows, K // 2), np.uint8)
    s = np.empty((rows, K // 16), np.uint8)
    _load().oracle_nvfp4_rotate_quantize(_p(x), 0 if bf16 else 1, rows, K, K, int(mode),
                                         float(np.float32(st)), _p(q), _p(s))
    return q, s


def nvfp4_gemm(aq, as_, bq, bs, alpha: float):
    """Exact NVFP4 product times alpha (the product of the two tensor scales) -> (ref, S)."""
    aq, as_, bq, bs = (_c(a, np.uint8) for a in (aq, as_, bq, bs))
    M, N, K = aq.shape[0], bq.shape[0], aq.shape[1] * 2
    ref = np.empty((M, N), np.float64)
    S = np.empty((M, N), np.float64)
    _load().oracle_nvfp4_gemm(_p(aq), _p(as_), _p(bq), _p(bs), M, N, K, float(alpha), _p(ref),
                              _p(S))
    return ref, S


def nvfp4_dequantize(q: np.ndarray, s: np.ndarray, st) -> np.ndarray:
    """NVFP4 matrix back to double: code value * E4M3(group byte) * st."""
    codes = unpack_codes(q).astype(np.int64)
    mag = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)[codes & 7]
    val = np.where(codes & 8, -mag, mag)
    sc = np.vectorize(e4m3_value)(s.astype(np.int64))
    return val * np.repeat(sc, 16, axis=1) * float(st)


def nvfp4_sf_to_physical(s: np.ndarray, K: int) -> np.ndarray:
    """Logical [rows, K/16] E4M3 bytes -> the tensor-core layout: the same 512-byte atoms
    as the MXFP4 scales with 16-element groups in place of 32-element blocks (so the map
    of an operand with 2K elements per row)."""
    return sf_to_physical(s, 2 * K)


def nvfp4_sf_bytes(rows: int, K: int) -> int:
    return sf_bytes(rows, 2 * K)


# ---------------------------------------------------------------- helpers

def bf16_round(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float64)
    out = np.empty_like(x)
    _load().oracle_bf16_round_array(_p(x), x.size, _p(out))
    return out


def inverse(A: np.ndarray) -> np.ndarray:
    A = _c(A, np.float64)
    n = A.shape[0]
    out = np.empty_like(A)
    if _load().oracle_inverse(_p(A), n, _p(out)) != 0:
        raise ValueError("singular matrix")
    return out


def kron_weight_factors(A, B):
    A = _c(A, np.float32)
    B = _c(B, np.float32)
    At = np.empty((4, 4), dtype=np.float32)
    Bt = np.empty((8, 8), dtype=np.float32)
    if _load().oracle_kron_weight_factors(_p(A), _p(B), _p(At), _p(Bt)) != 0:
        raise ValueError("singular Kronecker factor")
    return At, Bt


def sf_bytes(rows: int, K: int) -> int:
    return _load().oracle_sf_bytes(rows, K)


def sf_offset(row: int, kb: int, K: int) -> int:
    return _load().oracle_sf_offset(row, kb, K)


def sf_to_physical(s: np.ndarray, K: int) -> np.ndarray:
    s = _c(s, np.uint8)
    rows = s.shape[0]
    out = np.empty(sf_bytes(rows, K), dtype=np.uint8)
    _load().oracle_sf_to_physical(_p(s), rows, K, _p(out))
    return out


def sf_from_physical(phys: np.ndarray, rows: int, K: int) -> np.ndarray:
    phys = _c(phys, np.uint8)
    out = np.empty((rows, K // 32), dtype=np.uint8)
    _load().oracle_sf_from_physical(_p(phys), rows, K, _p(out))
    return out


def unpack_codes(q: np.ndarray) -> np.ndarray:
    """Packed [rows, K/2] -> unpacked [rows, K] codes (element 2j = low nibble of byte j)."""
    q = _c(q, np.uint8)
    out = np.empty((q.shape[0], q.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = q & 15
    out[:, 1::2] = q >> 4
    return out
