"""Python binding of libmxfp4, the MXFP4 W4A4 linear block for B200 (sm_100a).

Argument marshalling only: every step of the layer (rotation, quantisation,
block-scaled GEMM) runs in the library's CUDA kernels. PyTorch provides device
memory and the current stream. If ``libmxfp4.so`` is missing the import fails;
there is no fallback of any kind.

Functions mirror the C ABI in ``include/mxfp4.h``:
``quantize``, ``rotate_quantize``, ``gemm``, ``gemm_bias``, ``gemm_quantize``,
``linear``, ``linear_noalloc``, ``poll_status`` and
the host helpers ``sf_bytes``, ``sf_offset``, ``workspace_bytes``,
``status_string``.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmxfp4.so")

OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_ALIGN, ERR_WORKSPACE, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = range(8)
ROT_NONE, ROT_HADAMARD32, ROT_KRON_4x8, ROT_HADAMARD64, ROT_HADAMARD128 = 0, 1, 2, 3, 4
DT_BF16, DT_F32 = 0, 1
OP_QUANTIZE, OP_GEMM, OP_LINEAR, OP_NVFP4_LINEAR, OP_NORM_LINEAR = 0, 1, 2, 3, 4
NORM_LAYER, NORM_RMS = 0, 1
TEST_FAULT_NONE, TEST_FAULT_WITHHOLD_ACCUMULATOR = 0, 1
LINEAR_AUTO, LINEAR_ONE_KERNEL, LINEAR_TWO_KERNELS = 0, 1, 2

EXPORTS = (
    "mxfp4_sf_bytes", "mxfp4_sf_offset", "mxfp4_workspace_bytes", "mxfp4_status_string",
    "mxfp4_quantize", "mxfp4_rotate_quantize", "mxfp4_gemm", "mxfp4_linear",
    "mxfp4_poll_status", "mxfp4_linear_noalloc", "mxfp4_gemm_bias", "mxfp4_gemm_quantize",
    "mxfp4_nvfp4_sf_bytes", "mxfp4_nvfp4_tensor_scale", "mxfp4_nvfp4_quantize",
    "mxfp4_nvfp4_gemm", "mxfp4_nvfp4_linear", "mxfp4_norm_rotate_quantize", "mxfp4_norm_linear",
    "mxfp4_linear_kernel_count", "mxfp4_norm_linear_kernel_count",
    "mxfp4_kron_weight_factors", "mxfp4_test_set_fault", "mxfp4_set_linear_form",
    "mxfp4_nvfp4_linear_static",
)


class MXFP4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libmxfp4.so not found at {LIB_PATH}; build it with "
            "`python mxfp4_quantized_linear_block_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    sig = {
        "mxfp4_sf_bytes": ([i64, i64], sz),
        "mxfp4_sf_offset": ([i64, i64, i64], i64),
        "mxfp4_workspace_bytes": ([i32, i64, i64, i64], sz),
        "mxfp4_status_string": ([i32], ctypes.c_char_p),
        "mxfp4_quantize": ([vp, i32, i64, i64, i64, vp, vp, vp], i32),
        "mxfp4_rotate_quantize": ([vp, i32, i64, i64, i64, i32, vp, vp, vp, vp, vp], i32),
        "mxfp4_gemm": ([vp, vp, vp, vp, i64, i64, i64, vp, i32, i64, vp, sz, vp], i32),
        "mxfp4_linear": ([vp, i64, i64, i32, vp, vp, vp, vp, i64, vp, vp, sz, vp], i32),
        "mxfp4_poll_status": ([vp, vp], i32),
        "mxfp4_linear_noalloc": ([vp, i64, i64, i32, vp, vp, vp, vp, i64, vp, vp, vp], i32),
        "mxfp4_gemm_bias": ([vp, vp, vp, vp, i64, i64, i64, vp, vp, i32, i64, vp, sz, vp], i32),
        "mxfp4_gemm_quantize": ([vp, vp, vp, vp, i64, i64, i64, vp, i32, vp, vp, vp, vp, vp, sz,
                                 vp], i32),
        "mxfp4_nvfp4_sf_bytes": ([i64, i64], sz),
        "mxfp4_nvfp4_tensor_scale": ([vp, i32, i64, i64, i64, i32, vp, vp], i32),
        "mxfp4_nvfp4_quantize": ([vp, i32, i64, i64, i64, i32, vp, vp, vp, vp], i32),
        "mxfp4_nvfp4_gemm": ([vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, i32, i64, vp, sz, vp],
                             i32),
        "mxfp4_nvfp4_linear": ([vp, i64, i64, i32, vp, vp, vp, i64, vp, vp, sz, vp], i32),
        "mxfp4_nvfp4_linear_static": ([vp, i64, i64, i32, vp, vp, vp, vp, i64, vp, vp, sz, vp],
                                      i32),
        "mxfp4_norm_rotate_quantize": ([vp, i64, i64, i64, i32, ctypes.c_float, vp, vp, i32, vp,
                                        vp, vp, vp, vp, vp], i32),
        "mxfp4_norm_linear": ([vp, i64, i64, i32, ctypes.c_float, vp, vp, i32, vp, vp, vp, vp,
                               i64, vp, vp, sz, vp], i32),
        "mxfp4_linear_kernel_count": ([i64, i64, i64, i32], i32),
        "mxfp4_norm_linear_kernel_count": ([i64, i64, i64, i32], i32),
        "mxfp4_kron_weight_factors": ([vp, vp, vp, vp], i32),
        "mxfp4_test_set_fault": ([i32], i32),
        "mxfp4_set_linear_form": ([i32], i32),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


lib = _load()


# ---------------------------------------------------------------- host helpers

def sf_bytes(rows: int, K: int) -> int:
    return lib.mxfp4_sf_bytes(rows, K)


def sf_offset(row: int, kblock: int, K: int) -> int:
    return lib.mxfp4_sf_offset(row, kblock, K)


def workspace_bytes(op: int, M: int, N: int, K: int) -> int:
    return lib.mxfp4_workspace_bytes(op, M, N, K)


def status_string(status: int) -> str:
    return lib.mxfp4_status_string(status).decode()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise MXFP4Error(status, where)


# ---------------------------------------------------------------- device calls

def _torch():
    import torch
    return torch


def _stream_handle(stream) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _host_f32(a, n: int):
    """Host float32 copy of a small matrix (Kronecker factor) as a ctypes array."""
    if a is None:
        return None
    try:
        import numpy as np
        arr = np.ascontiguousarray(a.detach().cpu().numpy() if hasattr(a, "detach") else a,
                                   dtype=np.float32).reshape(-1)
    except Exception as e:  # pragma: no cover
        raise TypeError(f"Kronecker factor: {e}")
    if arr.size != n:
        raise ValueError(f"Kronecker factor must have {n} entries, got {arr.size}")
    return (ctypes.c_float * n)(*arr.tolist())


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return DT_BF16
    if t.dtype == torch.float32:
        return DT_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def new_workspace(nbytes: int, device=None):
    """Zero-initialised device workspace (the status word starts cleared)."""
    torch = _torch()
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def rotate_quantize(x, mode: int = ROT_HADAMARD32, kron_a=None, kron_b=None, q=None, sf=None,
                    stream=None):
    """x: [rows, K] bf16/fp32 CUDA tensor (row stride x.stride(0)) ->
    (q [rows, K/2] uint8 packed E2M1, sf [sf_bytes] uint8 scales in the tensor-core layout)."""
    torch = _torch()
    assert x.dim() == 2 and x.stride(1) == 1, "x must be row-major 2-D"
    rows, K = x.shape
    if q is None:
        q = torch.empty((rows, K // 2), dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty(max(sf_bytes(rows, K), 16), dtype=torch.uint8, device=x.device)
    a = _host_f32(kron_a, 16) if mode == ROT_KRON_4x8 else None
    b = _host_f32(kron_b, 64) if mode == ROT_KRON_4x8 else None
    st = lib.mxfp4_rotate_quantize(x.data_ptr(), _dtype_code(x), rows, K, x.stride(0), mode, a, b,
                                   q.data_ptr(), sf.data_ptr(), _stream_handle(stream))
    _check(st, "mxfp4_rotate_quantize")
    return q, sf


def quantize(x, q=None, sf=None, stream=None):
    """Plain MXFP4 quantisation (no rotation)."""
    return rotate_quantize(x, ROT_NONE, None, None, q, sf, stream)


def gemm(aq, asf, bq, bsf, M: int, N: int, K: int, y=None, out_dtype=None, ws=None, stream=None):
    """Block-scaled GEMM y[M, N] = A . B^T on the tensor cores (fp32 accumulate)."""
    torch = _torch()
    out_dtype = out_dtype or torch.bfloat16
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=aq.device)
    if ws is None:
        ws = new_workspace(workspace_bytes(OP_GEMM, M, N, K), aq.device)
    st = lib.mxfp4_gemm(aq.data_ptr(), asf.data_ptr(), bq.data_ptr(), bsf.data_ptr(), M, N, K,
                        y.data_ptr(), _dtype_code(y), y.stride(0), ws.data_ptr(), ws.numel(),
                        _stream_handle(stream))
    _check(st, "mxfp4_gemm")
    return y


def gemm_bias(aq, asf, bq, bsf, M: int, N: int, K: int, bias, y=None, out_dtype=None, ws=None,
              stream=None):
    """y = A . B^T + bias (bias: fp32 CUDA tensor [N], added once in fp32)."""
    torch = _torch()
    out_dtype = out_dtype or torch.bfloat16
    assert bias.dtype == torch.float32 and bias.numel() == N and bias.is_contiguous()
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=aq.device)
    if ws is None:
        ws = new_workspace(workspace_bytes(OP_GEMM, M, N, K), aq.device)
    st = lib.mxfp4_gemm_bias(aq.data_ptr(), asf.data_ptr(), bq.data_ptr(), bsf.data_ptr(), M, N,
                             K, bias.data_ptr(), y.data_ptr(), _dtype_code(y), y.stride(0),
                             ws.data_ptr(), ws.numel(), _stream_handle(stream))
    _check(st, "mxfp4_gemm_bias")
    return y


def gemm_quantize(aq, asf, bq, bsf, M: int, N: int, K: int, bias=None,
                  mode: int = ROT_HADAMARD32, kron_a=None, kron_b=None, yq=None, ysf=None,
                  ws=None, stream=None):
    """GEMM whose output is MXFP4, ready as the next layer's activation operand:
    (A . B^T + bias) with each 32-column block rotated (mode) and quantised.
    Returns (yq [M, N/2] uint8, ysf [sf_bytes(M, N)] uint8)."""
    torch = _torch()
    dev = aq.device
    if yq is None:
        yq = torch.empty((M, N // 2), dtype=torch.uint8, device=dev)
    if ysf is None:
        ysf = torch.empty(sf_bytes(M, N), dtype=torch.uint8, device=dev)
    if ws is None:
        ws = new_workspace(workspace_bytes(OP_GEMM, M, N, K), dev)
    a = _host_f32(kron_a, 16) if mode == ROT_KRON_4x8 else None
    b = _host_f32(kron_b, 64) if mode == ROT_KRON_4x8 else None
    st = lib.mxfp4_gemm_quantize(aq.data_ptr(), asf.data_ptr(), bq.data_ptr(), bsf.data_ptr(), M,
                                 N, K, bias.data_ptr() if bias is not None else None, mode, a, b,
                                 yq.data_ptr(), ysf.data_ptr(), ws.data_ptr(), ws.numel(),
                                 _stream_handle(stream))
    _check(st, "mxfp4_gemm_quantize")
    return yq, ysf


# ---------------------------------------------------------------- norm prologue

def norm_rotate_quantize(x, kind: int = NORM_LAYER, eps: float = 1e-6, g=None, b=None,
                         mode: int = ROT_HADAMARD32, kron_a=None, kron_b=None, q=None, sf=None,
                         stats=None, stream=None):
    """Normalise each bf16 row (LayerNorm / RMSNorm statistics, then * g + b), rotate and
    quantise. Returns (q, sf, stats [rows, 2] fp32: mu, rstd)."""
    torch = _torch()
    assert x.dim() == 2 and x.stride(1) == 1 and x.dtype == torch.bfloat16
    rows, K = x.shape
    if q is None:
        q = torch.empty((rows, K // 2), dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty(max(sf_bytes(rows, K), 16), dtype=torch.uint8, device=x.device)
    if stats is None:
        stats = torch.empty((rows, 2), dtype=torch.float32, device=x.device)
    a = _host_f32(kron_a, 16) if mode == ROT_KRON_4x8 else None
    bb = _host_f32(kron_b, 64) if mode == ROT_KRON_4x8 else None
    st = lib.mxfp4_norm_rotate_quantize(x.data_ptr(), rows, K, x.stride(0), kind, eps,
                                        g.data_ptr() if g is not None else None,
                                        b.data_ptr() if b is not None else None, mode, a, bb,
                                        q.data_ptr(), sf.data_ptr(), stats.data_ptr(),
                                        _stream_handle(stream))
    _check(st, "mxfp4_norm_rotate_quantize")
    return q, sf, stats


def norm_linear(x, wq, wsf, N: int, kind: int = NORM_LAYER, eps: float = 1e-6, g=None, b=None,
                mode: int = ROT_HADAMARD32, kron_a=None, kron_b=None, y=None, ws=None,
                stream=None):
    """The layer with the norm prologue (bf16 x in, bf16 y out)."""
    torch = _torch()
    assert x.dim() == 2 and x.is_contiguous() and x.dtype == torch.bfloat16
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = new_workspace(workspace_bytes(OP_NORM_LINEAR, M, N, K), x.device)
    a = _host_f32(kron_a, 16) if mode == ROT_KRON_4x8 else None
    bb = _host_f32(kron_b, 64) if mode == ROT_KRON_4x8 else None
    st = lib.mxfp4_norm_linear(x.data_ptr(), M, K, kind, eps,
                               g.data_ptr() if g is not None else None,
                               b.data_ptr() if b is not None else None, mode, a, bb,
                               wq.data_ptr(), wsf.data_ptr(), N, y.data_ptr(), ws.data_ptr(),
                               ws.numel(), _stream_handle(stream))
    _check(st, "mxfp4_norm_linear")
    return y


# ---------------------------------------------------------------- NVFP4

def nvfp4_sf_bytes(rows: int, K: int) -> int:
    return lib.mxfp4_nvfp4_sf_bytes(rows, K)


def nvfp4_tensor_scale(x, mode: int = ROT_NONE, scale2=None, stream=None):
    """Device fp32 tensor scale amax(rotated x) / 2688; returns a 2-float CUDA tensor whose
    element 0 is the scale."""
    torch = _torch()
    assert x.dim() == 2 and x.stride(1) == 1
    rows, K = x.shape
    if scale2 is None:
        scale2 = torch.zeros(2, dtype=torch.float32, device=x.device)
    st = lib.mxfp4_nvfp4_tensor_scale(x.data_ptr(), _dtype_code(x), rows, K, x.stride(0), mode,
                                      scale2.data_ptr(), _stream_handle(stream))
    _check(st, "mxfp4_nvfp4_tensor_scale")
    return scale2


def nvfp4_quantize(x, tensor_scale, mode: int = ROT_NONE, q=None, sf=None, stream=None):
    """x [rows, K] bf16/fp32 -> (q [rows, K/2], sf [nvfp4_sf_bytes]) with the device fp32
    tensor scale (a CUDA tensor whose first element is the scale)."""
    torch = _torch()
    assert x.dim() == 2 and x.stride(1) == 1
    rows, K = x.shape
    if q is None:
        q = torch.empty((rows, K // 2), dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty(max(nvfp4_sf_bytes(rows, K), 16), dtype=torch.uint8, device=x.device)
    st = lib.mxfp4_nvfp4_quantize(x.data_ptr(), _dtype_code(x), rows, K, x.stride(0), mode,
                                  tensor_scale.data_ptr(), q.data_ptr(), sf.data_ptr(),
                                  _stream_handle(stream))
    _check(st, "mxfp4_nvfp4_quantize")
    return q, sf


def nvfp4_gemm(aq, asf, a_scale, bq, bsf, b_scale, M: int, N: int, K: int, y=None,
               out_dtype=None, ws=None, stream=None):
    """NVFP4 GEMM y = a_scale * b_scale * A . B^T (scales: device fp32 tensors)."""
    torch = _torch()
    out_dtype = out_dtype or torch.bfloat16
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=aq.device)
    if ws is None:
        ws = new_workspace(workspace_bytes(OP_GEMM, M, N, K), aq.device)
    st = lib.mxfp4_nvfp4_gemm(aq.data_ptr(), asf.data_ptr(), a_scale.data_ptr(), bq.data_ptr(),
                              bsf.data_ptr(), b_scale.data_ptr(), M, N, K, y.data_ptr(),
                              _dtype_code(y), y.stride(0), ws.data_ptr(), ws.numel(),
                              _stream_handle(stream))
    _check(st, "mxfp4_nvfp4_gemm")
    return y


def nvfp4_linear(x, wq, wsf, w_scale, N: int, mode: int = ROT_NONE, y=None, ws=None,
                 stream=None):
    """The NVFP4 layer: tensor scale + quantise x, GEMM with NVFP4 weights (bf16 out)."""
    torch = _torch()
    assert x.dim() == 2 and x.is_contiguous() and x.dtype == torch.bfloat16
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = new_workspace(workspace_bytes(OP_NVFP4_LINEAR, M, N, K), x.device)
    st = lib.mxfp4_nvfp4_linear(x.data_ptr(), M, K, mode, wq.data_ptr(), wsf.data_ptr(),
                                w_scale.data_ptr(), N, y.data_ptr(), ws.data_ptr(), ws.numel(),
                                _stream_handle(stream))
    _check(st, "mxfp4_nvfp4_linear")
    return y


def nvfp4_linear_static(x, x_scale, wq, wsf, w_scale, N: int, mode: int = ROT_NONE, y=None,
                        ws=None, stream=None):
    """The NVFP4 layer with a static activation tensor scale (x_scale: a device fp32 tensor
    whose first element is the scale): quantise x with it, GEMM (bf16 out); two kernels."""
    torch = _torch()
    assert x.dim() == 2 and x.is_contiguous() and x.dtype == torch.bfloat16
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = new_workspace(workspace_bytes(OP_NVFP4_LINEAR, M, N, K), x.device)
    st = lib.mxfp4_nvfp4_linear_static(x.data_ptr(), M, K, mode, x_scale.data_ptr(),
                                       wq.data_ptr(), wsf.data_ptr(), w_scale.data_ptr(), N,
                                       y.data_ptr(), ws.data_ptr(), ws.numel(),
                                       _stream_handle(stream))
    _check(st, "mxfp4_nvfp4_linear_static")
    return y


def linear(x, wq, wsf, N: int, mode: int = ROT_HADAMARD32, kron_a=None, kron_b=None, y=None,
           ws=None, stream=None):
    """The whole layer: y[M, N] (bf16) = MXFP4(rotate(x)) . W^T with pre-quantised W."""
    torch = _torch()
    assert x.dim() == 2 and x.is_contiguous() and x.dtype == torch.bfloat16
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = new_workspace(workspace_bytes(OP_LINEAR, M, N, K), x.device)
    a = _host_f32(kron_a, 16) if mode == ROT_KRON_4x8 else None
    b = _host_f32(kron_b, 64) if mode == ROT_KRON_4x8 else None
    st = lib.mxfp4_linear(x.data_ptr(), M, K, mode, a, b, wq.data_ptr(), wsf.data_ptr(), N,
                          y.data_ptr(), ws.data_ptr(), ws.numel(), _stream_handle(stream))
    _check(st, "mxfp4_linear")
    return y


def linear_noalloc(x, wq, wsf, N: int, mode: int = ROT_HADAMARD32, kron_a=None, kron_b=None,
                   y=None, status=None, stream=None):
    """The layer without a workspace, for callers that cannot allocate device memory at
    call time: the quantised activations go to a fixed 32 MiB array inside the library
    (see mxfp4_linear_noalloc in include/mxfp4.h for the size limit and the sharing
    rules). `status`: optional zeroed int32 CUDA tensor that receives a timeout code."""
    torch = _torch()
    assert x.dim() == 2 and x.is_contiguous() and x.dtype == torch.bfloat16
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    a = _host_f32(kron_a, 16) if mode == ROT_KRON_4x8 else None
    b = _host_f32(kron_b, 64) if mode == ROT_KRON_4x8 else None
    st = lib.mxfp4_linear_noalloc(x.data_ptr(), M, K, mode, a, b, wq.data_ptr(), wsf.data_ptr(),
                                  N, y.data_ptr(), status.data_ptr() if status is not None else None,
                                  _stream_handle(stream))
    _check(st, "mxfp4_linear_noalloc")
    return y


def linear_kernel_count(M: int, N: int, K: int, mode: int = ROT_HADAMARD32) -> int:
    """Kernels that linear() launches for these sizes: 1 (x quantised inside the GEMM's
    CTAs), 2 (quantiser + GEMM), 0 (M == 0); -1 for arguments linear() rejects."""
    return int(lib.mxfp4_linear_kernel_count(M, N, K, mode))


def norm_linear_kernel_count(M: int, N: int, K: int, mode: int = ROT_HADAMARD32) -> int:
    """Kernels that norm_linear() launches: 2 (one-pass norm quantiser + GEMM, K <= 51168),
    3 (row statistics + quantiser + GEMM), 0 (M == 0); -1 for arguments it rejects."""
    return int(lib.mxfp4_norm_linear_kernel_count(M, N, K, mode))


def poll_status(ws) -> int:
    out = ctypes.c_int(0)
    _check(lib.mxfp4_poll_status(ws.data_ptr(), ctypes.byref(out)), "mxfp4_poll_status")
    return out.value


def kron_weight_factors(A, B):
    """Weight-side factors of the Kronecker mode, (A^-T, B^-T) as float32 arrays, from
    mxfp4_kron_weight_factors (double Gauss-Jordan inverses, rounded once to fp32)."""
    import numpy as np
    A = np.ascontiguousarray(A, dtype=np.float32)
    B = np.ascontiguousarray(B, dtype=np.float32)
    assert A.shape == (4, 4) and B.shape == (8, 8)
    At = np.empty((4, 4), dtype=np.float32)
    Bt = np.empty((8, 8), dtype=np.float32)
    _check(lib.mxfp4_kron_weight_factors(A.ctypes.data, B.ctypes.data, At.ctypes.data,
                                         Bt.ctypes.data), "mxfp4_kron_weight_factors")
    return At, Bt


def set_linear_form(form: int) -> None:
    """Which form linear() / linear_noalloc() take where they have a choice (LINEAR_AUTO,
    LINEAR_ONE_KERNEL, LINEAR_TWO_KERNELS); see mxfp4_set_linear_form in include/mxfp4.h."""
    _check(lib.mxfp4_set_linear_form(form), "mxfp4_set_linear_form")


def test_set_fault(fault: int) -> None:
    """Testing only: make later GEMM launches simulate `fault` (TEST_FAULT_*); see
    mxfp4_test_set_fault in include/mxfp4.h."""
    _check(lib.mxfp4_test_set_fault(fault), "mxfp4_test_set_fault")
