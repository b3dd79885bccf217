"""Seeded synthetic inputs for the MXFP4 W4A4 linear layer.

This module draws numbers and describes workloads; it contains none of the
layer's arithmetic, so both the CPU oracle and the CUDA path may take their
inputs from it. The generator is counter-based (splitmix64) and written in C
(``synth.c``); every element is a pure function of (seed, tensor id, index),
so results do not depend on thread count.

Workload recipes (``WORKLOADS``) stand in for the activations and weights of
the pages' models (FLUX.1-dev DiT blocks, Llama-class MLPs): no dataset or
checkpoint is used. Activations are N(0,1) with a fraction of K-channels
scaled up (outlier channels), rounded to bf16; weights are N(0, 0.02^2) fp32.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_synth.so")
_lib = None

# Stream ids, one per tensor role, so tensors of one workload never share draws.
TID_X = 1
TID_X_OUTLIERS = 2
TID_W = 10          # + layer index
TID_KRON_A = 20
TID_KRON_B = 21
TID_CODES = 30      # + operand index
TID_SCALES = 40     # + operand index


def build(force: bool = False) -> str:
    """Compile ``synth.c`` into ``_synth.so`` next to it (gcc, OpenMP)."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               src, "-o", _SO, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        u64, i64, i32, dbl = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        vp = ctypes.c_void_p
        lib.synth_raw_u64.argtypes = [u64, u64, i64, vp]
        lib.synth_normal_f32.argtypes = [u64, u64, i64, dbl, vp]
        lib.synth_normal_f64.argtypes = [u64, u64, i64, dbl, vp]
        lib.synth_outlier_channels.argtypes = [u64, u64, i64, i64, vp, vp]
        lib.synth_activation_bf16.argtypes = [u64, u64, i64, i64, vp, dbl, vp]
        lib.synth_f32_to_bf16.argtypes = [vp, i64, vp]
        lib.synth_uniform_u8.argtypes = [u64, u64, i64, i32, i32, vp]
        for f in (lib.synth_raw_u64, lib.synth_normal_f32, lib.synth_normal_f64,
                  lib.synth_outlier_channels, lib.synth_activation_bf16,
                  lib.synth_f32_to_bf16, lib.synth_uniform_u8):
            f.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def raw_u64(seed: int, tensor_id: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _load().synth_raw_u64(seed, tensor_id, n, _ptr(out))
    return out


def normal_f32(seed: int, tensor_id: int, shape, scale: float = 1.0) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    _load().synth_normal_f32(seed, tensor_id, out.size, float(scale), _ptr(out))
    return out


def normal_f64(seed: int, tensor_id: int, shape, scale: float = 1.0) -> np.ndarray:
    out = np.empty(shape, dtype=np.float64)
    _load().synth_normal_f64(seed, tensor_id, out.size, float(scale), _ptr(out))
    return out


def outlier_count(frac: float, K: int) -> int:
    """round(frac * K), halves away from zero."""
    return int(math.floor(frac * K + 0.5))


def outlier_channels(seed: int, tensor_id: int, K: int, count: int) -> np.ndarray:
    scratch = np.empty(K, dtype=np.int32)
    out = np.empty(count, dtype=np.int32)
    _load().synth_outlier_channels(seed, tensor_id, K, count, _ptr(scratch), _ptr(out))
    return out


def activation_bf16(seed: int, M: int, K: int, outlier_frac: float, factor: float,
                    tensor_id: int = TID_X) -> tuple[np.ndarray, np.ndarray]:
    """X[M, K] as bf16 bit patterns (uint16) and the outlier channel list."""
    count = outlier_count(outlier_frac, K)
    chans = outlier_channels(seed, TID_X_OUTLIERS + 1000 * (tensor_id - TID_X), K, count)
    flags = np.zeros(K, dtype=np.uint8)
    flags[chans] = 1
    out = np.empty((M, K), dtype=np.uint16)
    _load().synth_activation_bf16(seed, tensor_id, M, K, _ptr(flags), float(factor), _ptr(out))
    return out, chans


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().synth_f32_to_bf16(_ptr(x), x.size, _ptr(out))
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def uniform_u8(seed: int, tensor_id: int, shape, lo: int, hi: int) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint8)
    _load().synth_uniform_u8(seed, tensor_id, out.size, lo, hi, _ptr(out))
    return out


def weight_f32(seed: int, N: int, K: int, layer: int = 0, std: float = 0.02) -> np.ndarray:
    """W[N, K] ~ N(0, std^2) in fp32."""
    return normal_f32(seed, TID_W + layer, (N, K), std)


def kron_factors(seed: int) -> tuple[np.ndarray, np.ndarray]:
    """A = I4 + 0.1 N(0,1), B = I8 + 0.1 N(0,1), fp32 row-major."""
    A = (np.eye(4) + normal_f64(seed, TID_KRON_A, (4, 4), 0.1)).astype(np.float32)
    B = (np.eye(8) + normal_f64(seed, TID_KRON_B, (8, 8), 0.1)).astype(np.float32)
    return A, B


# --------------------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------------------

ROT_NONE, ROT_HADAMARD32, ROT_KRON_4x8 = 0, 1, 2


@dataclass(frozen=True)
class Linear:
    """One MXFP4 linear: Y[M, N] = X[M, K] . W[N, K]^T."""
    name: str
    M: int
    K: int
    N: int
    layer: int            # weight stream index
    x_tensor: int         # activation stream id
    outlier_frac: float
    outlier_factor: float

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K


@dataclass(frozen=True)
class Workload:
    name: str
    rotation: int
    linears: tuple = field(default_factory=tuple)
    seed: int = 0

    @property
    def flops(self) -> int:
        return sum(l.flops for l in self.linears)


def _dit(name: str, M: int) -> Workload:
    # FLUX-like DiT block: hidden 3072, MLP 12288; M tokens (3584 = 3072 image + 512 text per image).
    return Workload(name, ROT_HADAMARD32, (
        Linear("qkv", M, 3072, 9216, 0, TID_X, 0.01, 30.0),
        Linear("mlp_up", M, 3072, 12288, 1, TID_X, 0.01, 30.0),
        Linear("mlp_down", M, 12288, 3072, 2, TID_X + 1, 0.01, 30.0),
    ))


WORKLOADS = {
    "tiny": Workload("tiny", ROT_HADAMARD32, (
        Linear("tiny", 64, 256, 128, 0, TID_X, 0.02, 20.0),)),
    "dit_b1": _dit("dit_b1", 3584),
    "llm_small_m1": Workload("llm_small_m1", ROT_HADAMARD32, (
        Linear("up", 1, 4096, 14336, 0, TID_X, 0.005, 50.0),
        Linear("down", 1, 14336, 4096, 1, TID_X + 1, 0.005, 50.0))),
    "llm_small_m16": Workload("llm_small_m16", ROT_HADAMARD32, (
        Linear("up", 16, 4096, 14336, 0, TID_X, 0.005, 50.0),
        Linear("down", 16, 14336, 4096, 1, TID_X + 1, 0.005, 50.0))),
    "llm_small_m128": Workload("llm_small_m128", ROT_HADAMARD32, (
        Linear("up", 128, 4096, 14336, 0, TID_X, 0.005, 50.0),
        Linear("down", 128, 14336, 4096, 1, TID_X + 1, 0.005, 50.0))),
    # the DiT block's MLP alone (3584 tokens): up 3072 -> 12288, down 12288 -> 3072; run as
    # a chain, the down layer's input is the up layer's output
    "dit_mlp": Workload("dit_mlp", ROT_HADAMARD32, (
        Linear("mlp_up", 3584, 3072, 12288, 1, TID_X, 0.01, 30.0),
        Linear("mlp_down", 3584, 12288, 3072, 2, TID_X + 1, 0.01, 30.0))),
    "kron": Workload("kron", ROT_KRON_4x8, (
        Linear("kron", 3584, 3072, 3072, 0, TID_X, 0.01, 30.0),)),
    # the DiT block's MLP at batch 4 (14336 tokens): a mid-size case between dit_mlp and
    # dit_b16, small enough for full profiler captures
    "dit_b4": Workload("dit_b4", ROT_HADAMARD32, (
        Linear("mlp_up", 14336, 3072, 12288, 1, TID_X, 0.01, 30.0),
        Linear("mlp_down", 14336, 12288, 3072, 2, TID_X + 1, 0.01, 30.0))),
    "dit_b16": Workload("dit_b16", ROT_HADAMARD32, (
        Linear("mlp_up", 57344, 3072, 12288, 1, TID_X, 0.01, 30.0),
        Linear("mlp_down", 57344, 12288, 3072, 2, TID_X + 1, 0.01, 30.0))),
}
