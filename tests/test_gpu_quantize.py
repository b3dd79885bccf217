"""GPU parity of the rotate+quantise kernels against the oracle: packed codes and
E8M0 scale bytes (tensor-core layout, padding included) must be bit-identical."""
import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import quantize_parity

pytestmark = pytest.mark.gpu

MODES = [oracle.ROT_NONE, oracle.ROT_HADAMARD32, oracle.ROT_KRON_4x8]


def _kron(mode):
    return synth.kron_factors(0) if mode == oracle.ROT_KRON_4x8 else (None, None)


def _adversarial_f32() -> np.ndarray:
    """One block per row, each built to hit a rounding or scale edge case."""
    blocks = []
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float32)
    b = np.zeros(32, np.float32)
    b[:8] = ties
    b[8:16] = -ties
    b[16:24] = ties * 0.5
    b[24:32] = -ties * 0.5
    blocks.append(b)
    for e in (-140, -130, -127, -126, -100, -3, 0, 7, 100, 125):  # ties at many scales
        blocks.append(b * np.float32(2.0 ** e) if e > -127 else (b.astype(np.float64) * 2.0 ** e).astype(np.float32))
    blocks.append(np.float32(2.0) ** np.arange(-16, 16, dtype=np.float32))      # exact powers of two
    blocks.append(np.full(32, 7.0, np.float32) * np.where(np.arange(32) % 2, 1, -1))  # amax in (6, 8): saturation
    blocks.append(np.linspace(-7.99, 7.99, 32).astype(np.float32))
    blocks.append(np.zeros(32, np.float32))                                      # all zero
    blocks.append(-np.zeros(32, np.float32))                                     # all -0
    sub = np.arange(1, 33, dtype=np.uint32).view(np.float32)                     # subnormals
    blocks.append(sub)
    blocks.append(-sub * np.float32(3))
    o = np.full(32, 0.01, np.float32)
    o[17] = 1e30                                                                 # one huge outlier
    blocks.append(o)
    o2 = np.full(32, -1e-3, np.float32)
    o2[3] = -3e38                                                                # near fp32 max
    blocks.append(o2)
    blocks.append(np.full(32, 3e38, np.float32))                                 # overflows in the butterfly
    inf = np.ones(32, np.float32)
    inf[5] = np.inf
    blocks.append(inf)
    nan = np.ones(32, np.float32)
    nan[30] = np.nan
    blocks.append(nan)
    rng = np.random.default_rng(5)
    for _ in range(40):                                                          # values near midpoints
        e = rng.integers(-20, 20)
        mids = rng.choice([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], 32)
        jitter = rng.choice([0, 1, -1], 32)
        v = (mids * 2.0 ** e).astype(np.float32)
        v = np.where(jitter == 1, np.nextafter(v, np.float32(np.inf)),
                     np.where(jitter == -1, np.nextafter(v, np.float32(0)), v))
        v[0] = np.float32(6.0 * 2.0 ** e)
        blocks.append(v * rng.choice([-1, 1], 32).astype(np.float32))
    return np.stack(blocks).astype(np.float32)


@pytest.mark.parametrize("mode", MODES)
def test_adversarial_blocks_fp32_input(mode):
    x = _adversarial_f32()
    # several blocks per row, rows not a multiple of 128
    x = np.concatenate([x, x[::-1]], axis=1)
    A, B = _kron(mode)
    quantize_parity(x, mode, A, B)


@pytest.mark.parametrize("mode", MODES)
def test_adversarial_blocks_bf16_input(mode):
    x32 = _adversarial_f32()
    bits = synth.f32_to_bf16_bits(x32)
    A, B = _kron(mode)
    quantize_parity(bits, mode, A, B)


@pytest.mark.parametrize("rows", [1, 2, 127, 128, 129, 300])
@pytest.mark.parametrize("K", [32, 96, 256, 640])
def test_ragged_shapes_hadamard(rows, K):
    x, _ = synth.activation_bf16(rows * 7 + K, rows, K, 0.02, 20.0)
    quantize_parity(x, oracle.ROT_HADAMARD32)


@pytest.mark.parametrize("mode", MODES)
def test_strided_rows(mode):
    x, _ = synth.activation_bf16(3, 200, 512, 0.02, 20.0)
    A, B = _kron(mode)
    quantize_parity(x, mode, A, B, ld_pad=64)


@pytest.mark.parametrize("name", ["tiny", "dit_b1", "llm_small_m16", "kron"])
def test_workload_activations(name):
    wl = synth.WORKLOADS[name]
    A, B = synth.kron_factors(wl.seed) if wl.rotation == oracle.ROT_KRON_4x8 else (None, None)
    seen = set()
    for lin in wl.linears:
        key = (lin.M, lin.K, lin.x_tensor)
        if key in seen:
            continue
        seen.add(key)
        x, _ = synth.activation_bf16(wl.seed, lin.M, lin.K, lin.outlier_frac, lin.outlier_factor,
                                     lin.x_tensor)
        quantize_parity(x, wl.rotation, A, B)


@pytest.mark.parametrize("j", [0, 1])
def test_large_batch_activation_rows(j):
    """The two activations of the batch-16 DiT MLP, whole, on the GPU: 57344 x 3072
    (MLP-up input) and 57344 x 12288 (MLP-down input, 1.41 GB of bf16); every code and
    scale byte compared with the oracle's."""
    lin = synth.WORKLOADS["dit_b16"].linears[j]
    x, _ = synth.activation_bf16(0, lin.M, lin.K, lin.outlier_frac, lin.outlier_factor, lin.x_tensor)
    quantize_parity(x, oracle.ROT_HADAMARD32)


@pytest.mark.parametrize("mode", MODES)
def test_weight_preparation(mode):
    """Offline weight preparation through the same kernel (fp32 input; the
    Kronecker mode takes A^-T and B^-T)."""
    w = synth.weight_f32(0, 384, 3072)
    if mode == oracle.ROT_KRON_4x8:
        A, B = oracle.kron_weight_factors(*synth.kron_factors(0))
    else:
        A, B = None, None
    q, s = quantize_parity(w, mode, A, B)
    if mode != oracle.ROT_KRON_4x8:
        eq, es = oracle.prepare_weight(w, mode)
        assert np.array_equal(q, eq) and np.array_equal(s, es)


# ---- larger Hadamard blocks: 64- and 128-element rotation groups, scales per 32

WIDE = [oracle.ROT_HADAMARD64, oracle.ROT_HADAMARD128]


def _rows_of(x: np.ndarray, span: int) -> np.ndarray:
    """Adversarial 32-blocks regrouped into rows of `span` elements (zero blocks appended)."""
    per = span // 32
    n = -(-x.shape[0] // per) * per
    pad = np.zeros((n - x.shape[0], 32), x.dtype)
    return np.concatenate([x, pad]).reshape(-1, span)


@pytest.mark.parametrize("mode", WIDE)
def test_wide_adversarial_fp32_and_bf16(mode):
    span = oracle.rotation_span(mode)
    x = _rows_of(_adversarial_f32(), span)
    x = np.concatenate([x, x[::-1], -x], axis=1)  # 3 groups per row
    quantize_parity(x, mode)
    quantize_parity(synth.f32_to_bf16_bits(x), mode)


@pytest.mark.parametrize("mode", WIDE)
@pytest.mark.parametrize("rows", [1, 127, 129, 300])
@pytest.mark.parametrize("groups", [1, 3, 8])
def test_wide_ragged_shapes(mode, rows, groups):
    K = oracle.rotation_span(mode) * groups
    x, _ = synth.activation_bf16(rows + K, rows, K, 0.02, 20.0)
    quantize_parity(x, mode)


@pytest.mark.parametrize("mode", WIDE)
def test_wide_strided_rows_and_weights(mode):
    x, _ = synth.activation_bf16(4, 200, 1024, 0.02, 20.0)
    quantize_parity(x, mode, ld_pad=64)
    w = synth.weight_f32(1, 256, 3072)
    q, s = quantize_parity(w, mode, ld_pad=32)
    eq, es = oracle.prepare_weight(w, mode)
    assert np.array_equal(q, eq) and np.array_equal(s, es)


@pytest.mark.parametrize("mode", WIDE)
def test_wide_mode_rejects_k_not_a_multiple_of_the_group(mode):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    x = torch.zeros((4, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mx.MXFP4Error):
        mx.rotate_quantize(x, mode)
