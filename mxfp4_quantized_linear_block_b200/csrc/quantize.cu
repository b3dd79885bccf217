// quantize.cu -- online block rotation + MXFP4 quantisation (HBM-bound).
//
// One thread owns one 32-element block of a row. A warp owns 32 consecutive
// blocks: it loads them with fully coalesced 16-byte loads (lane L reads
// chunk 32*i + L of the warp's span), transposes them through a swizzled
// shared-memory buffer so that every thread holds its own block, rotates the
// block in registers, takes the E8M0 scale from the block amax and writes 16
// bytes of packed E2M1 codes plus one scale byte in the tensor-core scale
// layout. Padding rows / blocks of the scale layout are written as 0.
//
// Method: "Bridging the Gap Between Promise and Performance for Microscaling
// FP4 Quantization" ("Methodologie: MR-GPTQ" item 1: block-wise Hadamard
// rotation; "GPU Kernel Ondersteuning (QuTLASS)": rotation fused into the
// quantisation kernel, online) and "KroQuant: Effiziente Post-Training-
// Quantisierung fuer Diffusion Transformers mittels Kronecker-Produkt-Struktur"
// ("Tiefenanalyse": a Kronecker-structured transform on each 32-element
// block). MXFP4 format: "AMD Quark delivers MXFP4 quantization for FLUX.1-dev
// on Instinct MI350 with 1.92x speedup", "What is MXFP4 and why does it
// eliminate dequantization overhead?".
//
// Bit-exactness: every fp32 operation is an explicit round-to-nearest
// intrinsic (no contraction, no flush to zero), in the order the C ABI
// documents, so codes and scales are bit-identical to a sequential fp32
// evaluation of the same formulas.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace mxfp4 {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr float kInvSqrt32 = 0x1.6a09e6p-3f;  // fp32 nearest to 1/sqrt(32)

__device__ __forceinline__ uint4 ld_nc_v4(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_v4(uint8_t* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// Chunk swizzle of the per-warp transpose buffer (16-byte units): makes both
// the coalesced stores and the per-thread block reads bank-conflict free.
template <int CH>
__device__ __forceinline__ uint32_t chunk_swizzle(uint32_t t) {
  return CH == 4 ? ((t >> 1) & 3u) : (t & 7u);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// E2M1 pair: element `lo` -> bits 0-3, element `hi` -> bits 4-7; round to nearest
// even with saturation to +-6 by the hardware conversion, sign bit forced from
// the input so negatives that round to zero are -0 (code 8).
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  r |= ((__float_as_uint(lo) >> 28) & 0x8u) | ((__float_as_uint(hi) >> 24) & 0x80u);
  return r;
}

__device__ __forceinline__ float max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

__device__ __forceinline__ float max3_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Normalised Sylvester Hadamard of one block: butterfly stages with strides
// 1, 2, 4, 8, 16 ((a, b) -> (a + b, a - b)), then one multiply by kInvSqrt32.
// Stages 1..8 run on packed pairs (v[t], v[t + 16]); stage 16 pairs the two
// halves of each packed value.
__device__ __forceinline__ void hadamard32(float (&v)[32]) {
  float2 P[16];
#pragma unroll
  for (int t = 0; t < 16; ++t) P[t] = make_float2(v[t], v[t + 16]);
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i & h) continue;
      const float2 a = P[i], b = P[i + h];
      P[i] = __fadd2_rn(a, b);
      P[i + h] = __fadd2_rn(a, make_float2(-b.x, -b.y));
    }
  }
  const float2 c = make_float2(kInvSqrt32, kInvSqrt32);
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    const float a = P[t].x, b = P[t].y;
    const float2 s = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
    const float2 r = __fmul2_rn(s, c);
    v[t] = r.x;
    v[t + 16] = r.y;
  }
}

// y = (A (x) B) x: z[8j+k] = sum_l B[k][l] x[8j+l], y[8i+k] = sum_j A[i][j] z[8j+k],
// each sum a chain that starts with the first product and adds the rest by fma
// in ascending index order.
__device__ __forceinline__ void kron32(float (&v)[32], const KronCoeffs& kc) {
  float z[32];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float acc = __fmul_rn(kc.b[k * 8 + 0], v[8 * j + 0]);
#pragma unroll
      for (int l = 1; l < 8; ++l) acc = __fmaf_rn(kc.b[k * 8 + l], v[8 * j + l], acc);
      z[8 * j + k] = acc;
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float acc = __fmul_rn(kc.a[i * 4 + 0], z[k]);
#pragma unroll
      for (int j = 1; j < 4; ++j) acc = __fmaf_rn(kc.a[i * 4 + j], z[8 * j + k], acc);
      v[8 * i + k] = acc;
    }
  }
}

// Quantise one rotated block: returns the E8M0 byte and the 16 code bytes.
__device__ __forceinline__ uint32_t quantize_block(const float (&v)[32], uint4& codes) {
  // amax with NaN propagation (a NaN anywhere makes m NaN).
  float m = max_nan(fabsf(v[0]), fabsf(v[31]));
#pragma unroll
  for (int i = 1; i < 31; i += 2) m = max3_nan(m, fabsf(v[i]), fabsf(v[i + 1]));
  const uint32_t mb = __float_as_uint(m) & 0x7FFFFFFFu;
  if (mb >= 0x7F800000u) {  // Inf or NaN in the block
    codes = make_uint4(0u, 0u, 0u, 0u);
    return 0xFFu;
  }
  // e = max(floor(log2 amax) - 2, -127); byte = e + 127 = max(biased_exp, 2) - 2.
  const uint32_t be = mb >> 23;
  const uint32_t byte = (be > 2u ? be : 2u) - 2u;
  const float inv = __uint_as_float((254u - byte) << 23);  // 2^-e, always a normal number
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t acc = 0;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int i = 8 * q + 2 * p;
      const float2 s = __fmul2_rn(make_float2(v[i], v[i + 1]), make_float2(inv, inv));
      acc |= e2m1x2(s.x, s.y) << (8 * p);
    }
    w[q] = acc;
  }
  codes = make_uint4(w[0], w[1], w[2], w[3]);
  return byte;
}

template <int MODE, bool F32_IN>
__global__ void __launch_bounds__(kThreads) rotate_quantize_kernel(
    const uint8_t* __restrict__ x, uint32_t rows, uint32_t kb_real, uint32_t kb_pad,
    uint64_t ldx_bytes, uint64_t q_row_bytes, uint32_t n_units, uint32_t n_katoms,
    const __grid_constant__ KronCoeffs kc, uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  constexpr int CH = F32_IN ? 8 : 4;  // 16-byte chunks per 32-element block
  __shared__ uint4 stage[kWarps][32 * CH];
  const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
  uint4* buf = stage[warp];

  for (uint32_t base = blockIdx.x * kThreads + warp * 32u; base < n_units;
       base += gridDim.x * kThreads) {
    const uint32_t u = base + lane;
    const uint32_t r = u / kb_pad;
    const uint32_t kb = u - r * kb_pad;
    const bool live = u < n_units && r < rows && kb < kb_real;
    const unsigned long long src =
        live ? reinterpret_cast<unsigned long long>(x + (uint64_t)r * ldx_bytes +
                                                    (uint64_t)kb * (CH * 16))
             : 0ull;

    // Coalesced loads of the warp's 32 blocks, then transpose through shared memory.
    uint4 ld[CH];
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      const uint32_t g = 32u * i + lane, t = g / CH, c = g % CH;
      const unsigned long long p = __shfl_sync(0xffffffffu, src, t);
      ld[i] = p ? ld_nc_v4(reinterpret_cast<const uint8_t*>(p) + c * 16) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      const uint32_t g = 32u * i + lane, t = g / CH, c = g % CH;
      buf[t * CH + (c ^ chunk_swizzle<CH>(t))] = ld[i];
    }
    __syncwarp();
    float v[32];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const uint4 w = buf[lane * CH + (c ^ chunk_swizzle<CH>(lane))];
      if constexpr (F32_IN) {
        v[4 * c + 0] = __uint_as_float(w.x);
        v[4 * c + 1] = __uint_as_float(w.y);
        v[4 * c + 2] = __uint_as_float(w.z);
        v[4 * c + 3] = __uint_as_float(w.w);
      } else {
        v[8 * c + 0] = bf16_lo(w.x);
        v[8 * c + 1] = bf16_hi(w.x);
        v[8 * c + 2] = bf16_lo(w.y);
        v[8 * c + 3] = bf16_hi(w.y);
        v[8 * c + 4] = bf16_lo(w.z);
        v[8 * c + 5] = bf16_hi(w.z);
        v[8 * c + 6] = bf16_lo(w.w);
        v[8 * c + 7] = bf16_hi(w.w);
      }
    }
    __syncwarp();

    if (u < n_units) {
      uint32_t byte = 0;
      if (live) {
        if constexpr (MODE == 1) hadamard32(v);
        if constexpr (MODE == 2) kron32(v, kc);
        uint4 codes;
        byte = quantize_block(v, codes);
        st_v4(q + (uint64_t)r * q_row_bytes + (uint64_t)kb * 16u, codes);
      }
      const uint64_t off = ((uint64_t)(r >> 7) * n_katoms + (kb >> 2)) * 512u + (r & 31u) * 16u +
                           ((r >> 5) & 3u) * 4u + (kb & 3u);
      sf[off] = static_cast<uint8_t>(byte);
    }
  }
  // Let a dependent kernel (the GEMM of the fused layer) start its set-up; it
  // still waits for this grid's completion before reading q / sf.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <int MODE, bool F32_IN>
cudaError_t launch_mode(const void* x, int64_t rows, int64_t K, int64_t ldx, const KronCoeffs& kc,
                        uint8_t* q, uint8_t* sf, cudaStream_t stream) {
  const int64_t kb_real = K / 32;
  const int64_t kb_pad = sf_katoms(K) * 4;
  const int64_t rows_pad = sf_row_tiles(rows) * 128;
  const int64_t n_units = rows_pad * kb_pad;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t blocks_needed = (n_units + kThreads - 1) / kThreads;
  const int64_t cap = (int64_t)sms * 8;  // grid-stride beyond 8 CTAs per SM
  const int grid = (int)(blocks_needed < cap ? blocks_needed : cap);
  rotate_quantize_kernel<MODE, F32_IN><<<grid, kThreads, 0, stream>>>(
      static_cast<const uint8_t*>(x), (uint32_t)rows, (uint32_t)kb_real, (uint32_t)kb_pad,
      (uint64_t)ldx * (F32_IN ? 4u : 2u), (uint64_t)(K / 2), (uint32_t)n_units,
      (uint32_t)sf_katoms(K), kc, q, sf);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rotate_quantize(const void* x, bool x_is_f32, int64_t rows, int64_t K,
                                   int64_t ldx, int mode, const KronCoeffs* kc, uint8_t* q,
                                   uint8_t* sf, cudaStream_t stream) {
  KronCoeffs k{};
  if (kc) k = *kc;
  if (x_is_f32) {
    if (mode == 1) return launch_mode<1, true>(x, rows, K, ldx, k, q, sf, stream);
    if (mode == 2) return launch_mode<2, true>(x, rows, K, ldx, k, q, sf, stream);
    return launch_mode<0, true>(x, rows, K, ldx, k, q, sf, stream);
  }
  if (mode == 1) return launch_mode<1, false>(x, rows, K, ldx, k, q, sf, stream);
  if (mode == 2) return launch_mode<2, false>(x, rows, K, ldx, k, q, sf, stream);
  return launch_mode<0, false>(x, rows, K, ldx, k, q, sf, stream);
}

}  // namespace mxfp4
