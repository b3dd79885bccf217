// block_quant.cuh -- device math of one 32-element block: the online rotation
// (normalised Sylvester Hadamard-32 or Kronecker A (x) B) and the MXFP4
// quantisation (E8M0 scale from the block amax, E2M1 codes, round to nearest
// even, saturation to +-6), shared by the standalone rotate+quantise kernel and
// by the quantiser warps of the fused linear kernel.
//
// Method: "Bridging the Gap Between Promise and Performance for Microscaling
// FP4 Quantization" ("Methodologie: MR-GPTQ" item 1; "GPU Kernel Ondersteuning
// (QuTLASS)") and "KroQuant: Effiziente Post-Training-Quantisierung fuer
// Diffusion Transformers mittels Kronecker-Produkt-Struktur" ("Tiefenanalyse").
// Every fp32 operation is an explicit round-to-nearest intrinsic, in the order
// the C ABI documents, so results are bit-identical to a sequential fp32
// evaluation.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace mxfp4 {
namespace blockq {

constexpr float kInvSqrt32 = 0x1.6a09e6p-3f;  // fp32 nearest to 1/sqrt(32)

__device__ __forceinline__ void st_v4(uint8_t* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Eight scaled values -> one word of packed E2M1 codes (element 2j in the low
// nibble of byte j): round to nearest even with saturation to +-6 by the
// hardware conversion, which keeps the sign of values that round to zero
// (code 8), as the format rule requires.
__device__ __forceinline__ uint32_t e2m1x8(float s0, float s1, float s2, float s3, float s4,
                                           float s5, float s6, float s7) {
  uint32_t w;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(w)
      : "f"(s0), "f"(s1), "f"(s2), "f"(s3), "f"(s4), "f"(s5), "f"(s6), "f"(s7));
  return w;
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

// A 32-element block lives in 16 packed pairs P[j] = (v[2j], v[2j + 1]).
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// Block b (0 or 1) of bf16 row r of a 128-byte-swizzled shared tile (row address
// row_addr): 64 bytes -> 16 packed pairs. Reads of 8 consecutive rows hit 8
// different bank groups, so a warp's reads are conflict free.
__device__ __forceinline__ void load_block_bf16_sw128(uint32_t row_addr, uint32_t r, uint32_t b,
                                                      float2 (&P)[16]) {
#pragma unroll
  for (uint32_t c = 0; c < 4; ++c) {
    const uint4 w = ld_shared_v4(row_addr + (((b * 4u + c) ^ (r & 7u)) << 4));
    P[4 * c + 0] = make_float2(bf16_lo(w.x), bf16_hi(w.x));
    P[4 * c + 1] = make_float2(bf16_lo(w.y), bf16_hi(w.y));
    P[4 * c + 2] = make_float2(bf16_lo(w.z), bf16_hi(w.z));
    P[4 * c + 3] = make_float2(bf16_lo(w.w), bf16_hi(w.w));
  }
}

// Byte offset of (row, 32-block kb) in the tensor-core scale layout.
__device__ __forceinline__ uint64_t sf_offset(uint32_t row, uint32_t kb, uint32_t n_katoms) {
  return ((uint64_t)(row >> 7) * n_katoms + (kb >> 2)) * 512u + (row & 31u) * 16u +
         ((row >> 5) & 3u) * 4u + (kb & 3u);
}

#define BLK(P, i) (((i) & 1) ? (P)[(i) >> 1].y : (P)[(i) >> 1].x)

// Unnormalised Sylvester butterfly of one block: stages with strides 1, 2, 4, 8, 16
// ((a, b) -> (a + b, a - b)). Stride 1 pairs the two halves of each packed value;
// strides 2..16 pair whole packed values lane by lane (a - b as the exact fma
// b * -1 + a).
__device__ __forceinline__ void fwht32(float2 (&P)[16]) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float a = P[j].x, b = P[j].y;
    P[j] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
  }
  const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j & h) continue;
      const float2 a = P[j], b = P[j + h];
      P[j] = __fadd2_rn(a, b);
      P[j + h] = __ffma2_rn(b, m1, a);
    }
  }
}

// Normalised Sylvester Hadamard of one block: the butterfly, then one multiply by
// kInvSqrt32.
__device__ __forceinline__ void hadamard32(float2 (&P)[16]) {
  fwht32(P);
  const float2 c = make_float2(kInvSqrt32, kInvSqrt32);
#pragma unroll
  for (int j = 0; j < 16; ++j) P[j] = __fmul2_rn(P[j], c);
}

// y = (A (x) B) x: z[8j+k] = sum_l B[k][l] x[8j+l], y[8i+k] = sum_j A[i][j] z[8j+k],
// each sum a chain that starts with the first product and adds the rest by fma
// in ascending index order. Two outputs per packed fp32 operation, each lane doing that
// chain: z[8j+k], z[8j+k+1] with the coefficient pair (B[k][l], B[k+1][l]) and x[8j+l]
// in both lanes; y[8i+k], y[8i+k+1] with A[i][j] in both lanes.
__device__ __forceinline__ void kron32(float2 (&P)[16], const KronCoeffs& kc) {
  const float2* bt = reinterpret_cast<const float2*>(kc.bt);  // bt[4 l + kp]: k = 2 kp, 2 kp + 1
  const float2* a2 = reinterpret_cast<const float2*>(kc.a2);  // a2[4 i + j]: A[i][j] twice
  float2 zp[4][4];  // zp[j][kp] = (z[8j + 2kp], z[8j + 2kp + 1])
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int l = 0; l < 8; ++l) {
      const float xv = BLK(P, 8 * j + l);
      const float2 xd = make_float2(xv, xv);
#pragma unroll
      for (int kp = 0; kp < 4; ++kp)
        zp[j][kp] = l == 0 ? __fmul2_rn(bt[4 * l + kp], xd)
                           : __ffma2_rn(bt[4 * l + kp], xd, zp[j][kp]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int kp = 0; kp < 4; ++kp) {
      float2 y = __fmul2_rn(a2[4 * i + 0], zp[0][kp]);
#pragma unroll
      for (int j = 1; j < 4; ++j) y = __ffma2_rn(a2[4 * i + j], zp[j][kp], y);
      P[4 * i + kp] = y;
    }
  }
}

// Quantise one rotated block: returns the E8M0 byte and the 16 code bytes.
__device__ __forceinline__ uint32_t quantize_block(const float2 (&P)[16], uint4& codes) {
  // amax with NaN propagation (a NaN anywhere makes m NaN).
  float m = max_nan(fabsf(P[0].x), fabsf(P[0].y));
#pragma unroll
  for (int j = 1; j < 16; ++j) m = max3_nan(m, fabsf(P[j].x), fabsf(P[j].y));
  const uint32_t mb = __float_as_uint(m) & 0x7FFFFFFFu;
  if (mb >= 0x7F800000u) {  // Inf or NaN in the block
    codes = make_uint4(0u, 0u, 0u, 0u);
    return 0xFFu;
  }
  // e = max(floor(log2 amax) - 2, -127); byte = e + 127 = max(biased_exp, 2) - 2.
  const uint32_t be = mb >> 23;
  const uint32_t byte = (be > 2u ? be : 2u) - 2u;
  const float inv = __uint_as_float((254u - byte) << 23);  // 2^-e, always a normal number
  const float2 sc = make_float2(inv, inv);
  float2 S[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) S[j] = __fmul2_rn(P[j], sc);  // exact: power-of-two scale
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q)
    w[q] = e2m1x8(S[4 * q].x, S[4 * q].y, S[4 * q + 1].x, S[4 * q + 1].y, S[4 * q + 2].x,
                  S[4 * q + 2].y, S[4 * q + 3].x, S[4 * q + 3].y);
  codes = make_uint4(w[0], w[1], w[2], w[3]);
  return byte;
}

// ---------------------------------------------------------------- NVFP4 groups
//
// NVFP4 ("Bridging the Gap...", "Probleemstelling" item 1): 16-element groups with an
// unsigned E4M3 scale each and an fp32 tensor scale st. Per group: g = amax / (6 st)
// (two roundings), byte = nearest E4M3 of g (ties to even, saturating at 448),
// S = E4M3(byte) * st, r = 1 / S, code_i = nearest E2M1 of y_i * r; each step one
// IEEE fp32 rounding. st <= 0 (all-zero tensor) or S == 0 gives byte / codes 0.

__device__ __forceinline__ uint32_t e4m3_rn(float g) {
  uint16_t h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(g));
  return h & 0xFFu;  // the second source goes to the low byte
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
  uint32_t hh;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hh) : "h"((uint16_t)byte));
  return __half2float(__ushort_as_half((unsigned short)(hh & 0xFFFFu)));
}

// 8 packed pairs (16 rotated values) -> E4M3 byte, and 8 code bytes in w[0..1].
__device__ __forceinline__ uint32_t quantize_group16(const float2* P, float st, uint32_t (&w)[2]) {
  float m = fabsf(P[0].x);
#pragma unroll
  for (int j = 0; j < 8; ++j) m = fmaxf(m, fmaxf(fabsf(P[j].x), fabsf(P[j].y)));
  w[0] = w[1] = 0u;
  if (!(st > 0.0f)) return 0u;
  const float g = __fdiv_rn(m, __fmul_rn(6.0f, st));
  const uint32_t byte = e4m3_rn(g);
  const float S = __fmul_rn(e4m3_to_f32(byte), st);
  if (S == 0.0f) return byte;
  const float r = __frcp_rn(S);
  const float2 rr = make_float2(r, r);
  float2 v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = __fmul2_rn(P[j], rr);
  w[0] = e2m1x8(v[0].x, v[0].y, v[1].x, v[1].y, v[2].x, v[2].y, v[3].x, v[3].y);
  w[1] = e2m1x8(v[4].x, v[4].y, v[5].x, v[5].y, v[6].x, v[6].y, v[7].x, v[7].y);
  return byte;
}

}  // namespace blockq
}  // namespace mxfp4
