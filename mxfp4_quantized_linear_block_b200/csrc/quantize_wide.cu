// quantize_wide.cu -- rotation over 64- or 128-element groups + MXFP4 quantisation.
//
// Larger Hadamard blocks: H_n = H2^(x log2 n) / sqrt(n) with n = 64 or 128 (2 or 4 MX
// blocks), the contrast "KroQuant: Effiziente Post-Training-Quantisierung fuer Diffusion
// Transformers mittels Kronecker-Produkt-Struktur" ("Hintergrund") draws with block-wise
// Hadamard rotations of larger blocks; the E8M0 scale stays per 32 elements. Butterfly
// strides 1, 2, ..., n/2 in fp32, then one multiply by the fp32 nearest 1/sqrt(n).
//
// fp32 input (the offline weight preparation; bf16 activations take the tile quantiser).
// A rotation group is spread over the lanes of a warp: each lane holds EPL consecutive
// elements (4 fp32: one 16-byte load; the kernel is written for 8 bf16 as well), so a
// warp covers 32 * EPL consecutive elements of a row. Butterfly strides below EPL run inside a lane, the
// others pair lane l with l ^ (stride / EPL) through shuffles: the lower lane computes
// a + b, the upper a - b as fma(b, -1, a), i.e. every element sees the fp32 operations
// of a sequential evaluation, in the same order. amax and the scale are reduced over
// the 32 / EPL lanes of each 32-element block. No shared memory, no barriers.
#include <cuda_runtime.h>

#include <cstdint>

#include "block_quant.cuh"
#include "internal.h"

namespace mxfp4 {
namespace {

using namespace blockq;

constexpr int kThreads = 256;
constexpr uint32_t kUnroll = 2;  // warp segments per iteration (loads in flight)

// fp32 nearest 1/sqrt(n): 1/8 exactly, and half of the fp32 nearest 1/sqrt(32).
template <int SPAN>
__device__ __forceinline__ float inv_sqrt_span() {
  return SPAN == 64 ? 0.125f : 0x1.6a09e6p-4f;
}

// Two scaled values -> one byte of E2M1 codes (element 0 in the low nibble).
__device__ __forceinline__ uint32_t e2m1x2(float s0, float s1) {
  uint32_t b;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(b)
      : "f"(s0), "f"(s1));
  return b;
}

// One butterfly stage across lanes l and l ^ mask on a lane's packed pairs.
template <int NP>
__device__ __forceinline__ void butterfly_lanes(float2 (&P)[NP], uint32_t mask, bool upper) {
  const float2 s = upper ? make_float2(-1.0f, -1.0f) : make_float2(1.0f, 1.0f);
#pragma unroll
  for (int j = 0; j < NP; ++j) {
    float2 o;
    o.x = __shfl_xor_sync(0xffffffffu, P[j].x, mask);
    o.y = __shfl_xor_sync(0xffffffffu, P[j].y, mask);
    P[j] = __ffma2_rn(P[j], s, o);  // lower: own + other; upper: -own + other
  }
}

template <int EPL, int SPAN>
__global__ void __launch_bounds__(kThreads) rotate_quantize_wide_kernel(
    const void* __restrict__ x, uint64_t ldx, uint32_t rows, uint32_t rows_pad, uint32_t kb_real,
    uint32_t kb_pad, uint32_t segs_per_row, uint32_t n_segs, uint32_t n_katoms,
    uint64_t q_row_bytes, uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  constexpr uint32_t NP = EPL / 2;        // packed pairs per lane
  constexpr uint32_t LPB = 32 / EPL;      // lanes per 32-element block
  constexpr uint32_t BPW = 32 / LPB;      // blocks per warp segment
  constexpr uint32_t LPG = SPAN / EPL;    // lanes per rotation group
  static_assert(LPG <= 32, "a rotation group fits in a warp");
  // x and the previous kernel's readers of q / sf: wait for that kernel, then let the
  // next one start its set-up (programmatic dependent launch).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t c = lane % LPB;  // chunk of EPL elements inside the block
  const uint32_t bl = lane / LPB;  // block inside the segment
  const uint32_t warps = gridDim.x * (kThreads / 32);
  const uint32_t gw = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
  for (uint32_t s0 = gw; s0 < n_segs; s0 += kUnroll * warps) {
    float2 P[kUnroll][NP];
    uint32_t row[kUnroll], kb[kUnroll];
    bool valid[kUnroll];
#pragma unroll
    for (uint32_t u = 0; u < kUnroll; ++u) {
      const uint32_t sg = s0 + u * warps;
      row[u] = sg / segs_per_row;
      kb[u] = (sg - row[u] * segs_per_row) * BPW + bl;
      valid[u] = sg < n_segs && row[u] < rows && kb[u] < kb_real;
#pragma unroll
      for (uint32_t j = 0; j < NP; ++j) P[u][j] = make_float2(0.0f, 0.0f);
      if (valid[u]) {
        const uint64_t e = (uint64_t)row[u] * ldx + (uint64_t)kb[u] * 32u + c * EPL;
        if constexpr (EPL == 8) {
          const uint4 w = __ldcs(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + e));
          P[u][0] = make_float2(bf16_lo(w.x), bf16_hi(w.x));
          P[u][1] = make_float2(bf16_lo(w.y), bf16_hi(w.y));
          P[u][2] = make_float2(bf16_lo(w.z), bf16_hi(w.z));
          P[u][3] = make_float2(bf16_lo(w.w), bf16_hi(w.w));
        } else {
          const float4 w = __ldcs(reinterpret_cast<const float4*>(static_cast<const float*>(x) + e));
          P[u][0] = make_float2(w.x, w.y);
          P[u][1] = make_float2(w.z, w.w);
        }
      }
    }
#pragma unroll
    for (uint32_t u = 0; u < kUnroll; ++u) {
      if (s0 + u * warps >= n_segs) break;  // uniform across the warp
      float2 (&Q)[NP] = P[u];
      // strides 1 .. EPL / 2 inside the lane
#pragma unroll
      for (uint32_t j = 0; j < NP; ++j) {
        const float a = Q[j].x, b = Q[j].y;
        Q[j] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
      }
      const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
      for (uint32_t h = 1; h < NP; h <<= 1) {
#pragma unroll
        for (uint32_t j = 0; j < NP; ++j) {
          if (j & h) continue;
          const float2 a = Q[j], b = Q[j + h];
          Q[j] = __fadd2_rn(a, b);
          Q[j + h] = __ffma2_rn(b, m1, a);
        }
      }
      // strides EPL .. SPAN / 2 across lanes
#pragma unroll
      for (uint32_t m = 1; m < LPG; m <<= 1) butterfly_lanes<NP>(Q, m, (lane & m) != 0u);
      const float2 cn = make_float2(inv_sqrt_span<SPAN>(), inv_sqrt_span<SPAN>());
#pragma unroll
      for (uint32_t j = 0; j < NP; ++j) Q[j] = __fmul2_rn(Q[j], cn);
      // amax of the 32-element block (NaN-propagating) over its LPB lanes
      float mx = max_nan(fabsf(Q[0].x), fabsf(Q[0].y));
#pragma unroll
      for (uint32_t j = 1; j < NP; ++j) mx = max3_nan(mx, fabsf(Q[j].x), fabsf(Q[j].y));
#pragma unroll
      for (uint32_t m = 1; m < LPB; m <<= 1) mx = max_nan(mx, __shfl_xor_sync(0xffffffffu, mx, m));
      const uint32_t mb = __float_as_uint(mx) & 0x7FFFFFFFu;
      uint32_t byte, word = 0;
      if (mb >= 0x7F800000u) {  // Inf or NaN in the block
        byte = 0xFFu;
      } else {
        const uint32_t be = mb >> 23;
        byte = (be > 2u ? be : 2u) - 2u;  // e = max(floor(log2 amax) - 2, -127), + 127
        const float inv = __uint_as_float((254u - byte) << 23);  // 2^-e
        const float2 sc = make_float2(inv, inv);
#pragma unroll
        for (uint32_t j = 0; j < NP; ++j) {
          const float2 v = __fmul2_rn(Q[j], sc);
          word |= e2m1x2(v.x, v.y) << (8u * j);
        }
      }
      if (valid[u]) {
        uint8_t* dst = q + (uint64_t)row[u] * q_row_bytes + (uint64_t)kb[u] * 16u + c * (EPL / 2);
        if constexpr (EPL == 8)
          *reinterpret_cast<uint32_t*>(dst) = word;
        else
          *reinterpret_cast<uint16_t*>(dst) = (uint16_t)word;
      }
      if (c == 0 && row[u] < rows_pad && kb[u] < kb_pad)
        sf[sf_offset(row[u], kb[u], n_katoms)] = static_cast<uint8_t>(valid[u] ? byte : 0u);
    }
  }
}

template <int EPL, int SPAN>
cudaError_t launch_wide(const void* x, int64_t rows, int64_t K, int64_t ldx, uint8_t* q,
                        uint8_t* sf, cudaStream_t stream) {
  constexpr int64_t BPW = EPL == 8 ? 8 : 4;
  auto kern = rotate_quantize_wide_kernel<EPL, SPAN>;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  static int per_sm[64] = {};
  static int sms[64] = {};
  if (!per_sm[dev]) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, 0) != cudaSuccess ||
        n <= 0)
      n = 1;
    cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    per_sm[dev] = n;
  }
  const int64_t kb_real = K / 32;
  const int64_t kb_pad = sf_katoms(K) * 4;
  const int64_t rows_pad = sf_row_tiles(rows) * 128;
  const int64_t segs_per_row = (kb_pad + BPW - 1) / BPW;
  const int64_t n_segs = rows_pad * segs_per_row;
  const int64_t warps_needed = (n_segs + kUnroll - 1) / kUnroll;
  const int64_t ctas_needed = (warps_needed + kThreads / 32 - 1) / (kThreads / 32);
  const int64_t cap = (int64_t)sms[dev] * per_sm[dev];
  const int grid = (int)(ctas_needed < cap ? ctas_needed : cap);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, x, (uint64_t)ldx, (uint32_t)rows, (uint32_t)rows_pad,
                            (uint32_t)kb_real, (uint32_t)kb_pad, (uint32_t)segs_per_row,
                            (uint32_t)n_segs, (uint32_t)sf_katoms(K), (uint64_t)(K / 2), q, sf);
}

}  // namespace

cudaError_t launch_rotate_quantize_wide(const void* x, bool x_is_f32, int64_t rows, int64_t K,
                                        int64_t ldx, int span, uint8_t* q, uint8_t* sf,
                                        cudaStream_t stream) {
  // bf16 rows take the tile quantiser (quantize.cu, modes 3 and 4)
  if (!x_is_f32) return cudaErrorNotSupported;
  return span == 64 ? launch_wide<4, 64>(x, rows, K, ldx, q, sf, stream)
                    : launch_wide<4, 128>(x, rows, K, ldx, q, sf, stream);
}

}  // namespace mxfp4
