// quantize.cu -- online block rotation + MXFP4 quantisation (HBM-bound).
//
// Persistent CTAs stream the input through a 4-stage ring of shared-memory
// tiles filled by TMA (128 rows x 128 bytes per tile, 128-byte swizzle): a
// tile holds two 32-element blocks of each of 128 bf16 rows (or one block of
// each of 256 fp32 rows). One thread owns one block: it reads its 64 (128)
// bytes from the swizzled tile -- bank-conflict free because of the swizzle --
// rotates the block in registers, takes the E8M0 scale from the block amax and
// writes 16 bytes of packed E2M1 codes plus one scale byte in the tensor-core
// scale layout. Padding rows / blocks of the scale layout are written as 0.
// Bytes in flight are set by the ring (48-96 KB per SM), not by registers.
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
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "block_quant.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace mxfp4 {
namespace {

using namespace blockq;

constexpr int kThreads = 256;
constexpr uint32_t kStages = 4;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
constexpr int kTimeoutCode = 7;                  // MXFP4_ERR_TIMEOUT

// A stage is BOXES TMA boxes of ROWS rows x 128 bytes, side by side along K (two for
// 128-element Hadamard groups, so that a group is in one stage).
template <bool F32_IN, int MODE = 0>
struct TileShape {
  static constexpr uint32_t BOXES = MODE == 4 ? 2 : 1;
  static constexpr uint32_t ROWS = F32_IN ? 256 : 128;       // rows per TMA box
  static constexpr uint32_t BPR = F32_IN ? 1 : 2 * BOXES;    // 32-element blocks per row per stage
  static constexpr uint32_t BOX_BYTES = ROWS * 128;          // 128 bytes per row
  static constexpr uint32_t STAGE = BOXES * BOX_BYTES;       // bytes per stage
  static constexpr uint32_t STAGES = MODE == 4 ? 3 : kStages;
  static constexpr uint32_t THREADS = MODE == 4 ? 512 : kThreads;  // one per block of a stage
  static constexpr uint32_t SMEM = STAGES * STAGE + 64 + 1024;
};

// Norm prologue (per-row statistics from row_stats_kernel, optional g / b of length K).
struct NormArgs {
  const float* stats;  // [rows][2]: mu, rstd
  const float* g;      // or null (1)
  const float* b;      // or null (0)
};

// MODE 3 / 4 (64- / 128-element Hadamard groups) take bf16 input without norm or NVFP4: a
// group is one (two) 128-byte row chunks of a stage, held by 2 (4) consecutive lanes.
template <int MODE, bool F32_IN, bool NV, bool NORM = false>
__global__ void __launch_bounds__(TileShape<F32_IN, MODE>::THREADS) rotate_quantize_kernel(
    const __grid_constant__ CUtensorMap tmap_x, uint32_t rows, uint32_t rows_pad, uint32_t kb_real,
    uint32_t k_boxes, uint32_t tiles, uint32_t n_katoms, uint64_t q_row_bytes,
    const __grid_constant__ KronCoeffs kc, uint8_t* __restrict__ q, uint8_t* __restrict__ sf,
    int* status, const float* __restrict__ tensor_scale, const NormArgs norm) {
  using namespace sm100;
  using T = TileShape<F32_IN, MODE>;
  constexpr uint32_t kStages = T::STAGES;
  static_assert(MODE < 3 || (!F32_IN && !NV && !NORM), "wide groups: bf16, MXFP4");
  constexpr int CH = F32_IN ? 8 : 4;  // 16-byte chunks per 32-element block
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;  // 128-byte swizzle needs 1024-byte alignment
  const uint32_t bar_full = sbase + kStages * T::STAGE;
  volatile int* abort_flag =
      reinterpret_cast<volatile int*>(smem_raw + (bar_full - raw_addr) + 8 * kStages);

  const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
  // thread -> (row inside the tile, block inside the row's part of the stage)
  const uint32_t r_loc = F32_IN ? warp * 32u + lane
                                : (MODE == 4 ? warp * 8u + (lane >> 2) : warp * 16u + (lane >> 1));
  const uint32_t b_loc = F32_IN ? 0u : (MODE == 4 ? (lane & 3u) : (lane & 1u));
  const uint32_t box = MODE == 4 ? b_loc >> 1 : 0u;     // TMA box of the block
  const uint32_t b_box = MODE == 4 ? b_loc & 1u : b_loc;  // block inside the box row

  if (threadIdx.x == 0) {
    for (uint32_t s = 0; s < kStages; ++s) mbar_init(bar_full + 8 * s, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_x);
  }
  __syncthreads();
  // Launched with programmatic dependent launch: the kernel before this one may still
  // be writing x or reading q / sf. Wait for it to finish before the first access,
  // then let the next kernel start its own set-up.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // NVFP4: the fp32 tensor scale (written by an earlier kernel; waited for above)
  float st = 0.0f;
  if constexpr (NV) st = __ldg(tensor_scale);

  auto issue = [&](uint32_t tile, uint32_t s) {
    const uint32_t rt = tile / k_boxes, kx = tile - rt * k_boxes;
    mbar_arrive_expect_tx(bar_full + 8 * s, T::STAGE);
#pragma unroll
    for (uint32_t bx = 0; bx < T::BOXES; ++bx)
      tma_load_2d(sbase + s * T::STAGE + bx * T::BOX_BYTES, &tmap_x, bar_full + 8 * s,
                  (int32_t)((kx * T::BOXES + bx) * (F32_IN ? 32 : 64)), (int32_t)(rt * T::ROWS));
  };
  uint32_t issued = 0;
  if (threadIdx.x == 0)
    for (uint32_t j = 0; j < kStages; ++j) {
      const uint32_t t = blockIdx.x + j * gridDim.x;
      if (t < tiles) {
        issue(t, j);
        ++issued;
      }
    }

  // tile -> (row tile, k box), advanced incrementally by the grid stride
  const uint32_t step_rt = gridDim.x / k_boxes, step_kx = gridDim.x - step_rt * k_boxes;
  uint32_t rt = blockIdx.x / k_boxes, kx = blockIdx.x - rt * k_boxes;
  uint32_t i = 0;
  for (uint32_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++i) {
    const uint32_t s = i % kStages;
    const bool ok = mbar_wait_bounded(bar_full + 8 * s, (i / kStages) & 1u, abort_flag, kWaitLimitNs);
    if (__syncthreads_or(!ok)) {
      if (threadIdx.x == 0 && status) atomicExch(status, kTimeoutCode);
      break;
    }
    const uint32_t row = rt * T::ROWS + r_loc;
    const uint32_t kb = kx * T::BPR + b_loc;

    float2 P[16];
    const uint32_t rbase = sbase + s * T::STAGE + box * T::BOX_BYTES + r_loc * 128u;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const uint32_t chunk = ((b_box * CH + (uint32_t)c) ^ (r_loc & 7u)) << 4;
      const uint4 w = ld_shared_v4(rbase + chunk);
      if constexpr (F32_IN) {
        P[2 * c + 0] = make_float2(__uint_as_float(w.x), __uint_as_float(w.y));
        P[2 * c + 1] = make_float2(__uint_as_float(w.z), __uint_as_float(w.w));
      } else {
        P[4 * c + 0] = make_float2(bf16_lo(w.x), bf16_hi(w.x));
        P[4 * c + 1] = make_float2(bf16_lo(w.y), bf16_hi(w.y));
        P[4 * c + 2] = make_float2(bf16_lo(w.z), bf16_hi(w.z));
        P[4 * c + 3] = make_float2(bf16_lo(w.w), bf16_hi(w.w));
      }
    }
    __syncthreads();  // every thread has its block in registers: the stage may be refilled
    if (threadIdx.x == 0) {
      const uint32_t next = tile + kStages * gridDim.x;
      if (next < tiles) {
        issue(next, s);
        ++issued;
      }
    }
    if constexpr (MODE == 3) {
      // 64-element Hadamard: the two blocks of a row chunk sit in lanes 2i and 2i + 1.
      // Butterfly strides 1..16 inside each block, stride 32 across the lane pair (lower
      // lane a + b, upper lane a - b, each as one fma with +-1), then the multiply by
      // 1/8. Every lane takes part (the shuffles need the whole warp); rows and blocks
      // past the input only carry zeros and are not stored.
      fwht32(P);
      const float2 sg = b_loc ? make_float2(-1.0f, -1.0f) : make_float2(1.0f, 1.0f);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float2 o;
        o.x = __shfl_xor_sync(0xffffffffu, P[j].x, 1);
        o.y = __shfl_xor_sync(0xffffffffu, P[j].y, 1);
        P[j] = __fmul2_rn(__ffma2_rn(P[j], sg, o), make_float2(0.125f, 0.125f));
      }
    }
    if constexpr (MODE == 4) {
      // 128-element Hadamard: the four blocks of a group sit in lanes 4i .. 4i + 3.
      // Strides 1..16 inside each block, then stride 32 (lanes l, l ^ 1) and stride 64
      // (lanes l, l ^ 2) across lanes as for 64-element groups, then the multiply by the
      // fp32 nearest 1/sqrt(128) (half the fp32 nearest 1/sqrt(32), exactly).
      fwht32(P);
#pragma unroll
      for (uint32_t m = 1; m <= 2; m <<= 1) {
        const float2 sg = (b_loc & m) ? make_float2(-1.0f, -1.0f) : make_float2(1.0f, 1.0f);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          float2 o;
          o.x = __shfl_xor_sync(0xffffffffu, P[j].x, m);
          o.y = __shfl_xor_sync(0xffffffffu, P[j].y, m);
          P[j] = __ffma2_rn(P[j], sg, o);
        }
      }
      const float2 c128 = make_float2(0x1.6a09e6p-4f, 0x1.6a09e6p-4f);
#pragma unroll
      for (int j = 0; j < 16; ++j) P[j] = __fmul2_rn(P[j], c128);
    }

    if (row < rows_pad) {
      if constexpr (NV) {
        // two 16-element groups: scale bytes 2 kb and 2 kb + 1 are adjacent in an atom
        uint32_t b2 = 0;
        if (row < rows && kb < kb_real) {
          if constexpr (MODE == 1) hadamard32(P);
          uint32_t w0[2], w1[2];
          const uint32_t b0 = quantize_group16(&P[0], st, w0);
          const uint32_t b1 = quantize_group16(&P[8], st, w1);
          st_v4(q + (uint64_t)row * q_row_bytes + (uint64_t)kb * 16u,
                make_uint4(w0[0], w0[1], w1[0], w1[1]));
          b2 = b0 | (b1 << 8);
        }
        if (2u * kb < 4u * n_katoms)
          *reinterpret_cast<uint16_t*>(sf + sf_offset(row, 2u * kb, n_katoms)) = (uint16_t)b2;
      } else {
        uint32_t byte = 0;
        if (row < rows && kb < kb_real) {
          if constexpr (NORM) {
            // v = ((x - mu) * rstd) * g + b, each an fp32 operation in that order
            const float2 st = __ldg(reinterpret_cast<const float2*>(norm.stats) + row);
            const float2 nmu = make_float2(-st.x, -st.x), rs = make_float2(st.y, st.y);
#pragma unroll
            for (int j = 0; j < 16; ++j) P[j] = __fmul2_rn(__fadd2_rn(P[j], nmu), rs);
            if (norm.g != nullptr) {
              const float2* gv = reinterpret_cast<const float2*>(norm.g + kb * 32u);
#pragma unroll
              for (int j = 0; j < 16; ++j) P[j] = __fmul2_rn(P[j], __ldg(gv + j));
            }
            if (norm.b != nullptr) {
              const float2* bv = reinterpret_cast<const float2*>(norm.b + kb * 32u);
#pragma unroll
              for (int j = 0; j < 16; ++j) P[j] = __fadd2_rn(P[j], __ldg(bv + j));
            }
          }
          if constexpr (MODE == 1) hadamard32(P);
          if constexpr (MODE == 2) kron32(P, kc);
          uint4 codes;
          byte = quantize_block(P, codes);
          st_v4(q + (uint64_t)row * q_row_bytes + (uint64_t)kb * 16u, codes);
        }
        sf[sf_offset(row, kb, n_katoms)] = static_cast<uint8_t>(byte);
      }
    }
    kx += step_kx;
    rt += step_rt;
    if (kx >= k_boxes) {
      kx -= k_boxes;
      ++rt;
    }
  }
  // After an early stop, loads already issued still land in this CTA's shared memory.
  if (threadIdx.x == 0 && *abort_flag) {
    volatile int never = 0;
    for (uint32_t j = i; j < issued; ++j)
      mbar_wait_bounded(bar_full + 8 * (j % kStages), (j / kStages) & 1u, &never, kWaitLimitNs);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

template <int MODE, bool F32_IN, bool NV = false, bool NORM = false>
cudaError_t launch_mode(const void* x, int64_t rows, int64_t K, int64_t ldx, const KronCoeffs& kc,
                        uint8_t* q, uint8_t* sf, int* status, cudaStream_t stream,
                        const float* tensor_scale = nullptr, NormArgs norm = NormArgs{}) {
  using T = TileShape<F32_IN, MODE>;
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  CUtensorMap map;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ldx * (F32_IN ? 4u : 2u)};
  cuuint32_t box[2] = {F32_IN ? 32u : 64u, T::ROWS};
  cuuint32_t estr[2] = {1, 1};
  if (fn(&map, F32_IN ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
         const_cast<void*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  auto kern = rotate_quantize_kernel<MODE, F32_IN, NV, NORM>;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  static int per_sm[64] = {};
  static int sms[64] = {};
  if (!per_sm[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, T::SMEM);
    if (e != cudaSuccess) return e;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, T::THREADS, T::SMEM) !=
            cudaSuccess ||
        n <= 0)
      n = 1;
    cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    per_sm[dev] = n;
  }
  const int64_t kb_real = K / 32;
  const int64_t kb_pad = sf_katoms(K) * 4;
  const int64_t rows_pad = sf_row_tiles(rows) * 128;
  const int64_t k_boxes = kb_pad / T::BPR;
  const int64_t row_tiles = (rows_pad + T::ROWS - 1) / T::ROWS;
  const int64_t tiles = row_tiles * k_boxes;
  const int64_t cap = (int64_t)sms[dev] * per_sm[dev];
  const int grid = (int)(tiles < cap ? tiles : cap);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(T::THREADS);
  cfg.dynamicSmemBytes = T::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // scale atoms per 128-row group: 4 scales each, of 32 (MXFP4) or 16 (NVFP4) elements
  const uint32_t n_katoms = (uint32_t)sf_katoms(NV ? 2 * K : K);
  return cudaLaunchKernelEx(&cfg, kern, map, (uint32_t)rows, (uint32_t)rows_pad,
                            (uint32_t)kb_real, (uint32_t)k_boxes, (uint32_t)tiles, n_katoms,
                            (uint64_t)(K / 2), kc, q, sf, status, tensor_scale, norm);
}

// NVFP4 tensor scale: amax of the (rotated) tensor by a grid-stride pass with one
// atomicMax per warp on the fp32 bits (non-negative floats order like their bits, and
// max is order-free, so the result is deterministic), then st = amax / (6 * 448).
template <int MODE, bool F32_IN>
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const void* __restrict__ x, uint64_t ldx,
                                                         uint32_t rows, uint32_t kb_real,
                                                         unsigned int* __restrict__ amax_bits,
                                                         unsigned int* done, float* scale_out) {
  const uint64_t n = (uint64_t)rows * kb_real;
  float m = 0.0f;
  for (uint64_t b = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; b < n;
       b += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t row = b / kb_real, kb = b - row * kb_real;
    float2 P[16];
    if constexpr (F32_IN) {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(x) +
                                                          row * ldx + kb * 32u);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float4 w = __ldcs(src + c);
        P[2 * c] = make_float2(w.x, w.y);
        P[2 * c + 1] = make_float2(w.z, w.w);
      }
    } else {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) +
                                                        row * ldx + kb * 32u);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 w = __ldcs(src + c);
        P[4 * c + 0] = make_float2(bf16_lo(w.x), bf16_hi(w.x));
        P[4 * c + 1] = make_float2(bf16_lo(w.y), bf16_hi(w.y));
        P[4 * c + 2] = make_float2(bf16_lo(w.z), bf16_hi(w.z));
        P[4 * c + 3] = make_float2(bf16_lo(w.w), bf16_hi(w.w));
      }
    }
    if constexpr (MODE == 1) hadamard32(P);
#pragma unroll
    for (int j = 0; j < 16; ++j) m = fmaxf(m, fmaxf(fabsf(P[j].x), fabsf(P[j].y)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31u) == 0) atomicMax(amax_bits, __float_as_uint(m));
  // The last block to finish turns the maximum into the scale and leaves the maximum (and
  // a separate counter) zero for the next pass. `done` may be scale_out itself, which
  // the caller zeroed; the scale then simply replaces it.
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(done, 1u) == gridDim.x - 1u) {
      __threadfence();
      const unsigned int bits = atomicExch(amax_bits, 0u);
      if (done != reinterpret_cast<unsigned int*>(scale_out)) atomicExch(done, 0u);
      scale_out[0] = __fdiv_rn(__uint_as_float(bits), 2688.0f);
    }
  }
}

// Norm prologue statistics: one warp per bf16 row, two passes (sum, then squared
// deviations; RMSNorm: squares), fp32 sums, mu = sum / K, rstd = 1 / sqrt(var + eps)
// correctly rounded. The quantiser applies them; the oracle checks them against exact
// arithmetic and repeats the per-element steps with these fp32 values.
template <int KIND>
__global__ void __launch_bounds__(256) row_stats_kernel(const uint16_t* __restrict__ x,
                                                        uint64_t ldx, uint32_t rows, uint32_t K,
                                                        float eps, float* __restrict__ stats) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t row = blockIdx.x * 8u + (threadIdx.x >> 5);
  if (row >= rows) return;
  const uint16_t* xr = x + (uint64_t)row * ldx;
  // Each lane reads 8 elements at k, k + 256, k + 512, k + 768 per step (4 loads in flight)
  // into 4 independent partial sums, added in a fixed order at the end.
  float mu = 0.0f;
  if constexpr (KIND == 0) {
    float s4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (uint32_t k0 = lane * 8u; k0 < K; k0 += 1024u) {
      uint4 w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (k0 + 256u * j < K) w[j] = __ldg(reinterpret_cast<const uint4*>(xr + k0 + 256u * j));
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (k0 + 256u * j < K)
          s4[j] += bf16_lo(w[j].x) + bf16_hi(w[j].x) + bf16_lo(w[j].y) + bf16_hi(w[j].y) +
                   bf16_lo(w[j].z) + bf16_hi(w[j].z) + bf16_lo(w[j].w) + bf16_hi(w[j].w);
    }
    float s = (s4[0] + s4[1]) + (s4[2] + s4[3]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    mu = __fdiv_rn(s, (float)K);
  }
  float v4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (uint32_t k0 = lane * 8u; k0 < K; k0 += 1024u) {
    uint4 w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (k0 + 256u * j < K) w[j] = __ldg(reinterpret_cast<const uint4*>(xr + k0 + 256u * j));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (k0 + 256u * j >= K) continue;
      const float e[8] = {bf16_lo(w[j].x), bf16_hi(w[j].x), bf16_lo(w[j].y), bf16_hi(w[j].y),
                          bf16_lo(w[j].z), bf16_hi(w[j].z), bf16_lo(w[j].w), bf16_hi(w[j].w)};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float d = e[i] - mu;
        v4[j] = __fmaf_rn(d, d, v4[j]);
      }
    }
  }
  float v = (v4[0] + v4[1]) + (v4[2] + v4[3]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) {
    stats[2u * row] = mu;
    stats[2u * row + 1u] = __frsqrt_rn(__fadd_rn(__fdiv_rn(v, (float)K), eps));
  }
}

}  // namespace

cudaError_t launch_norm_rotate_quantize(const void* x, int64_t rows, int64_t K, int64_t ldx,
                                       int kind, float eps, const float* g, const float* b,
                                       int mode, const KronCoeffs* kc, uint8_t* q, uint8_t* sf,
                                       float* stats, int* status, cudaStream_t stream) {
  // One pass (quantize_norm.cu) while two buffers of a row fit one SM's shared memory.
  if (norm_one_pass(K))
    return launch_norm_one_pass(x, rows, K, ldx, kind, eps, g, b, mode, kc, q, sf, stats, status,
                                stream);
  // Longer rows: statistics kernel, then the quantiser in its norm form.
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)((rows + 7) / 8));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  cudaError_t e =
      kind == 1 ? cudaLaunchKernelEx(&cfg, row_stats_kernel<1>, xb, (uint64_t)ldx, (uint32_t)rows,
                                     (uint32_t)K, eps, stats)
                : cudaLaunchKernelEx(&cfg, row_stats_kernel<0>, xb, (uint64_t)ldx, (uint32_t)rows,
                                     (uint32_t)K, eps, stats);
  if (e != cudaSuccess) return e;
  KronCoeffs k{};
  if (kc) k = *kc;
  const NormArgs na{stats, g, b};
  if (mode == 1)
    return launch_mode<1, false, false, true>(x, rows, K, ldx, k, q, sf, status, stream, nullptr,
                                              na);
  if (mode == 2)
    return launch_mode<2, false, false, true>(x, rows, K, ldx, k, q, sf, status, stream, nullptr,
                                              na);
  return launch_mode<0, false, false, true>(x, rows, K, ldx, k, q, sf, status, stream, nullptr,
                                            na);
}

cudaError_t launch_nvfp4_tensor_scale(const void* x, bool x_is_f32, int64_t rows, int64_t K,
                                     int64_t ldx, int mode, float* scale2, cudaStream_t stream,
                                     unsigned int* state) {
  // With `state` (two words, zero, left zero): one kernel. Without: scale2[0] serves as
  // the block counter and scale2[1] as the running maximum, zeroed first.
  unsigned int* bits;
  unsigned int* done;
  if (state != nullptr) {
    bits = state;
    done = state + 1;
  } else {
    cudaError_t e = cudaMemsetAsync(scale2, 0, 2 * sizeof(float), stream);
    if (e != cudaSuccess) return e;
    done = reinterpret_cast<unsigned int*>(scale2);
    bits = reinterpret_cast<unsigned int*>(scale2 + 1);
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const uint64_t blocks = (uint64_t)rows * (uint64_t)(K / 32);
  uint64_t grid = (blocks + 255) / 256;
  if (grid > (uint64_t)sms * 8) grid = (uint64_t)sms * 8;
  if (grid == 0) grid = 1;
  const unsigned g = (unsigned)grid;
  if (x_is_f32) {
    if (mode == 1)
      nvfp4_amax_kernel<1, true><<<g, 256, 0, stream>>>(x, ldx, rows, K / 32, bits, done, scale2);
    else
      nvfp4_amax_kernel<0, true><<<g, 256, 0, stream>>>(x, ldx, rows, K / 32, bits, done, scale2);
  } else {
    if (mode == 1)
      nvfp4_amax_kernel<1, false><<<g, 256, 0, stream>>>(x, ldx, rows, K / 32, bits, done, scale2);
    else
      nvfp4_amax_kernel<0, false><<<g, 256, 0, stream>>>(x, ldx, rows, K / 32, bits, done, scale2);
  }
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_quantize(const void* x, bool x_is_f32, int64_t rows, int64_t K,
                                  int64_t ldx, int mode, const float* tensor_scale, uint8_t* q,
                                  uint8_t* sf, int* status, cudaStream_t stream) {
  const KronCoeffs k{};
  if (x_is_f32)
    return mode == 1 ? launch_mode<1, true, true>(x, rows, K, ldx, k, q, sf, status, stream,
                                                  tensor_scale)
                     : launch_mode<0, true, true>(x, rows, K, ldx, k, q, sf, status, stream,
                                                  tensor_scale);
  return mode == 1 ? launch_mode<1, false, true>(x, rows, K, ldx, k, q, sf, status, stream,
                                                 tensor_scale)
                   : launch_mode<0, false, true>(x, rows, K, ldx, k, q, sf, status, stream,
                                                 tensor_scale);
}

cudaError_t launch_rotate_quantize(const void* x, bool x_is_f32, int64_t rows, int64_t K,
                                   int64_t ldx, int mode, const KronCoeffs* kc, uint8_t* q,
                                   uint8_t* sf, int* status, cudaStream_t stream) {
  KronCoeffs k{};
  if (kc) k = *kc;
  // 64- / 128-element groups of bf16 rows: the tile kernel (a group is one or two row
  // chunks of a stage); fp32 input (weight preparation): the warp-shuffle kernel.
  if (mode == 3 && !x_is_f32)
    return launch_mode<3, false>(x, rows, K, ldx, k, q, sf, status, stream);
  if (mode == 4 && !x_is_f32)
    return launch_mode<4, false>(x, rows, K, ldx, k, q, sf, status, stream);
  if (mode == 3 || mode == 4)
    return launch_rotate_quantize_wide(x, x_is_f32, rows, K, ldx, (int)rotation_span(mode), q, sf,
                                       stream);
  if (x_is_f32) {
    if (mode == 1) return launch_mode<1, true>(x, rows, K, ldx, k, q, sf, status, stream);
    if (mode == 2) return launch_mode<2, true>(x, rows, K, ldx, k, q, sf, status, stream);
    return launch_mode<0, true>(x, rows, K, ldx, k, q, sf, status, stream);
  }
  if (mode == 1) return launch_mode<1, false>(x, rows, K, ldx, k, q, sf, status, stream);
  if (mode == 2) return launch_mode<2, false>(x, rows, K, ldx, k, q, sf, status, stream);
  return launch_mode<0, false>(x, rows, K, ldx, k, q, sf, status, stream);
}

}  // namespace mxfp4
