// quantize_norm.cu -- the norm prologue in one pass over x: LayerNorm / RMSNorm
// statistics, normalisation, online rotation and MXFP4 quantisation of bf16 rows.
//
// One CTA per SM (512 threads) walks groups of R whole rows. Each group is copied
// into shared memory by one bulk copy per row while the previous group is being
// worked on (two row buffers); the CTA then takes every row's statistics from
// that copy (16 / R warps per row, partial sums combined in a fixed order) and
// normalises, rotates and quantises all of the group's 32-element blocks from the
// same copy. x is read from HBM once, where a statistics kernel followed by the
// quantiser would read it twice.
//
// Method: the normalisation that makes the transform online ("KroQuant:
// Effiziente Post-Training-Quantisierung fuer Diffusion Transformers mittels
// Kronecker-Produkt-Struktur", "Hintergrund"), then the block rotation and the
// MXFP4 quantisation of the quantiser ("Bridging the Gap Between Promise and
// Performance for Microscaling FP4 Quantization", "Methodologie: MR-GPTQ" item
// 1; "What is MXFP4 and why does it eliminate dequantization overhead?").
//
// Per element, v = ((x - mu) * rstd) * g + b, each an fp32 operation in that
// order, as in the quantiser's norm form, so codes and scales are bit-identical
// to a sequential fp32 evaluation with the same statistics. The statistics are
// fp32 sums in this kernel's own order (mu = sum / K, var = sum (x - mu)^2 / K,
// rstd = 1 / sqrt(var + eps) correctly rounded; RMSNorm: mu = 0).
#include <cuda_runtime.h>

#include <cstdint>

#include "block_quant.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace mxfp4 {
namespace {

using namespace blockq;

constexpr uint32_t kNormThreads = 512;
constexpr uint32_t kNormWarps = kNormThreads / 32;
constexpr uint32_t kNormBufBudget = 200 * 1024;  // both row buffers; one CTA per SM
constexpr uint64_t kNormWaitLimitNs = 2000000000ull;
constexpr int kNormTimeoutCode = 7;  // MXFP4_ERR_TIMEOUT

// Rows per group: the largest power of two <= 16 whose two buffers of rows (2K bytes
// plus a 16-byte pad each) fit the budget; 0 if one row per buffer does not fit.
uint32_t rows_per_group(int64_t K) {
  const uint64_t pitch = (uint64_t)K * 2 + 16;
  uint32_t R = 16;
  while (R > 1 && 2ull * R * pitch > kNormBufBudget) R >>= 1;
  return 2ull * R * pitch <= kNormBufBudget ? R : 0;
}

// Shared memory: [row buffer 0 | row buffer 1] (R rows each, `pitch` bytes apart: the
// 16-byte pad puts consecutive rows on different bank groups), two mbarriers, the abort
// flag, per-row (mu, rstd), per-warp partial sums.
struct NormSmem {
  uint32_t pitch, buf_bytes, bar, abort_off, st_off, part_off, total;
  __host__ __device__ NormSmem(uint32_t K, uint32_t R) {
    pitch = K * 2u + 16u;
    buf_bytes = R * pitch;
    bar = 2u * buf_bytes;  // two 8-byte mbarriers
    abort_off = bar + 16u;
    st_off = abort_off + 16u;
    part_off = st_off + 16u * 8u;
    total = part_off + kNormWarps * 4u;
  }
};

template <int KIND, int MODE>
__global__ void __launch_bounds__(kNormThreads, 1) norm_rows_kernel(
    const uint16_t* __restrict__ x, uint64_t ldx, uint32_t rows, uint32_t rows_pad, uint32_t K,
    uint32_t R, uint32_t n_katoms, float eps, const __grid_constant__ KronCoeffs kc,
    const float* __restrict__ g, const float* __restrict__ b, uint8_t* __restrict__ q,
    uint8_t* __restrict__ sf, float* __restrict__ stats, int* status) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_addr(smem_raw) + 127u) & ~127u;
  uint8_t* sptr = smem_raw + (sbase - smem_addr(smem_raw));
  const NormSmem L(K, R);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + L.abort_off);
  float2* st_s = reinterpret_cast<float2*>(sptr + L.st_off);
  float* part = reinterpret_cast<float*>(sptr + L.part_off);
  const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
  const uint32_t row_bytes = K * 2u;  // a multiple of 64 (K % 32 == 0)
  const uint32_t chunks = row_bytes / 16u;
  const uint32_t kb_real = K / 32u, kb_pad = n_katoms * 4u;
  const uint32_t n_groups = rows_pad / R;
  const uint32_t W = kNormWarps / R;  // warps per row in the statistics passes

  if (tid == 0) {
    mbar_init(sbase + L.bar, 1);
    mbar_init(sbase + L.bar + 8u, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Launched with programmatic dependent launch: the kernel before this one may still be
  // writing x or reading q / sf / stats. Wait for it before the first access.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  auto real_rows = [&](uint32_t grp) -> uint32_t {
    const uint32_t row0 = grp * R;
    return row0 >= rows ? 0u : (rows - row0 < R ? rows - row0 : R);
  };
  uint32_t pending = 0;  // thread 0: bit i set while a copy into buffer i is in flight
  auto issue = [&](uint32_t grp, uint32_t bi) {
    const uint32_t n = real_rows(grp);
    if (n == 0) return;
    const uint32_t bar = sbase + L.bar + 8u * bi;
    mbar_arrive_expect_tx(bar, n * row_bytes);
    for (uint32_t r = 0; r < n; ++r)
      bulk_load(sbase + bi * L.buf_bytes + r * L.pitch, x + (uint64_t)(grp * R + r) * ldx,
                row_bytes, bar);
    pending |= 1u << bi;
  };

  uint32_t phase = 0;  // bit i: parity of buffer i's next completion
  bool aborted = false;
  if (tid == 0 && blockIdx.x < n_groups) issue(blockIdx.x, 0);
  uint32_t it = 0;
  for (uint32_t grp = blockIdx.x; grp < n_groups; grp += gridDim.x, ++it) {
    const uint32_t bi = it & 1u;
    // The other buffer was released by the barrier that ended the previous group.
    if (tid == 0 && grp + gridDim.x < n_groups) issue(grp + gridDim.x, bi ^ 1u);
    const uint32_t row0 = grp * R;
    const uint32_t nreal = real_rows(grp);
    const uint32_t buf = sbase + bi * L.buf_bytes;
    if (nreal > 0) {
      const bool ok = mbar_wait_bounded(sbase + L.bar + 8u * bi, (phase >> bi) & 1u,
                                        abort_flag, kNormWaitLimitNs);
      if (__syncthreads_or(!ok)) {
        if (tid == 0 && status) atomicExch(status, kNormTimeoutCode);
        aborted = true;
        break;
      }
      phase ^= 1u << bi;
      if (tid == 0) pending &= ~(1u << bi);

      // Statistics: warp w takes slice w % W of row w / W; lane l takes the 16-byte chunks
      // (w % W) 32 + l + 32 W i, i = 0, 1, ..., into four partial sums by i mod 4 (each
      // adds a chunk's 8 elements in order), added as (p0 + p1) + (p2 + p3); the warp's
      // lanes are then added by a butterfly and the W slices of a row in slice order.
      const uint32_t r = warp / W, sl = warp - r * W;
      const uint32_t rbase = buf + r * L.pitch;
      const uint32_t cstep = 32u * W;
      float mu = 0.0f;
      if constexpr (KIND == 0) {
        float p4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (r < nreal)
          for (uint32_t c0 = sl * 32u + lane; c0 < chunks; c0 += 4u * cstep) {
#pragma unroll
            for (uint32_t j = 0; j < 4; ++j) {
              const uint32_t c = c0 + j * cstep;
              if (c < chunks) {
                const uint4 w = ld_shared_v4(rbase + c * 16u);
                p4[j] += bf16_lo(w.x) + bf16_hi(w.x) + bf16_lo(w.y) + bf16_hi(w.y) +
                         bf16_lo(w.z) + bf16_hi(w.z) + bf16_lo(w.w) + bf16_hi(w.w);
              }
            }
          }
        float s = (p4[0] + p4[1]) + (p4[2] + p4[3]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) part[warp] = s;
        __syncthreads();
        if (tid < nreal) {
          float t = part[tid * W];
          for (uint32_t k = 1; k < W; ++k) t += part[tid * W + k];
          st_s[tid].x = __fdiv_rn(t, (float)K);
        }
        __syncthreads();
        if (r < nreal) mu = st_s[r].x;
      }
      float q4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      if (r < nreal)
        for (uint32_t c0 = sl * 32u + lane; c0 < chunks; c0 += 4u * cstep) {
#pragma unroll
          for (uint32_t j = 0; j < 4; ++j) {
            const uint32_t c = c0 + j * cstep;
            if (c < chunks) {
              const uint4 w = ld_shared_v4(rbase + c * 16u);
              const float e[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                                  bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float d = e[i] - mu;
                q4[j] = __fmaf_rn(d, d, q4[j]);
              }
            }
          }
        }
      float v = (q4[0] + q4[1]) + (q4[2] + q4[3]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) part[warp] = v;
      __syncthreads();
      if (tid < nreal) {
        float t = part[tid * W];
        for (uint32_t k = 1; k < W; ++k) t += part[tid * W + k];
        const float m = KIND == 0 ? st_s[tid].x : 0.0f;
        const float rstd = __frsqrt_rn(__fadd_rn(__fdiv_rn(t, (float)K), eps));
        st_s[tid] = make_float2(m, rstd);
        stats[2u * (row0 + tid)] = m;
        stats[2u * (row0 + tid) + 1u] = rstd;
      }
      __syncthreads();

      // Blocks: thread i takes blocks i, i + 512, ... of the group, row index fastest,
      // so the 16-byte reads of a warp fall on every bank group.
      for (uint32_t blk = tid; blk < nreal * kb_real; blk += kNormThreads) {
        const uint32_t kb = blk / nreal, rr = blk - kb * nreal;
        const uint32_t baddr = buf + rr * L.pitch + kb * 64u;
        float2 P[16];
#pragma unroll
        for (uint32_t c = 0; c < 4; ++c) {
          const uint4 w = ld_shared_v4(baddr + c * 16u);
          P[4 * c + 0] = make_float2(bf16_lo(w.x), bf16_hi(w.x));
          P[4 * c + 1] = make_float2(bf16_lo(w.y), bf16_hi(w.y));
          P[4 * c + 2] = make_float2(bf16_lo(w.z), bf16_hi(w.z));
          P[4 * c + 3] = make_float2(bf16_lo(w.w), bf16_hi(w.w));
        }
        const float2 stv = st_s[rr];
        const float2 nmu = make_float2(-stv.x, -stv.x), rs = make_float2(stv.y, stv.y);
#pragma unroll
        for (int j = 0; j < 16; ++j) P[j] = __fmul2_rn(__fadd2_rn(P[j], nmu), rs);
        if (g != nullptr) {  // 16-byte loads: g and b are 16-byte aligned, kb 32 floats apart
          const float4* gv = reinterpret_cast<const float4*>(g + kb * 32u);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 t = __ldg(gv + j);
            P[2 * j] = __fmul2_rn(P[2 * j], make_float2(t.x, t.y));
            P[2 * j + 1] = __fmul2_rn(P[2 * j + 1], make_float2(t.z, t.w));
          }
        }
        if (b != nullptr) {
          const float4* bv = reinterpret_cast<const float4*>(b + kb * 32u);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 t = __ldg(bv + j);
            P[2 * j] = __fadd2_rn(P[2 * j], make_float2(t.x, t.y));
            P[2 * j + 1] = __fadd2_rn(P[2 * j + 1], make_float2(t.z, t.w));
          }
        }
        if constexpr (MODE == 1) hadamard32(P);
        if constexpr (MODE == 2) kron32(P, kc);
        uint4 codes;
        const uint32_t byte = quantize_block(P, codes);
        st_v4(q + (uint64_t)(row0 + rr) * (K / 2u) + (uint64_t)kb * 16u, codes);
        sf[sf_offset(row0 + rr, kb, n_katoms)] = static_cast<uint8_t>(byte);
      }
    }
    // Padding of the scale layout: blocks kb_real..kb_pad of real rows, every block of
    // the padding rows (>= rows) of this group.
    const uint32_t pad_real = kb_pad - kb_real;
    for (uint32_t i = tid; i < nreal * pad_real + (R - nreal) * kb_pad; i += kNormThreads) {
      uint32_t rr, kb;
      if (i < nreal * pad_real) {
        rr = i / pad_real;
        kb = kb_real + (i - rr * pad_real);
      } else {
        const uint32_t j = i - nreal * pad_real;
        rr = nreal + j / kb_pad;
        kb = j - (rr - nreal) * kb_pad;
      }
      sf[sf_offset(row0 + rr, kb, n_katoms)] = 0;
    }
    __syncthreads();  // this buffer is read: the next-but-one group may be copied into it
  }
  // After an early stop, copies already issued still land in this CTA's shared memory.
  if (aborted && tid == 0) {
    volatile int never = 0;
    for (uint32_t bi = 0; bi < 2; ++bi)
      if ((pending >> bi) & 1u)
        mbar_wait_bounded(sbase + L.bar + 8u * bi, (phase >> bi) & 1u, &never, kNormWaitLimitNs);
  }
}

template <int KIND, int MODE>
cudaError_t launch_kind_mode(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx, float eps,
                             const KronCoeffs& kc, const float* g, const float* b, uint8_t* q,
                             uint8_t* sf, float* stats, int* status, uint32_t R,
                             cudaStream_t stream) {
  auto kern = norm_rows_kernel<KIND, MODE>;
  const size_t smem = 128 + NormSmem((uint32_t)K, R).total;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  static size_t smem_set[64] = {};
  static int sms[64] = {};
  if (smem_set[dev] < smem) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    smem_set[dev] = smem;
  }
  if (!sms[dev]) cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
  const int64_t rows_pad = sf_row_tiles(rows) * 128;
  const int64_t groups = rows_pad / R;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(groups < sms[dev] ? groups : sms[dev]));
  cfg.blockDim = dim3(kNormThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, x, (uint64_t)ldx, (uint32_t)rows, (uint32_t)rows_pad,
                            (uint32_t)K, R, (uint32_t)sf_katoms(K), eps, kc, g, b, q, sf, stats,
                            status);
}

}  // namespace

bool norm_one_pass(int64_t K) { return rows_per_group(K) != 0; }

cudaError_t launch_norm_one_pass(const void* x, int64_t rows, int64_t K, int64_t ldx, int kind,
                                 float eps, const float* g, const float* b, int mode,
                                 const KronCoeffs* kc, uint8_t* q, uint8_t* sf, float* stats,
                                 int* status, cudaStream_t stream) {
  const uint32_t R = rows_per_group(K);
  if (R == 0) return cudaErrorNotSupported;
  KronCoeffs k{};
  if (kc) k = *kc;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
#define MXFP4_NORM_ROWS(KINDV, MODEV)                                                  \
  return launch_kind_mode<KINDV, MODEV>(xb, rows, K, ldx, eps, k, g, b, q, sf, stats, \
                                        status, R, stream)
  if (kind == 1) {
    if (mode == 1) MXFP4_NORM_ROWS(1, 1);
    if (mode == 2) MXFP4_NORM_ROWS(1, 2);
    MXFP4_NORM_ROWS(1, 0);
  }
  if (mode == 1) MXFP4_NORM_ROWS(0, 1);
  if (mode == 2) MXFP4_NORM_ROWS(0, 2);
  MXFP4_NORM_ROWS(0, 0);
#undef MXFP4_NORM_ROWS
}

}  // namespace mxfp4
