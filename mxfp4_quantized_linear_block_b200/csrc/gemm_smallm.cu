// gemm_smallm.cu -- block-scaled MXFP4 GEMM for a few activation rows (M <= 128).
//
// With few tokens the layer is a stream over the weights (HBM-bound), so the
// roles of the operands are swapped: a 128-row tile of W is the MMA's M side
// and the (padded) tokens are its N side, tcgen05.mma.kind::mxf4 M=128 x N=NT
// (NT = 16, 32, 64 or 128) x K=64. K is split S ways (1 <= S <= 8) so that
// (W tiles x S) CTAs stream the weights through all SMs at once.
//
// The S CTAs of one W tile form a thread-block cluster. Each accumulates its K
// range in tensor memory and leaves the fp32 partial [NT tokens x 128 columns]
// in its own shared memory (over the drained operand stages). After a cluster
// barrier, CTA r adds the S partials of its share of the 128 columns through
// distributed shared memory, in split order 0, 1, ..., S-1 (deterministic),
// and writes that part of Y with coalesced row stores. No atomics, no second
// kernel. For more than 32 tokens and 4 or more splits the partials are large
// (up to 64 KB per CTA, mostly remote) and distributed shared memory moves them
// at only a few tens of GB/s per SM, so they go through L2 instead: each CTA
// writes its partial rows to a global scratch, and after the cluster barrier
// (release / acquire at cluster scope) CTA r reads its share of all S partials
// from L2 and adds them in the same order, so both forms give the same bits.
//
// The whole layer for up to 8 tokens (FX variant): the CTA's epilogue warps
// rotate and quantise the CTA's K range of the bf16 activations themselves,
// straight into the B-operand layout in shared memory, while the weight stream
// is in flight -- no separate quantiser kernel, no activation round trip
// through global memory, and the weight stream starts as soon as the kernel
// before the layer has finished.
//
// ("AMD Quark delivers MXFP4 quantization for FLUX.1-dev on Instinct MI350
// with 1.92x speedup", opening section: MXFP4 GEMM without dequantisation;
// "Bridging the Gap Between Promise and Performance for Microscaling FP4
// Quantization", "GPU Kernel Ondersteuning (QuTLASS)".)
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "block_quant.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace mxfp4 {
namespace {

using namespace sm100;

constexpr uint32_t kThreads = 192;  // warp 0: TMA, warp 1: MMA, warps 2-5: epilogue
constexpr uint32_t kFirstEpiWarp = 2;
constexpr uint32_t kMaxSplits = 8;  // portable cluster size
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kTimeoutCode = 7;
// Fused layer: at most this many k-tiles (256 elements) of activations per CTA, all
// resident in shared memory at once, and at most this many rows. Every CTA of a K split
// reads the same slice of x, so the reads grow with the rows times the W tiles; beyond 8
// rows (B200, 4096 <-> 14336) they slow the weight stream more than the separate
// quantiser launch costs.
constexpr uint32_t kFxMaxKt = 12;
constexpr int64_t kFxMaxRows = 8;

template <uint32_t NT, bool NV = false, bool FX = false>
struct SmallConfig {
  // scale atoms (128 rows x 4 scales) per k-tile of 256 elements: 2 for MXFP4, 4 for NVFP4
  static constexpr uint32_t AT = NV ? 4 : 2;
  static constexpr uint32_t A_STAGE = 128 * 128;          // 128 rows of W x 256 elements
  static constexpr uint32_t B_STAGE = FX ? 0 : NT * 128;  // NT token rows x 256 elements
  static constexpr uint32_t SF_STAGE = AT * 512;          // AT scale atoms
  // FX: the quantised activations of the CTA's whole K range (B-operand tiles and their
  // scale atoms, one of each per k-tile), written by the CTA itself.
  static constexpr uint32_t XQ_KT = NT * 128;
  static constexpr uint32_t XQ_BYTES = FX ? kFxMaxKt * XQ_KT : 0;
  static constexpr uint32_t XSF_BYTES = FX ? kFxMaxKt * SF_STAGE : 0;
  // Up to 64 tokens two CTAs per SM: as many stages (at most 5) as let 2 x SMEM_BYTES fit
  // an SM's shared memory (233472 bytes, 1 KB of it reserved per CTA). 128 tokens: one
  // CTA per SM with as many stages as fit (6 of the 12 allowed), so that half as many K
  // splits keep the same bytes in flight (B200, 128 x 14336 <-> 4096: 12.4 / 12.6 -> 11.8 /
  // 11.0 us; at 1 and 16 tokens the same change cost 0.2-0.8 us, the sums being small there).
  static constexpr bool WIDE = NT == 128;
  static constexpr uint32_t STAGE_BYTES = A_STAGE + B_STAGE + (FX ? 1 : 2) * SF_STAGE;
  static constexpr uint32_t BUDGET =
      (WIDE ? 232448 : 116736) - 1024 - 1024 - 512 - XQ_BYTES - XSF_BYTES;
  static constexpr uint32_t MAX_STAGES = WIDE ? 12 : 5;
  static constexpr uint32_t STAGES =
      BUDGET / STAGE_BYTES < MAX_STAGES ? BUDGET / STAGE_BYTES : MAX_STAGES;
  static constexpr uint32_t OFF_A = 0;
  static constexpr uint32_t OFF_B = OFF_A + STAGES * A_STAGE;
  static constexpr uint32_t OFF_XQ = OFF_B + STAGES * B_STAGE;
  static constexpr uint32_t OFF_SFA = OFF_XQ + XQ_BYTES;
  static constexpr uint32_t OFF_SFB = OFF_SFA + STAGES * SF_STAGE;
  static constexpr uint32_t OFF_XSF = OFF_SFB + (FX ? 0 : STAGES * SF_STAGE);
  static constexpr uint32_t OFF_BAR = OFF_XSF + XSF_BYTES;
  static constexpr uint32_t NUM_BARS = 2 * STAGES + 2 + (FX ? kFxMaxKt : 0);
  static constexpr uint32_t OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;
  // fp32 partial [NT][128] at offset 0, over the A/B stages once every MMA has completed
  static constexpr uint32_t RED_BYTES = NT * 128 * 4;
  static constexpr uint32_t SFA_COL = NT;
  static constexpr uint32_t SFB_COL = NT + 4 * AT;
  static constexpr uint32_t COLS_USED = NT + 8 * AT;
  static constexpr uint32_t TMEM_COLS = COLS_USED <= 32 ? 32 : COLS_USED <= 64 ? 64
                                        : COLS_USED <= 128 ? 128 : 256;
  static_assert(NT % 16 == 0 && NT >= 16 && NT <= 128, "token tile");
  static_assert(RED_BYTES <= OFF_SFA, "partial fits over the operand stages");
  static_assert(!FX || (!NV && STAGES >= 3), "fused layer: MXFP4, a ring of 3 or more");
  static_assert(OFF_XQ % 1024 == 0 && XQ_KT % 1024 == 0, "128-byte swizzle atoms");
  static_assert(WIDE ? SMEM_BYTES <= 232448 : 2 * (SMEM_BYTES + 1024) <= 233472,
                "one CTA per SM (128 tokens), else two");
};

struct SmallParams {
  const uint8_t* wsf;   // W scales (tensor-core layout)
  const uint8_t* xsf;   // X scales
  void* y;
  int* status;
  uint32_t M, N, K;
  uint64_t ldy;
  uint32_t k_tiles, k_atoms, splits, kt_per_split;
  uint32_t w_early;     // W may be loaded before the previous kernel has finished
  const float* bias;    // [N] or null
  uint8_t* ysf;         // MXFP4 output: scales (tensor-core layout of an [M, N] operand)
  uint32_t qmode;       // MXFP4 output: rotation of each 32-column block
  uint32_t n_katoms_y;  // MXFP4 output: scale atoms per 128-row group of Y
  const float* a_scale; // NVFP4: tensor scales (device fp32) of X and W
  const float* b_scale;
  float* red_g;         // K-split partials [unit][min(M, NT)][128] fp32 in L2, or null
  const void* x;        // FX: bf16 activations [M, K], row stride ldx elements
  uint64_t ldx;
  uint32_t xmode;       // FX: rotation of each 32-element block of X (0, 1, 2)
};

__device__ __forceinline__ void record_timeout(int* status) {
  if (status) atomicExch(status, kTimeoutCode);
}

// Byte offset of the 4 fp32 values of (token m, 4-column group g) in a CTA's partial
// [NT][128]: groups are XOR-swizzled by m % 8 within each 32-column block, so the 16-byte
// reads of consecutive tokens (same g) fall on different banks, and a warp's stores of
// one token still cover 512 contiguous bytes.
__device__ __forceinline__ uint32_t red_off(uint32_t m, uint32_t g) {
  return (m * 128u + ((g ^ (m & 7u)) * 4u)) * 4u;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Cross-CTA sum of one W tile's K splits. CTA `sp` of the cluster owns the 4-column
// groups [sp * 32 / S, (sp + 1) * 32 / S) of the tile's 128 columns, for every token; an
// item is one (token, group): 4 fp32 values in each split's shared memory. The 128
// epilogue threads take items tid, tid + 128, ...; IB items at a time, whose loads from
// all S splits are issued together, then added in split order 0, 1, ..., S-1.
// L2: the partials come from p.red_g (written by the cluster's CTAs in this launch, so
// read at L2, not through the incoherent L1 path) instead of distributed shared memory.
template <uint32_t NT, int OUT, uint32_t S, bool L2 = false>
__device__ __forceinline__ void reduce_store(const SmallParams& p, uint32_t sbase, uint32_t wt,
                                             uint32_t sp, uint32_t tid, float alpha) {
  constexpr uint32_t IB = 16 / S;  // 16 loads in flight per thread
  const uint32_t g0 = sp * 32u / S, g1 = (sp + 1u) * 32u / S, width = g1 - g0;
  const uint32_t rows = p.M < NT ? p.M : NT;
  const uint32_t items = rows * width;
  const float* red_tile = L2 ? p.red_g + (uint64_t)wt * S * rows * 128u : nullptr;
  for (uint32_t it0 = tid; it0 < items; it0 += 128u * IB) {
    float4 t[IB][S];
    uint32_t tok[IB], col[IB];
#pragma unroll
    for (uint32_t i = 0; i < IB; ++i) {
      const uint32_t it = it0 + i * 128u;
      tok[i] = it / width;
      const uint32_t g = g0 + (it - tok[i] * width);
      col[i] = wt * 128u + g * 4u;  // N % 16 == 0: the 4 columns are all in or all out
      if (it < items) {
        if constexpr (L2) {
#pragma unroll
          for (uint32_t s = 0; s < S; ++s)
            t[i][s] = __ldcg(reinterpret_cast<const float4*>(
                red_tile + ((uint64_t)s * rows + tok[i]) * 128u + g * 4u));
        } else {
          const uint32_t off = sbase + red_off(tok[i], g);
#pragma unroll
          for (uint32_t s = 0; s < S; ++s) t[i][s] = ld_shared_cluster_v4(map_to_rank(off, s));
        }
      }
    }
#pragma unroll
    for (uint32_t i = 0; i < IB; ++i) {
      if (it0 + i * 128u >= items || col[i] >= p.N) continue;
      float4 acc = t[i][0];
#pragma unroll
      for (uint32_t s = 1; s < S; ++s) {
        acc.x += t[i][s].x;
        acc.y += t[i][s].y;
        acc.z += t[i][s].z;
        acc.w += t[i][s].w;
      }
      if (alpha != 1.0f) {  // NVFP4: the product of the tensor scales, on the full sum
        acc.x = __fmul_rn(acc.x, alpha);
        acc.y = __fmul_rn(acc.y, alpha);
        acc.z = __fmul_rn(acc.z, alpha);
        acc.w = __fmul_rn(acc.w, alpha);
      }
      if (p.bias != nullptr) {
        const float4 b = __ldg(reinterpret_cast<const float4*>(p.bias + col[i]));
        acc.x += b.x;
        acc.y += b.y;
        acc.z += b.z;
        acc.w += b.w;
      }
      if constexpr (OUT == kOutF32) {
        *reinterpret_cast<float4*>(static_cast<float*>(p.y) + (uint64_t)tok[i] * p.ldy + col[i]) =
            acc;
      } else {
        uint2 b;
        b.x = pack_bf16x2(acc.x, acc.y);
        b.y = pack_bf16x2(acc.z, acc.w);
        *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.y) + (uint64_t)tok[i] * p.ldy +
                                  col[i]) = b;
      }
    }
  }
}

// MXFP4 output: CTA sp owns the 32-column blocks b (0..3 of the tile) with b % S == sp;
// an item is one (row, block) of the 128-row scale tile: for rows m < M the 32 values of
// every split are added in split order (two splits' loads in flight), the bias added,
// the block rotated and quantised like an activation block; rows m >= M only get their
// zero scale byte (padding of the scale layout).
template <uint32_t NT>
__device__ __forceinline__ void reduce_store_mxfp4(const SmallParams& p, const KronCoeffs& kc,
                                                   uint32_t sbase, uint32_t wt, uint32_t sp,
                                                   uint32_t S, uint32_t tid) {
  uint32_t own[4], n_own = 0;
#pragma unroll
  for (uint32_t b = 0; b < 4; ++b)
    if (b % S == sp) own[n_own++] = b;
  for (uint32_t it = tid; it < 128u * n_own; it += 128u) {
    const uint32_t m = it / n_own;
    const uint32_t b = own[it - m * n_own];
    const uint32_t col = wt * 128u + b * 32u;
    const uint32_t kb = col / 32u;
    uint32_t byte = 0;
    if (m < p.M && col < p.N) {  // N % 32 == 0: the block is all in or all out
      float2 P[16];
      for (uint32_t s0 = 0; s0 < S; s0 += 2) {  // two splits' loads in flight, added in order
        float4 t[2][8];
#pragma unroll
        for (uint32_t h = 0; h < 2; ++h)
#pragma unroll
          for (uint32_t i = 0; i < 8; ++i)
            if (s0 + h < S)
              t[h][i] = ld_shared_cluster_v4(map_to_rank(sbase + red_off(m, b * 8u + i), s0 + h));
#pragma unroll
        for (uint32_t h = 0; h < 2; ++h) {
          if (s0 + h >= S) break;
#pragma unroll
          for (uint32_t i = 0; i < 8; ++i) {
            if (s0 + h == 0) {
              P[2 * i] = make_float2(t[h][i].x, t[h][i].y);
              P[2 * i + 1] = make_float2(t[h][i].z, t[h][i].w);
            } else {
              P[2 * i] = make_float2(P[2 * i].x + t[h][i].x, P[2 * i].y + t[h][i].y);
              P[2 * i + 1] = make_float2(P[2 * i + 1].x + t[h][i].z, P[2 * i + 1].y + t[h][i].w);
            }
          }
        }
      }
      if (p.bias != nullptr) {
#pragma unroll
        for (uint32_t i = 0; i < 8; ++i) {
          const float4 bb = __ldg(reinterpret_cast<const float4*>(p.bias + col + 4u * i));
          P[2 * i] = make_float2(__fadd_rn(P[2 * i].x, bb.x), __fadd_rn(P[2 * i].y, bb.y));
          P[2 * i + 1] =
              make_float2(__fadd_rn(P[2 * i + 1].x, bb.z), __fadd_rn(P[2 * i + 1].y, bb.w));
        }
      }
      if (p.qmode == 1) blockq::hadamard32(P);
      if (p.qmode == 2) blockq::kron32(P, kc);
      uint4 codes;
      byte = blockq::quantize_block(P, codes);
      blockq::st_v4(static_cast<uint8_t*>(p.y) + (uint64_t)m * p.ldy + col / 2u, codes);
    }
    if (kb < p.n_katoms_y * 4u) p.ysf[blockq::sf_offset(m, kb, p.n_katoms_y)] = (uint8_t)byte;
  }
}

// FX: the 128 epilogue threads rotate and quantise X[m, 256 kt0 .. 256 kt1) for the 16
// token rows of the tile (rows >= M and blocks past K give zero codes and scales) into
// the CTA's activation tiles, one k-tile at a time: thread (m, j) = (tid / 8, tid % 8)
// does block j of row m in every k-tile, keeping the loads of the next four k-tiles in
// flight, and releases the k-tile's barrier once it is written, so the MMAs of k-tile t
// wait only for k-tile t. Codes of k-tile t, row m, block j (16 bytes) go to
// XQ + t 2048 + m 128 + ((j ^ (m % 8)) 16) -- the K-major, 128-byte-swizzled operand
// layout the tensor core reads -- and the scale byte to the k-tile's scale atoms, laid out
// as in a global scale tensor. X comes from the kernel before this one: it is read only
// after waiting for it.
template <uint32_t NT>
__device__ __forceinline__ void quantize_x_slice(const SmallParams& p, const KronCoeffs& kc,
                                                 uint32_t sbase, uint32_t kt0, uint32_t kt1,
                                                 uint32_t bar_x) {
  using C = SmallConfig<NT, false, true>;
  static_assert(NT * 8 == 128, "one block per epilogue thread and k-tile");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint32_t tid = threadIdx.x - kFirstEpiWarp * 32u;
  const uint32_t nkt = kt1 - kt0;
  for (uint32_t i = tid; i < nkt * C::SF_STAGE / 16u; i += 128u)
    st_shared_v4(sbase + C::OFF_XSF + i * 16u, 0u, 0u, 0u, 0u);
  asm volatile("bar.sync 1, 128;" ::: "memory");  // the four epilogue warps
  const uint32_t kb_real = p.K / 32u;
  const uint32_t m = tid >> 3, j = tid & 7u;
  const bool row_ok = m < p.M;
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.x) +
                                                    (uint64_t)(row_ok ? m : 0u) * p.ldx);
  // Four k-tiles of loads in flight per thread (a ring of registers, slot t % 4).
  uint4 buf[4][4];
  auto load = [&](uint32_t t, uint4 (&w)[4]) {
    const uint32_t kb = (kt0 + t) * 8u + j;
    if (t < nkt && row_ok && kb < kb_real) {
#pragma unroll
      for (int c = 0; c < 4; ++c) w[c] = __ldg(src + kb * 4u + c);
    }
  };
#pragma unroll
  for (uint32_t u = 0; u < 4; ++u) load(u, buf[u]);
  for (uint32_t t0 = 0; t0 < nkt; t0 += 4) {
#pragma unroll
    for (uint32_t u = 0; u < 4; ++u) {
      const uint32_t t = t0 + u;
      if (t >= nkt) break;
      const uint32_t kb = (kt0 + t) * 8u + j;
      uint4 codes = make_uint4(0u, 0u, 0u, 0u);
      if (row_ok && kb < kb_real) {
        float2 P[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 w = buf[u][c];
          P[4 * c + 0] = make_float2(blockq::bf16_lo(w.x), blockq::bf16_hi(w.x));
          P[4 * c + 1] = make_float2(blockq::bf16_lo(w.y), blockq::bf16_hi(w.y));
          P[4 * c + 2] = make_float2(blockq::bf16_lo(w.z), blockq::bf16_hi(w.z));
          P[4 * c + 3] = make_float2(blockq::bf16_lo(w.w), blockq::bf16_hi(w.w));
        }
        load(t + 4, buf[u]);  // the slot is free again: refill it four k-tiles ahead
        if (p.xmode == 1) blockq::hadamard32(P);
        if (p.xmode == 2) blockq::kron32(P, kc);
        const uint32_t byte = blockq::quantize_block(P, codes);
        const uint32_t sf_addr = sbase + C::OFF_XSF + (t * C::AT + (j >> 2)) * 512u +
                                 (m & 31u) * 16u + (m >> 5) * 4u + (j & 3u);
        asm volatile("st.shared.u8 [%0], %1;" ::"r"(sf_addr), "r"(byte) : "memory");
      }
      st_shared_v4(sbase + C::OFF_XQ + t * C::XQ_KT + m * 128u + ((j ^ (m & 7u)) << 4),
                   codes.x, codes.y, codes.z, codes.w);
      fence_proxy_async_smem();  // the tensor core reads these tiles through the async proxy
      mbar_arrive(bar_x + 8u * t);
    }
  }
}

template <uint32_t NT, int OUT, bool NV, bool FX>
__global__ void __launch_bounds__(kThreads, 2) mxf4_gemm_smallm_kernel(
    const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
    const SmallParams p, const __grid_constant__ KronCoeffs kc) {
  using C = SmallConfig<NT, NV, FX>;
  constexpr uint32_t STAGES = C::STAGES;
  constexpr uint32_t AT = C::AT;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_addr + pad;
  const uint32_t warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31u;

  // The S CTAs of a W tile are consecutive along x: one cluster, rank = K split.
  const uint32_t S = p.splits;
  const uint32_t wt = blockIdx.x / S;       // W row tile (128 output columns)
  const uint32_t sp = blockIdx.x - wt * S;  // K split == cluster rank
  const uint32_t kt0 = sp * p.kt_per_split;
  const uint32_t kt1 = kt0 + p.kt_per_split < p.k_tiles ? kt0 + p.kt_per_split : p.k_tiles;
  const uint32_t pre = (kt1 - kt0) < STAGES ? (kt1 - kt0) : STAGES;  // stages filled up front

  const uint32_t bar_full = sbase + C::OFF_BAR;
  const uint32_t bar_empty = bar_full + 8 * STAGES;
  const uint32_t bar_tfull = bar_empty + 8 * STAGES;
  const uint32_t bar_mma_done = bar_tfull + 8;
  const uint32_t bar_xready = bar_mma_done + 8;  // FX: one per k-tile of activations
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    for (uint32_t s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_tfull, 1);
    mbar_init(bar_mma_done, 1);
    if constexpr (FX)
      for (uint32_t t = 0; t < kFxMaxKt; ++t) mbar_init(bar_xready + 8 * t, 128);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
    prefetch_tmap(&tmap_w);
    if constexpr (!FX) prefetch_tmap(&tmap_x);
    // When the kernel just before this one does not write W (the layer's own
    // quantiser), the first stages' W loads go out now, ahead of the set-up below
    // and of the wait for that kernel. Each stage's barrier expects its X bytes too.
    const uint64_t pol_w = l2_policy_evict_first();  // W is read once per call
    for (uint32_t i = 0; i < (p.w_early ? pre : 0u); ++i) {
      const uint32_t kt = kt0 + i;
      const uint32_t atoms = (p.k_atoms - AT * kt) >= AT ? AT : p.k_atoms - AT * kt;
      const uint32_t fb = bar_full + 8 * i;
      mbar_arrive_expect_tx(fb, C::A_STAGE + C::B_STAGE + (FX ? 1u : 2u) * atoms * 512u);
      tma_load_2d_hint(sbase + C::OFF_A + i * C::A_STAGE, &tmap_w, fb, (int32_t)(kt * 128u),
                       (int32_t)(wt * 128u), pol_w);
      bulk_load_hint(sbase + C::OFF_SFA + i * C::SF_STAGE,
                     p.wsf + ((uint64_t)wt * p.k_atoms + AT * kt) * 512u, atoms * 512u, fb, pol_w);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (elect_one()) {
      // X (and W, unless w_early) may come from the previous kernel: wait for it, then
      // let the next kernel start its set-up.
      asm volatile("griddepcontrol.wait;" ::: "memory");
      asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
      const uint64_t pol_w = l2_policy_evict_first();
      for (uint32_t i = 0; i < pre; ++i) {
        const uint32_t kt = kt0 + i;
        const uint32_t atoms = (p.k_atoms - AT * kt) >= AT ? AT : p.k_atoms - AT * kt;
        const uint32_t fb = bar_full + 8 * i;
        if (!p.w_early) {
          mbar_arrive_expect_tx(fb, C::A_STAGE + C::B_STAGE + (FX ? 1u : 2u) * atoms * 512u);
          tma_load_2d_hint(sbase + C::OFF_A + i * C::A_STAGE, &tmap_w, fb, (int32_t)(kt * 128u),
                           (int32_t)(wt * 128u), pol_w);
          bulk_load_hint(sbase + C::OFF_SFA + i * C::SF_STAGE,
                         p.wsf + ((uint64_t)wt * p.k_atoms + AT * kt) * 512u, atoms * 512u, fb,
                         pol_w);
        }
        if constexpr (!FX) {
          tma_load_2d(sbase + C::OFF_B + i * C::B_STAGE, &tmap_x, fb, (int32_t)(kt * 128u), 0);
          bulk_load(sbase + C::OFF_SFB + i * C::SF_STAGE, p.xsf + (uint64_t)(AT * kt) * 512u,
                    atoms * 512u, fb);
        }
      }
      uint32_t stage = pre % STAGES, phase = pre == STAGES ? 1u : 0u, issued = pre;
      bool ok = true;
      for (uint32_t kt = kt0 + pre; kt < kt1; ++kt) {
        if (!mbar_wait_bounded(bar_empty + 8 * stage, phase ^ 1u, abort_flag, kWaitLimitNs)) {
          ok = false;
          break;
        }
        const uint32_t atoms = (p.k_atoms - AT * kt) >= AT ? AT : p.k_atoms - AT * kt;
        const uint32_t fb = bar_full + 8 * stage;
        mbar_arrive_expect_tx(fb, C::A_STAGE + C::B_STAGE + (FX ? 1u : 2u) * atoms * 512u);
        tma_load_2d_hint(sbase + C::OFF_A + stage * C::A_STAGE, &tmap_w, fb, (int32_t)(kt * 128u),
                         (int32_t)(wt * 128u), pol_w);
        bulk_load_hint(sbase + C::OFF_SFA + stage * C::SF_STAGE,
                       p.wsf + ((uint64_t)wt * p.k_atoms + AT * kt) * 512u, atoms * 512u, fb,
                       pol_w);
        if constexpr (!FX) {
          tma_load_2d(sbase + C::OFF_B + stage * C::B_STAGE, &tmap_x, fb, (int32_t)(kt * 128u),
                      0);
          bulk_load(sbase + C::OFF_SFB + stage * C::SF_STAGE, p.xsf + (uint64_t)(AT * kt) * 512u,
                    atoms * 512u, fb);
        }
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) record_timeout(p.status);
      // Drain: every issued copy has landed before shared memory is reused or released.
      uint32_t s = stage, ph = phase;
      for (uint32_t i = 0; i < STAGES && i < issued; ++i) {
        if (s == 0) {
          s = STAGES - 1;
          ph ^= 1u;
        } else {
          --s;
        }
        volatile int never = 0;
        mbar_wait_bounded(bar_full + 8 * s, ph, &never, kWaitLimitNs);
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (uint32_t kt = kt0; kt < kt1; ++kt) {
        if (!mbar_wait_bounded(bar_full + 8 * stage, phase, abort_flag, kWaitLimitNs) ||
            (FX && !mbar_wait_bounded(bar_xready + 8 * (kt - kt0), 0, abort_flag, kWaitLimitNs))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t atoms = (p.k_atoms - AT * kt) >= AT ? AT : p.k_atoms - AT * kt;
        const uint32_t sfb_src = FX ? sbase + C::OFF_XSF + (kt - kt0) * C::SF_STAGE
                                    : sbase + C::OFF_SFB + stage * C::SF_STAGE;
        for (uint32_t a = 0; a < atoms; ++a) {
          tmem_cp_32x128b_warpx4(tmem_base + C::SFA_COL + 4 * a,
                                 smem_desc_sf(sbase + C::OFF_SFA + stage * C::SF_STAGE + a * 512));
          tmem_cp_32x128b_warpx4(tmem_base + C::SFB_COL + 4 * a, smem_desc_sf(sfb_src + a * 512));
        }
        const uint32_t k_left = p.K - kt * 256u;
        const uint32_t steps = k_left >= 256u ? 4u : (k_left + 63u) / 64u;
        const uint32_t a_tile = sbase + C::OFF_A + stage * C::A_STAGE;
        const uint32_t b_tile = FX ? sbase + C::OFF_XQ + (kt - kt0) * C::XQ_KT
                                   : sbase + C::OFF_B + stage * C::B_STAGE;
        for (uint32_t k = 0; k < steps; ++k) {
          const uint32_t sf_id = (k & 1u) * 2u;
          const uint32_t acc_in = (kt != kt0 || k != 0) ? 1u : 0u;
          if constexpr (NV)  // one atom (4 scales of 16) per K = 64 step
            mma_nvf4(tmem_base, smem_desc_sw128(a_tile + k * 32u), smem_desc_sw128(b_tile + k * 32u),
                     idesc_nvf4(128, NT), tmem_base + C::SFA_COL + 4 * k,
                     tmem_base + C::SFB_COL + 4 * k, acc_in);
          else  // an atom (4 scales of 32) per two K = 64 steps
            mma_mxf4(tmem_base, smem_desc_sw128(a_tile + k * 32u), smem_desc_sw128(b_tile + k * 32u),
                     idesc_mxf4(128, NT, sf_id, sf_id), tmem_base + C::SFA_COL + 4 * (k >> 1),
                     tmem_base + C::SFB_COL + 4 * (k >> 1), acc_in);
        }
        mma_commit(bar_empty + 8 * stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) mma_commit(bar_tfull);
      else record_timeout(p.status);
      mma_commit(bar_mma_done);
      volatile int never = 0;
      mbar_wait_bounded(bar_mma_done, 0, &never, kWaitLimitNs);
    }
  } else {
    // TMEM lane = W row = output column c of the tile, TMEM column = token m. The
    // accumulator goes to shared memory as red[m][c] (fp32): a warp's stores for one
    // token are 128 consecutive bytes.
    if constexpr (FX) quantize_x_slice<NT>(p, kc, sbase, kt0, kt1, bar_xready);
    const uint32_t c = (warp & 3u) * 32u + lane;
    const bool ok = mbar_wait_bounded(bar_tfull, 0, abort_flag, kWaitLimitNs);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      float* red = reinterpret_cast<float*>(smem);
      const uint32_t taddr = tmem_base + (((warp & 3u) * 32u) << 16);
      // L2 form: this CTA's partial rows m < min(M, NT) at red_g[unit][m][c]; a warp's
      // stores for one token are 128 consecutive bytes.
      const uint32_t rows = p.M < NT ? p.M : NT;
      float* red_g = p.red_g ? p.red_g + (uint64_t)blockIdx.x * rows * 128u + c : nullptr;
#pragma unroll
      for (uint32_t c0 = 0; c0 < NT; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x16(taddr + c0, &v[0]);
        if (c0 + 16 < NT) tmem_ld_32x32b_x16(taddr + c0 + 16, &v[16]);
        tmem_ld_wait();
        if (red_g != nullptr) {
#pragma unroll
          for (uint32_t j = 0; j < 32; ++j)
            if (c0 + j < NT && c0 + j < rows)
              __stcg(red_g + (c0 + j) * 128u, __uint_as_float(v[j]));
        } else {
#pragma unroll
          for (uint32_t j = 0; j < 32; ++j)
            if (c0 + j < NT)
              red[red_off(c0 + j, c >> 2) / 4u + (c & 3u)] = __uint_as_float(v[j]);
        }
      }
    } else if (lane == 0) {
      record_timeout(p.status);
    }
  }

  // Every partial of the cluster is in shared memory and every tensor-memory read is done.
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  } else if (warp >= kFirstEpiWarp) {
    const uint32_t tid = threadIdx.x - kFirstEpiWarp * 32u;
    float alpha = 1.0f;  // scales written by earlier kernels: this grid has waited for them
    if constexpr (NV) alpha = __fmul_rn(__ldg(p.a_scale), __ldg(p.b_scale));
    if constexpr (OUT == kOutMxfp4) {
      reduce_store_mxfp4<NT>(p, kc, sbase, wt, sp, S, tid);
    } else if (p.red_g != nullptr) {
      switch (S) {
        case 2: reduce_store<NT, OUT, 2, true>(p, sbase, wt, sp, tid, alpha); break;
        case 3: reduce_store<NT, OUT, 3, true>(p, sbase, wt, sp, tid, alpha); break;
        case 4: reduce_store<NT, OUT, 4, true>(p, sbase, wt, sp, tid, alpha); break;
        case 5: reduce_store<NT, OUT, 5, true>(p, sbase, wt, sp, tid, alpha); break;
        case 6: reduce_store<NT, OUT, 6, true>(p, sbase, wt, sp, tid, alpha); break;
        case 7: reduce_store<NT, OUT, 7, true>(p, sbase, wt, sp, tid, alpha); break;
        default: reduce_store<NT, OUT, 8, true>(p, sbase, wt, sp, tid, alpha); break;
      }
    } else {
      switch (S) {
        case 1: reduce_store<NT, OUT, 1>(p, sbase, wt, sp, tid, alpha); break;
        case 2: reduce_store<NT, OUT, 2>(p, sbase, wt, sp, tid, alpha); break;
        case 3: reduce_store<NT, OUT, 3>(p, sbase, wt, sp, tid, alpha); break;
        case 4: reduce_store<NT, OUT, 4>(p, sbase, wt, sp, tid, alpha); break;
        case 5: reduce_store<NT, OUT, 5>(p, sbase, wt, sp, tid, alpha); break;
        case 6: reduce_store<NT, OUT, 6>(p, sbase, wt, sp, tid, alpha); break;
        case 7: reduce_store<NT, OUT, 7>(p, sbase, wt, sp, tid, alpha); break;
        default: reduce_store<NT, OUT, 8>(p, sbase, wt, sp, tid, alpha); break;
      }
    }
  }
  // No CTA leaves (and releases its shared memory) while a peer may still read it.
  if (p.red_g == nullptr) cluster_sync();
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool operand_map(CUtensorMap* map, const uint8_t* base, uint64_t rows, uint64_t row_bytes,
                 uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Plan {
  uint32_t nt, splits, kt_per_split, units, w_tiles, k_tiles;
};

uint32_t token_tile(int64_t M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128; }

// Units (W tile x K split) are sized so that all of them are resident at once on the
// 148 SMs of a B200: two CTAs per SM, one for 128 tokens.
constexpr uint32_t kSms = 148;

Plan make_plan(int64_t M, int64_t N, int64_t K) {
  Plan pl{};
  pl.nt = token_tile(M);
  pl.w_tiles = (uint32_t)((N + 127) / 128);
  pl.k_tiles = (uint32_t)((K + 255) / 256);
  uint32_t splits = (pl.nt == 128 ? kSms : 2 * kSms) / pl.w_tiles;
  if (splits > kMaxSplits) splits = kMaxSplits;
  if (splits < 1) splits = 1;
  if (splits > pl.k_tiles) splits = pl.k_tiles;
  pl.kt_per_split = (pl.k_tiles + splits - 1) / splits;
  pl.splits = (pl.k_tiles + pl.kt_per_split - 1) / pl.kt_per_split;  // every split has work
  pl.units = pl.w_tiles * pl.splits;
  return pl;
}

// L2 bytes of the K-split partials (the data part of the GEMM scratch): for more
// than 32 tokens split 4 or more ways; 0 means the sum goes through distributed shared
// memory. (B200, 128 tokens: 8 splits 15.0 -> 13.2 us through L2; 2 splits, where half
// of the reads are the CTA's own shared memory, 13.1 -> 13.9 us, so they stay on chip.)
size_t red_bytes(const Plan& pl, int64_t M) {
  if (pl.splits < 4 || pl.nt < 64) return 0;
  const int64_t rows = M < (int64_t)pl.nt ? M : (int64_t)pl.nt;
  return (size_t)pl.units * (size_t)rows * 128u * sizeof(float);
}

// FX: aq / asf unused; x (bf16, row stride ldx) is rotated by xmode and quantised inside.
template <uint32_t NT, int OUT, bool NV, bool FX = false>
cudaError_t launch_nt(const Plan& pl, const uint8_t* aq, const uint8_t* asf, const uint8_t* bq,
                      const uint8_t* bsf, int64_t M, int64_t N, int64_t K, void* y,
                      const Epilogue& ep, int64_t ldy, int* status, bool w_early,
                      cudaStream_t stream, const void* x = nullptr, int64_t ldx = 0,
                      int xmode = 0, const KronCoeffs* xkc = nullptr, float* red_g = nullptr) {
  using C = SmallConfig<NT, NV, FX>;
  CUtensorMap tw, tx{};
  if (!operand_map(&tw, bq, (uint64_t)N, (uint64_t)(K / 2), 128) ||
      (!FX && !operand_map(&tx, aq, (uint64_t)M, (uint64_t)(K / 2), NT)))
    return cudaErrorInvalidValue;
  auto kern = mxf4_gemm_smallm_kernel<NT, OUT, NV, FX>;
  int dev = 0;
  cudaGetDevice(&dev);
  static bool attr_done[64] = {};
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  SmallParams p{};
  p.wsf = bsf;
  p.xsf = asf;
  p.y = y;
  p.status = status;
  p.M = (uint32_t)M;
  p.N = (uint32_t)N;
  p.K = (uint32_t)K;
  p.ldy = (uint64_t)ldy;
  p.k_tiles = pl.k_tiles;
  p.k_atoms = (uint32_t)sf_katoms(NV ? 2 * K : K);  // atoms of 4 scales per 128-row group
  p.splits = pl.splits;
  p.kt_per_split = pl.kt_per_split;
  p.w_early = w_early ? 1u : 0u;
  p.bias = ep.bias;
  p.ysf = ep.ysf;
  p.qmode = (uint32_t)ep.mode;
  p.n_katoms_y = (uint32_t)sf_katoms(N);
  p.a_scale = ep.a_scale;
  p.b_scale = ep.b_scale;
  p.x = x;
  p.ldx = (uint64_t)ldx;
  p.xmode = (uint32_t)xmode;
  p.red_g = OUT == kOutMxfp4 ? nullptr : red_g;  // the MXFP4 epilogue sums on chip
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(pl.units);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = pl.splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, tw, tx, p, FX ? *xkc : ep.kc);
}

}  // namespace

bool linear_smallm_fits(int64_t M, int64_t N, int64_t K, int mode) {
  if (M < 1 || M > kFxMaxRows || mode < 0 || mode > 2) return false;
  if (g_linear_form.load(std::memory_order_relaxed) == MXFP4_LINEAR_TWO_KERNELS) return false;
  const Plan pl = make_plan(M, N, K);
  return pl.nt == 16 && pl.kt_per_split <= kFxMaxKt;
}

cudaError_t launch_linear_smallm(const void* x, int64_t ldx, int mode, const KronCoeffs* kc,
                                 const uint8_t* wq, const uint8_t* wsf, int64_t M, int64_t N,
                                 int64_t K, void* y, int64_t ldy, int* status,
                                 cudaStream_t stream) {
  if (!linear_smallm_fits(M, N, K, mode)) return cudaErrorNotSupported;
  const Plan pl = make_plan(M, N, K);
  return launch_nt<16, kOutBf16, false, true>(pl, nullptr, nullptr, wq, wsf, M, N, K, y,
                                              Epilogue{}, ldy, status, false, stream, x, ldx,
                                              mode, kc);
}

size_t gemm_smallm_scratch_bytes(int64_t M, int64_t N, int64_t K) {
  return red_bytes(make_plan(M, N, K), M);
}

cudaError_t launch_gemm_smallm(const uint8_t* aq, const uint8_t* asf, const uint8_t* bq,
                               const uint8_t* bsf, int64_t M, int64_t N, int64_t K, void* y,
                               const Epilogue& ep, int64_t ldy, int* status,
                               const GemmScratch& scratch, bool b_early, cudaStream_t stream) {
  const Plan pl = make_plan(M, N, K);
  // K-split partials through L2 when the caller's scratch holds them, else on chip
  const size_t rb = red_bytes(pl, M);
  float* red = rb && scratch.data && scratch.data_bytes >= rb
                   ? reinterpret_cast<float*>(scratch.data)
                   : nullptr;
#define MXFP4_SMALLM_LAUNCH(NTV, OUTV, NVV)                                           \
  return launch_nt<NTV, OUTV, NVV>(pl, aq, asf, bq, bsf, M, N, K, y, ep, ldy, status, \
                                   b_early, stream, nullptr, 0, 0, nullptr, red)
#define MXFP4_SMALLM(NTV)                                                             \
  if (ep.nvfp4) {                                                                     \
    if (ep.out == kOutF32) MXFP4_SMALLM_LAUNCH(NTV, kOutF32, true);                   \
    MXFP4_SMALLM_LAUNCH(NTV, kOutBf16, true);                                         \
  }                                                                                   \
  switch (ep.out) {                                                                   \
    case kOutF32: MXFP4_SMALLM_LAUNCH(NTV, kOutF32, false);                           \
    case kOutMxfp4: MXFP4_SMALLM_LAUNCH(NTV, kOutMxfp4, false);                       \
    default: MXFP4_SMALLM_LAUNCH(NTV, kOutBf16, false);                               \
  }
  switch (pl.nt) {
    case 16: MXFP4_SMALLM(16)
    case 32: MXFP4_SMALLM(32)
    case 64: MXFP4_SMALLM(64)
    default: MXFP4_SMALLM(128)
  }
#undef MXFP4_SMALLM
#undef MXFP4_SMALLM_LAUNCH
}

}  // namespace mxfp4
