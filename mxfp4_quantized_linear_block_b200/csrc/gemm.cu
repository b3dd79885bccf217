// gemm.cu -- block-scaled MXFP4 x MXFP4 GEMM on the sm_100a tensor cores.
//
// y[M, N] = A[M, K] . B[N, K]^T with E2M1 operands and one E8M0 scale per 32
// elements of each operand row, accumulated in fp32 in tensor memory, written
// as bf16 (round to nearest even) or fp32. The operands stay FP4 all the way
// into the MMA: there is no dequantisation step ("AMD Quark delivers MXFP4
// quantization for FLUX.1-dev on Instinct MI350 with 1.92x speedup", opening
// section; "Bridging the Gap Between Promise and Performance for Microscaling
// FP4 Quantization", "GPU Kernel Ondersteuning (QuTLASS)").
//
// Structure: persistent clusters of two CTAs (one CTA per SM, 320 threads each)
// share 256 x 256 output tiles through tcgen05.mma.cta_group::2 (a last round that
// would leave half of the pairs idle runs as 256 x 128 units instead):
//   warp 0      TMA producer: this CTA's 128 rows of A and 128 rows of B per
//               stage (128-byte swizzled tiles) and the scale atoms, into a
//               ring of shared-memory stages;
//   warp 1      allocates tensor memory; in the leader CTA one lane copies each
//               stage's scales into tensor memory (tcgen05.cp) and issues the
//               tcgen05.mma kind::mxf4 block_scale instructions for the pair;
//   warps 2..9  epilogue: tensor memory -> registers -> bf16/fp32 -> swizzled
//               shared memory -> TMA store.
// 256 K-elements (128 bytes) per stage, four MMAs of K = 64 per stage. Every
// barrier wait is bounded in time; on expiry the CTA records MXFP4_ERR_TIMEOUT
// in the status word, drains its own copies, releases tensor memory and
// returns. Problems of at most 128 activation rows go to the weight-streaming
// kernel in gemm_smallm.cu instead.
//
// The same kernel runs a whole layer of more than 128 rows as one launch (FQ):
//   warps 10..15 quantiser: rotate and quantise x into the A operand in global
//               memory, publishing rows per 128-row group with a GPU-scope
//               release and a counter; the producer of each CTA waits for its
//               group before its first A load of a unit (fused_quantise_rows).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "block_quant.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace mxfp4 {
namespace {

using namespace sm100;

constexpr uint32_t BK_BYTES = 128;       // packed bytes of K per stage (256 elements)
constexpr uint32_t MMA_K_BYTES = 32;     // 64 elements per MMA
constexpr uint32_t kProducerWarp = 0;
constexpr uint32_t kMmaWarp = 1;
constexpr uint32_t kFirstEpiWarp = 2;
constexpr uint32_t kEpiWarps = 8;
constexpr uint32_t kThreads = (kFirstEpiWarp + kEpiWarps) * 32;
// The one-launch layer adds quantiser warps 10..15 (see fused_quantise_rows): 16 warps,
// four per SM sub-partition, so every warp keeps up to 128 registers.
constexpr uint32_t kQuantWarps = 6;
constexpr uint32_t kFirstQuantWarp = kFirstEpiWarp + kEpiWarps;
constexpr uint32_t kThreadsFused = (kFirstQuantWarp + kQuantWarps) * 32;
constexpr uint32_t kQDepth = 2;  // steps of x loads in flight per quantiser lane
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
constexpr int kTimeoutCode = 7;                  // MXFP4_ERR_TIMEOUT

struct Params {
  const uint8_t* asf;
  const uint8_t* bsf;
  void* y;
  int* status;
  uint32_t M, N, K;
  uint32_t m_tiles, n_tiles;
  uint32_t k_tiles;        // ceil(K / 256)
  uint32_t k_atoms;        // scale atoms per 128-row group: ceil(K / 128), NVFP4 ceil(K / 64)
  uint32_t b_row_tiles;    // ceil(N / 128)
  uint64_t ldy;            // elements
  // Work units: tiles [0, full_units) whole (256 x 256); each later tile is two units of
  // 256 x 128 (unit full_units + 2 t + h: column half h of tile full_units + t).
  uint32_t full_units, units;
  const float* bias;       // [N] or null
  uint8_t* yq;             // MXFP4 output: codes [M, ldy bytes per row]
  uint8_t* ysf;            // MXFP4 output: scales, tensor-core layout of an [M, N] operand
  uint32_t qmode;          // MXFP4 output: rotation of each 32-column block
  uint32_t rows_pad, n_katoms_y;
  const float* a_scale;    // NVFP4: tensor scales of A and B (device fp32)
  const float* b_scale;
  uint64_t tfull_wait_ns;  // bound of the epilogue's wait for an accumulator
  uint32_t skip_commit;    // testing only: 1 = pair 0 never signals its first accumulator
  // One-launch layer: A is quantised from x by the kernel's own quantiser warps.
  const uint16_t* x;       // bf16 [M, K], row stride K
  uint8_t* xq;             // A codes (what tmap_a reads)
  uint8_t* xsf;            // A scales
  uint32_t* rows_done;     // per 128-row group of A: rows published (zero at launch)
  uint32_t xmode;          // rotation of x: 0 none, 1 Hadamard-32, 2 Kronecker
  uint32_t rows_per_item;  // rows per quantiser work item (a power of two, <= 128)
  uint32_t* next_item;     // the next work item to hand out (zero at launch)
};

struct Unit {
  uint32_t tile;
  uint32_t half;  // 128-column unit: which half of the tile's 256 columns
  bool n128;      // a 256 x 128 unit (the last round's tiles, two units each)
};

__device__ __forceinline__ Unit unit_at(uint32_t u, const Params& p) {
  Unit w;
  if (u < p.full_units) {
    w.tile = u;
    w.half = 0;
    w.n128 = false;
  } else {
    const uint32_t v = u - p.full_units;
    w.tile = p.full_units + (v >> 1);
    w.half = v & 1u;
    w.n128 = true;
  }
  return w;
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void record_timeout(int* status) {
  if (status) atomicExch(status, kTimeoutCode);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---------------------------------------------------------------- fused quantiser warps
//
// The one-launch layer's quantiser: rotate (xmode) and quantise x into the A operand
// (codes and scales in the tensor-core layout) while the other warps of the grid run
// the GEMM on the rows already done. Rows go out in items of rows_per_item consecutive
// rows (an item never crosses a 128-row group), handed out in order by an atomic counter,
// so the running quantiser warps walk down the rows together, in the order the persistent
// tile loop asks for them, and do all of them whichever CTAs happen to be resident. Lane l
// handles the 32-element blocks l, l + 32, ...
// of a row: one step is a 1024-element stretch of one row (the lanes past the row's
// scale padding idle), and each lane keeps the x loads of the next kQDepth steps in
// flight in registers. A finished item is published: every lane orders its stores
// before the async proxy (the GEMM reads the codes with TMA) and fences at GPU scope,
// then lane 0 adds the item's rows to its group's counter, which the TMA producers wait
// on. Scale bytes of the K padding (blocks K/32 .. 4 ceil(K/128) - 1) are written 0.
__device__ __forceinline__ void fused_quantise_rows(const Params& p, const KronCoeffs& kc,
                                                    uint32_t lane) {
  const uint32_t kb_real = p.K / 32u;        // blocks of a row
  const uint32_t kb_pad = p.k_atoms * 4u;    // scale bytes of a row, K padding included
  const uint32_t spr = (kb_pad + 31u) / 32u;  // steps per row
  const uint32_t rpi = p.rows_per_item;
  const uint32_t n_items = (p.M + rpi - 1u) / rpi;
  const uint64_t pol = l2_policy_evict_first();  // x is read once
  // The load cursor runs kQDepth steps ahead of the compute cursor, so it takes each item
  // from the counter first; the items between the two wait in a 4-slot queue kept one per
  // lane (slot s in lane s: at most kQDepth items lie between the cursors).
  static_assert(kQDepth <= 3, "the item queue has 4 slots");
  uint32_t queue = 0;
  auto grab = [&](uint32_t seq) -> uint32_t {
    uint32_t it = 0;
    if (lane == 0) it = atomicAdd(p.next_item, 1u);
    it = __shfl_sync(0xffffffffu, it, 0);
    if (lane == (seq & 3u)) queue = it;
    return it;
  };
  struct Cursor {
    uint32_t item, r, j, seq;  // work item, row within it, step within the row, item number
  };
  auto advance = [&](Cursor& c, bool loads) {
    if (++c.j == spr) {
      c.j = 0;
      if (++c.r == rpi || c.item * rpi + c.r >= p.M) {
        c.r = 0;
        ++c.seq;
        c.item = loads ? grab(c.seq) : __shfl_sync(0xffffffffu, queue, c.seq & 3u);
      }
    }
  };
  auto load = [&](const Cursor& c, uint4 (&w)[4]) {
    const uint32_t kb = c.j * 32u + lane;
    if (c.item < n_items && kb < kb_real) {
      const uint4* src =
          reinterpret_cast<const uint4*>(p.x + (uint64_t)(c.item * rpi + c.r) * p.K + kb * 32u);
#pragma unroll
      for (int q = 0; q < 4; ++q) w[q] = ld_nc_v4_hint(src + q, pol);
    }
  };
  Cursor ld{grab(0u), 0u, 0u, 0u};
  Cursor cp = ld;
  uint4 buf[kQDepth][4];
#pragma unroll
  for (uint32_t d = 0; d < kQDepth; ++d) {
    load(ld, buf[d]);
    advance(ld, true);
  }
  while (cp.item < n_items) {
#pragma unroll
    for (uint32_t d = 0; d < kQDepth; ++d) {
      if (cp.item >= n_items) break;
      const uint32_t row = cp.item * rpi + cp.r;
      const uint32_t kb = cp.j * 32u + lane;
      const bool has = kb < kb_real;
      float2 P[16];
      if (has) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 w = buf[d][c];
          P[4 * c + 0] = make_float2(blockq::bf16_lo(w.x), blockq::bf16_hi(w.x));
          P[4 * c + 1] = make_float2(blockq::bf16_lo(w.y), blockq::bf16_hi(w.y));
          P[4 * c + 2] = make_float2(blockq::bf16_lo(w.z), blockq::bf16_hi(w.z));
          P[4 * c + 3] = make_float2(blockq::bf16_lo(w.w), blockq::bf16_hi(w.w));
        }
      }
      load(ld, buf[d]);  // the slot is free again: refill it kQDepth steps ahead
      advance(ld, true);
      uint32_t byte = 0;
      if (has) {
        if (p.xmode == 1) blockq::hadamard32(P);
        if (p.xmode == 2) blockq::kron32(P, kc);
        uint4 codes;
        byte = blockq::quantize_block(P, codes);
        blockq::st_v4(p.xq + (uint64_t)row * (p.K / 2u) + kb * 16u, codes);
      }
      // lane 4i writes the scale word of blocks 4i .. 4i + 3 (one word of an atom row)
      const uint32_t b1 = __shfl_down_sync(0xffffffffu, byte, 1);
      const uint32_t b2 = __shfl_down_sync(0xffffffffu, byte, 2);
      const uint32_t b3 = __shfl_down_sync(0xffffffffu, byte, 3);
      if ((lane & 3u) == 0u && kb < kb_pad)
        *reinterpret_cast<uint32_t*>(p.xsf + blockq::sf_offset(row, kb, p.k_atoms)) =
            byte | (b1 << 8) | (b2 << 16) | (b3 << 24);
      if (cp.j + 1u == spr && (cp.r + 1u == rpi || row + 1u >= p.M)) {  // item done
        fence_proxy_async_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(p.rows_done + (row >> 7), cp.r + 1u);
      }
      advance(cp, false);
    }
  }
}

// ---------------------------------------------------------------- CTA-pair kernel
//
// Two CTAs of a cluster share one 256 x 256 output tile through
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 64): each CTA loads its own
// 128 rows of A and its own 128 rows of B, so each SM streams half the operand
// bytes per MMA that a single-CTA 128 x 256 tile needs. The leader (even rank)
// issues the MMAs and the scale copies for both; both CTAs run producers and
// epilogues. Tile loads of both CTAs complete on the leader's stage barrier;
// the leader's commits arrive on both CTAs' barriers. No load is multicast.


template <uint32_t STAGES, bool NV = false>
struct PairConfig {
  // scale atoms (128 rows x 4 scales) per stage of 256 K-elements and 128 rows: 2 for
  // MXFP4 (32-element blocks), 4 for NVFP4 (16-element groups)
  static constexpr uint32_t AT = NV ? 4 : 2;
  static constexpr uint32_t BN = 256;                 // N per pair tile
  static constexpr uint32_t A_STAGE = 128 * BK_BYTES;  // own 128 rows of A
  static constexpr uint32_t B_STAGE = 128 * BK_BYTES;  // own 128 rows of B
  static constexpr uint32_t SFA_STAGE = AT * 512;      // own rows: AT scale atoms
  static constexpr uint32_t SFB_STAGE = 2 * AT * 512;  // all 256 rows of B: 2 groups x AT atoms
  static constexpr uint32_t STAGE_TX = A_STAGE + B_STAGE + SFA_STAGE + SFB_STAGE;
  static constexpr uint32_t OFF_A = 0;
  static constexpr uint32_t OFF_B = OFF_A + STAGES * A_STAGE;
  static constexpr uint32_t OFF_SFA = OFF_B + STAGES * B_STAGE;
  static constexpr uint32_t OFF_SFB = OFF_SFA + STAGES * SFA_STAGE;
  static constexpr uint32_t EPI_BUF = 32 * 128;  // per epilogue warp: 32 rows x 128 bytes
  static constexpr uint32_t OFF_EPI = OFF_SFB + STAGES * SFB_STAGE;
  static constexpr uint32_t OFF_BAR = OFF_EPI + kEpiWarps * EPI_BUF;
  static constexpr uint32_t NUM_BARS = 2 * STAGES + 3;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;
  // Two 256-column accumulators that share 64 columns: tile i uses columns
  // [0, 256) or [192, 448) alternately. The epilogue drains the shared 64
  // columns first and then hands the accumulator back, so the next tile's MMAs
  // overlap the rest of the drain.
  static constexpr uint32_t ACC1_COL = 192;
  static constexpr uint32_t SFA_COL = ACC1_COL + BN;  // 448
  static constexpr uint32_t SFB_COL = SFA_COL + 4 * AT;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(SFB_COL + 8 * AT <= TMEM_COLS, "tensor memory budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <uint32_t STAGES, int OUT, bool NV, bool FQ>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(FQ ? kThreadsFused : kThreads, 1)
    mxf4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                          const __grid_constant__ CUtensorMap tmap_b,
                          const __grid_constant__ CUtensorMap tmap_b64,
                          const __grid_constant__ CUtensorMap tmap_sfa,
                          const __grid_constant__ CUtensorMap tmap_sfb,
                          const __grid_constant__ CUtensorMap tmap_y, const Params p,
                          const __grid_constant__ KronCoeffs kc) {
  constexpr bool Y_F32 = OUT == kOutF32;
  using C = PairConfig<STAGES, NV>;
  constexpr uint32_t BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_addr + pad;

  const uint32_t warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t rank = cluster_ctarank();  // 0: leader
  const uint32_t pair = blockIdx.x >> 1;
  const uint32_t num_pairs = gridDim.x >> 1;

  const uint32_t bar_full = sbase + C::OFF_BAR;        // [STAGES], leader's count both CTAs
  const uint32_t bar_empty = bar_full + 8 * STAGES;    // [STAGES]
  const uint32_t bar_tfull = bar_empty + 8 * STAGES;   // accumulator ready
  const uint32_t bar_tempty = bar_tfull + 8;           // leader: shared columns drained
  const uint32_t bar_mma_done = bar_tempty + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    for (uint32_t s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_tfull, 1);
    mbar_init(bar_tempty, 2 * (kEpiWarps / 2));  // the 4 warps draining the shared columns, x2 CTAs
    mbar_init(bar_mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_b64);
    prefetch_tmap(&tmap_sfa);
    prefetch_tmap(&tmap_sfb);
    if constexpr (OUT != kOutMxfp4) prefetch_tmap(&tmap_y);  // unused (zero) map otherwise
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(smem_addr(tmem_slot), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Operands may be produced by the kernel launched just before this one (programmatic
  // dependent launch): wait for it, then let the next kernel start its set-up.
  griddep_wait();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == kProducerWarp) {
    if (elect_one()) {
      const uint32_t full_at_leader = map_to_rank(bar_full, 0);
      uint32_t stage = 0, phase = 0, issued = 0;
      uint32_t ready_group = 0xffffffffu;  // one-launch layer: last A group seen complete
      bool ok = true;
      for (uint32_t u = pair; u < p.units && ok; u += num_pairs) {
        const Unit w = unit_at(u, p);
        const uint32_t mt = w.tile / p.n_tiles, nt = w.tile % p.n_tiles;  // 256-row m tiles
        const int32_t m_cta = (int32_t)(mt * 256u + rank * 128u);
        if constexpr (FQ) {
          // This CTA's 128 rows of A come from the grid's quantiser warps: wait until all
          // of them are published (a group past M has none).
          const uint32_t g = 2u * mt + rank;
          const uint32_t left = p.M > 128u * g ? p.M - 128u * g : 0u;
          if (g != ready_group && left != 0u) {
            if (!wait_count_bounded(p.rows_done + g, left < 128u ? left : 128u, abort_flag,
                                    kWaitLimitNs)) {
              ok = false;
              break;
            }
            fence_proxy_async_global();
            ready_group = g;
          }
        }
        // B rows of this CTA: 128 of the tile's 256, or 64 of a 128-column unit's 128
        const int32_t n_cta =
            (int32_t)(nt * BN + (w.n128 ? w.half * 128u + rank * 64u : rank * 128u));
        const uint32_t tx = 2u * (w.n128 ? C::STAGE_TX - C::B_STAGE / 2u : C::STAGE_TX);
        for (uint32_t kt = 0; kt < p.k_tiles; ++kt) {
          if (!mbar_wait_bounded(bar_empty + 8 * stage, phase ^ 1u, abort_flag, kWaitLimitNs)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(bar_full + 8 * stage, tx);
          const uint32_t fb = full_at_leader + 8 * stage;
          tma_load_2d_pair(sbase + C::OFF_A + stage * C::A_STAGE, &tmap_a, fb,
                           (int32_t)(kt * BK_BYTES), m_cta);
          tma_load_2d_pair(sbase + C::OFF_B + stage * C::B_STAGE, w.n128 ? &tmap_b64 : &tmap_b,
                           fb, (int32_t)(kt * BK_BYTES), n_cta);
          // scale atoms: A's are rows of a [row_tiles * k_atoms, 128-word] view, B's a
          // [row_tiles, k_atoms, 128-word] view (both 128-row groups of the tile)
          tma_load_2d_pair(sbase + C::OFF_SFA + stage * C::SFA_STAGE, &tmap_sfa, fb, 0,
                           (int32_t)((uint32_t)(m_cta / 128) * p.k_atoms + C::AT * kt));
          tma_load_3d_pair(sbase + C::OFF_SFB + stage * C::SFB_STAGE, &tmap_sfb, fb, 0,
                           (int32_t)(C::AT * kt), (int32_t)(nt * 2u));
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) record_timeout(p.status);
      if (rank == 0) {
        // Both CTAs' loads into the last stages have landed (they count on these barriers).
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
    }
  } else if (warp == kMmaWarp) {
    if (rank == 0 && elect_one()) {
      uint32_t stage = 0, phase = 0, acc_phase = 0;
      bool ok = true;
      for (uint32_t u = pair; u < p.units && ok; u += num_pairs) {
        const Unit w = unit_at(u, p);
        if (!mbar_wait_bounded(bar_tempty, acc_phase ^ 1u, abort_flag, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (acc_phase ? C::ACC1_COL : 0u);
        // A 128-column unit: N = 128, and its B rows are the scale group of its half.
        const uint32_t n_mma = w.n128 ? 128u : BN;
        const uint32_t sfb_half = w.n128 ? 4u * w.half : 0u;
        for (uint32_t kt = 0; kt < p.k_tiles; ++kt) {
          if (!mbar_wait_bounded(bar_full + 8 * stage, phase, abort_flag, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_s = sbase + C::OFF_SFA + stage * C::SFA_STAGE;
          const uint32_t sfb_s = sbase + C::OFF_SFB + stage * C::SFB_STAGE;
          const uint32_t sfa_t = tmem_base + C::SFA_COL;
          const uint32_t sfb_t = tmem_base + C::SFB_COL;
          for (uint32_t a = 0; a < C::AT; ++a) {
            tmem_cp_32x128b_warpx4_pair(sfa_t + 4 * a, smem_desc_sf(sfa_s + a * 512));
            for (uint32_t g = 0; g < 2; ++g)
              tmem_cp_32x128b_warpx4_pair(sfb_t + 4 * (2 * a + g),
                                          smem_desc_sf(sfb_s + (g * C::AT + a) * 512));
          }
          const uint32_t k_left = p.K - kt * 256u;
          const uint32_t steps = k_left >= 256u ? 4u : (k_left + 63u) / 64u;
          const uint32_t a_tile = sbase + C::OFF_A + stage * C::A_STAGE;
          const uint32_t b_tile = sbase + C::OFF_B + stage * C::B_STAGE;
          for (uint32_t k = 0; k < steps; ++k) {
            const uint32_t acc_in = (kt != 0u || k != 0u) ? 1u : 0u;
            if constexpr (NV) {
              // NVFP4: one atom (4 scales of 16 per row) per K = 64 step
              mma_nvf4_pair(d_tmem, smem_desc_sw128(a_tile + k * MMA_K_BYTES),
                            smem_desc_sw128(b_tile + k * MMA_K_BYTES), idesc_nvf4(256, n_mma),
                            sfa_t + 4 * k, sfb_t + 8 * k + sfb_half, acc_in);
            } else {
              // MXFP4: an atom (4 scales of 32 per row) serves two K = 64 steps
              const uint32_t sf_id = (k & 1u) * 2u;
              mma_mxf4_pair(d_tmem, smem_desc_sw128(a_tile + k * MMA_K_BYTES),
                            smem_desc_sw128(b_tile + k * MMA_K_BYTES),
                            idesc_mxf4(256, n_mma, sf_id, sf_id), sfa_t + 4 * (k >> 1),
                            sfb_t + 8 * (k >> 1) + sfb_half, acc_in);
            }
          }
          mma_commit_pair_both(bar_empty + 8 * stage);  // frees the stage in both CTAs
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        // both halves of the accumulator are ready (the test hook withholds pair 0's first)
        if (!(p.skip_commit && u == 0u)) mma_commit_pair_both(bar_tfull);
        acc_phase ^= 1u;
      }
      if (!ok) record_timeout(p.status);
      mma_commit_pair_leader(bar_mma_done);
      volatile int never = 0;
      mbar_wait_bounded(bar_mma_done, 0, &never, kWaitLimitNs);
    }
  } else if (warp < kFirstQuantWarp) {
    // Epilogue. Warp w owns TMEM lanes 32 * (w % 4) .. +31 and two of the tile's
    // four 64-column chunks; the half-0 warps take the chunk the other
    // accumulator overlaps first and release the accumulator after reading it.
    // A 128-column unit has two chunks, both drained by the half-0 warps.
    // Each chunk goes TMEM -> registers -> bf16/fp32 -> the warp's swizzled
    // shared buffer -> TMA store (which clips rows >= M and columns >= N).
    const uint32_t quad = warp & 3u;
    const uint32_t half = (warp - kFirstEpiWarp) / 4u;
    const uint32_t tempty_at_leader = map_to_rank(bar_tempty, 0);
    // NVFP4: y = alpha * sum, alpha = product of the tensor scales (written by earlier
    // kernels; this grid has waited for its predecessor above)
    float alpha = 1.0f;
    if constexpr (NV) alpha = __fmul_rn(__ldg(p.a_scale), __ldg(p.b_scale));
    const uint32_t buf = sbase + C::OFF_EPI + (warp - kFirstEpiWarp) * C::EPI_BUF;
    const uint32_t rowoff = buf + lane * 128u;
    constexpr uint32_t CCOLS = Y_F32 ? 32 : 64;  // columns per 128-byte staged row
    uint32_t acc_phase = 0;
    for (uint32_t u = pair; u < p.units; u += num_pairs) {
      const Unit w = unit_at(u, p);
      const uint32_t mt = w.tile / p.n_tiles, nt = w.tile % p.n_tiles;
      if (w.n128 && half == 1) {  // the half-0 warps drain a 128-column unit
        acc_phase ^= 1u;
        continue;
      }
      const bool ok = mbar_wait_bounded(bar_tfull, acc_phase, abort_flag, p.tfull_wait_ns);
      if (!__all_sync(0xffffffffu, ok)) {  // leave together so .aligned ops stay convergent
        if (lane == 0) record_timeout(p.status);
        break;
      }
      tc_fence_after();
      const uint32_t acc_col = acc_phase ? C::ACC1_COL : 0u;
      const uint32_t shared_chunk = acc_phase ? 0u : 3u;
      const uint32_t col_tile = nt * BN + (w.n128 ? w.half * 128u : 0u);  // first column
      uint32_t ch[2];
      if (w.n128) {
        ch[0] = 0;
        ch[1] = 1;
      } else if (half == 0) {
        ch[0] = shared_chunk;
        ch[1] = acc_phase ? 1u : 2u;
      } else {
        ch[0] = acc_phase ? 2u : 0u;
        ch[1] = acc_phase ? 3u : 1u;
      }
      const uint32_t taddr = tmem_base + ((quad * 32u) << 16) + acc_col;
      const int32_t row0 = (int32_t)(mt * 256u + rank * 128u + quad * 32u);
      uint32_t sfw = 0;  // MXFP4 output: this row's 4 scale bytes of the warp's 128 columns
#pragma unroll
      for (uint32_t r = 0; r < 2; ++r) {
        uint32_t v[2][32];
        tmem_ld_32x32b_x32(taddr + ch[r] * 64u, v[0]);
        tmem_ld_32x32b_x32(taddr + ch[r] * 64u + 32u, v[1]);
        tmem_ld_wait();
        if (r == 0 && half == 0) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(tempty_at_leader);
        }
        const uint32_t col_base = col_tile + ch[r] * 64u;  // first column of this chunk
        if constexpr (NV) {  // the two tensor scales, once, on the full sum
#pragma unroll
          for (uint32_t h = 0; h < 2; ++h)
#pragma unroll
            for (uint32_t j = 0; j < 32; ++j)
              v[h][j] = __float_as_uint(__fmul_rn(__uint_as_float(v[h][j]), alpha));
        }
        if (p.bias != nullptr) {
#pragma unroll
          for (uint32_t h = 0; h < 2; ++h) {
#pragma unroll
            for (uint32_t j = 0; j < 32; j += 4) {
              const uint32_t col = col_base + h * 32u + j;  // N % 16 == 0: 4 in or 4 out
              const float4 b = col < p.N ? __ldg(reinterpret_cast<const float4*>(p.bias + col))
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
              v[h][j + 0] = __float_as_uint(__fadd_rn(__uint_as_float(v[h][j + 0]), b.x));
              v[h][j + 1] = __float_as_uint(__fadd_rn(__uint_as_float(v[h][j + 1]), b.y));
              v[h][j + 2] = __float_as_uint(__fadd_rn(__uint_as_float(v[h][j + 2]), b.z));
              v[h][j + 3] = __float_as_uint(__fadd_rn(__uint_as_float(v[h][j + 3]), b.w));
            }
          }
        }
        if constexpr (OUT == kOutMxfp4) {
          // Each 32 columns of this thread's row are one block of the next layer's
          // operand: rotate, quantise, store 16 code bytes; collect the scale byte.
          const uint32_t row = (uint32_t)row0 + lane;
#pragma unroll
          for (uint32_t h = 0; h < 2; ++h) {
            float2 P[16];
#pragma unroll
            for (uint32_t j = 0; j < 16; ++j)
              P[j] = make_float2(__uint_as_float(v[h][2 * j]), __uint_as_float(v[h][2 * j + 1]));
            if (p.qmode == 1) blockq::hadamard32(P);
            if (p.qmode == 2) blockq::kron32(P, kc);
            uint4 codes;
            const uint32_t byte = blockq::quantize_block(P, codes);
            const uint32_t col = col_base + h * 32u;
            const bool inside = row < p.M && col < p.N;
            if (inside) blockq::st_v4(p.yq + (uint64_t)row * p.ldy + col / 2u, codes);
            sfw |= (inside ? byte : 0u) << (((col / 32u) & 3u) * 8u);
          }
        } else {
#pragma unroll
          for (uint32_t c = 0; c < 64 / CCOLS; ++c) {
            const int32_t col0 = (int32_t)(col_base + c * CCOLS);
            if (lane == 0) bulk_wait_read_all();  // the buffer's previous store has read it
            __syncwarp();
#pragma unroll
            for (uint32_t j = 0; j < 8; ++j) {
              const uint32_t addr = rowoff + ((j ^ (lane & 7u)) << 4);
              if constexpr (Y_F32) {
                const uint32_t* src = &v[c][4 * j];
                st_shared_v4(addr, src[0], src[1], src[2], src[3]);
              } else {
                const uint32_t* src = &v[j / 4][(8 * j) % 32];
                st_shared_v4(addr, pack_bf16x2(__uint_as_float(src[0]), __uint_as_float(src[1])),
                             pack_bf16x2(__uint_as_float(src[2]), __uint_as_float(src[3])),
                             pack_bf16x2(__uint_as_float(src[4]), __uint_as_float(src[5])),
                             pack_bf16x2(__uint_as_float(src[6]), __uint_as_float(src[7])));
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmap_y, buf, col0, row0);
              bulk_commit_group();
            }
          }
        }
      }
      if constexpr (OUT == kOutMxfp4) {
        // The warp's two chunks are 128 aligned columns: one word of a scale atom per row.
        const uint32_t row = (uint32_t)row0 + lane;
        const uint32_t ka = (col_tile + (ch[0] >= 2u ? 128u : 0u)) / 128u;
        if (row < p.rows_pad && ka < p.n_katoms_y)
          *reinterpret_cast<uint32_t*>(p.ysf + ((uint64_t)(row >> 7) * p.n_katoms_y + ka) * 512u +
                                       (row & 31u) * 16u + ((row >> 5) & 3u) * 4u) = sfw;
      }
      acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait_all();  // this warp's output stores are complete
    __syncwarp();
  } else if constexpr (FQ) {
    fused_quantise_rows(p, kc, lane);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the pair's MMAs or copies may touch it
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
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

// 2-D map over a [rows, K/2]-byte operand, box = 128 bytes x box_rows, 128-byte swizzle.
bool make_operand_map(CUtensorMap* map, const uint8_t* base, uint64_t rows, uint64_t row_bytes,
                      uint32_t box_rows) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {BK_BYTES, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Scale atoms of an operand as 128-word (512-byte) rows: 2-D [row_tiles * k_atoms, 128]
// (box: `at` consecutive atoms) or 3-D [row_tiles, k_atoms, 128] (box: `at` atoms x 2 row
// tiles).
bool make_scale_map(CUtensorMap* map, const uint8_t* sf, uint64_t row_tiles, uint64_t k_atoms,
                    bool three_d, uint32_t at) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r;
  if (three_d) {
    cuuint64_t dims[3] = {128, k_atoms, row_tiles};
    cuuint64_t strides[2] = {512, k_atoms * 512};
    cuuint32_t box[3] = {128, at, 2};
    r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint8_t*>(sf), dims, strides, box,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    cuuint64_t dims[2] = {128, row_tiles * k_atoms};
    cuuint64_t strides[1] = {512};
    cuuint32_t box[2] = {128, at};
    r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint8_t*>(sf), dims, strides, box,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  return r == CUDA_SUCCESS;
}

// Output map: [M, N] row-major bf16 / fp32, box = 128 bytes of a row x 32 rows, 128-byte swizzle.
bool make_output_map(CUtensorMap* map, void* y, uint64_t M, uint64_t N, uint64_t ldy, bool f32) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {N, M};
  cuuint64_t strides[1] = {ldy * (f32 ? 4u : 2u)};
  cuuint32_t box[2] = {f32 ? 32u : 64u, 32u};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Work plan of the persistent pair kernel. Whole 256 x 256 tiles go round-robin over the
// CTA pairs. When the last round would leave at least half of the pairs idle, each of its
// tiles becomes two 256 x 128 units (N = 128 MMAs on the tile's column halves), so that
// round takes about half as long and needs no exchange between pairs. (The earlier form
// split those tiles along K and added fp32 partials through L2: at 3584 x 3072 -> 3072
// the hand-over took about 8 us against 1.3 us of MMAs.)
struct PairPlan {
  uint32_t tiles, full_units, units;
};

PairPlan pair_plan(int64_t M, int64_t N, uint32_t pairs) {
  PairPlan pl{};
  pl.tiles = (uint32_t)(((M + 255) / 256) * ((N + 255) / 256));
  pl.full_units = pl.units = pl.tiles;
  const uint32_t tail = pairs ? pl.tiles % pairs : 0;
  if (tail != 0 && 2u * tail <= pairs) {
    pl.full_units = pl.tiles - tail;
    pl.units = pl.full_units + 2u * tail;
  }
  return pl;
}

// The one-launch layer's x (quantised into aq / asf by the kernel itself).
struct FusedX {
  const void* x;
  int mode;
  uint32_t* rows_done;
};

template <uint32_t STAGES, int OUT, bool NV, bool FQ = false>
cudaError_t launch_pair(const uint8_t* aq, const uint8_t* asf, const uint8_t* bq,
                        const uint8_t* bsf, int64_t M, int64_t N, int64_t K, void* y,
                        const Epilogue& ep, int64_t ldy, int* status, cudaStream_t stream,
                        const FusedX* fx = nullptr) {
  using C = PairConfig<STAGES, NV>;
  constexpr uint32_t threads = FQ ? kThreadsFused : kThreads;
  // scale atoms per 128-row group: one per 4 scales, i.e. per 128 (MXFP4) or 64 (NVFP4) K
  const uint64_t k_atoms = (uint64_t)sf_katoms(NV ? 2 * K : K);
  CUtensorMap ta, tb, tb64, tsa, tsb, ty{};
  if (!make_operand_map(&ta, aq, (uint64_t)M, (uint64_t)(K / 2), 128) ||
      !make_operand_map(&tb, bq, (uint64_t)N, (uint64_t)(K / 2), 128) ||
      !make_operand_map(&tb64, bq, (uint64_t)N, (uint64_t)(K / 2), 64) ||
      !make_scale_map(&tsa, asf, (uint64_t)sf_row_tiles(M), k_atoms, false, C::AT) ||
      !make_scale_map(&tsb, bsf, (uint64_t)sf_row_tiles(N), k_atoms, true, C::AT) ||
      (OUT != kOutMxfp4 &&
       !make_output_map(&ty, y, (uint64_t)M, (uint64_t)N, (uint64_t)ldy, OUT == kOutF32)))
    return cudaErrorInvalidValue;
  auto kern = mxf4_gemm_pair_kernel<STAGES, OUT, NV, FQ>;
  int dev = 0;
  cudaGetDevice(&dev);
  static bool attr_done[64] = {};
  static int max_clusters[64] = {};
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t q{};
    q.gridDim = dim3(2);
    q.blockDim = dim3(threads);
    q.dynamicSmemBytes = C::SMEM_BYTES;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &q) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      int sms = 148;
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      n = sms / 2;
    }
    max_clusters[dev] = n;
    attr_done[dev] = true;
  }
  Params p{};
  p.asf = asf;
  p.bsf = bsf;
  p.y = y;
  p.status = status;
  p.M = (uint32_t)M;
  p.N = (uint32_t)N;
  p.K = (uint32_t)K;
  p.m_tiles = (uint32_t)((M + 255) / 256);
  p.n_tiles = (uint32_t)((N + C::BN - 1) / C::BN);
  p.k_tiles = (uint32_t)((K + 255) / 256);
  p.k_atoms = (uint32_t)k_atoms;
  p.b_row_tiles = (uint32_t)sf_row_tiles(N);
  p.ldy = (uint64_t)ldy;
  const PairPlan pl = pair_plan(M, N, (uint32_t)max_clusters[dev]);
  p.full_units = pl.full_units;
  p.units = pl.units;
  p.bias = ep.bias;
  p.yq = OUT == kOutMxfp4 ? static_cast<uint8_t*>(y) : nullptr;
  p.ysf = ep.ysf;
  p.qmode = (uint32_t)ep.mode;
  p.rows_pad = (uint32_t)(sf_row_tiles(M) * 128);
  p.n_katoms_y = (uint32_t)sf_katoms(N);
  p.a_scale = ep.a_scale;
  p.b_scale = ep.b_scale;
  p.tfull_wait_ns = kWaitLimitNs;
  p.skip_commit = 0;
  if (g_test_fault.load(std::memory_order_relaxed) == MXFP4_TEST_FAULT_WITHHOLD_ACCUMULATOR) {
    p.skip_commit = 1;             // pair 0, first unit
    p.tfull_wait_ns = 1000000ull;  // 1 ms
  }
  if constexpr (FQ) {
    p.x = static_cast<const uint16_t*>(fx->x);
    p.xq = const_cast<uint8_t*>(aq);
    p.xsf = const_cast<uint8_t*>(asf);
    p.rows_done = fx->rows_done;
    p.next_item = fx->rows_done + (M + 127) / 128;  // the word after the row counters
    p.xmode = (uint32_t)fx->mode;
  }
  const uint32_t pairs =
      pl.units < (uint32_t)max_clusters[dev] ? pl.units : (uint32_t)max_clusters[dev];
  if constexpr (FQ) {
    // Work items of up to about 24 steps of 1024 elements (one publication per item), but
    // at least four items per quantiser warp, so that the rows the first tiles need are
    // spread over all the warps and published early.
    const uint32_t spr = (uint32_t)((k_atoms * 4 + 31) / 32);
    const uint64_t qwarps = 2ull * pairs * kQuantWarps;
    uint32_t rpi = 1;
    while (rpi < 16 && 2 * rpi * spr <= 24 && (uint64_t)M >= 2ull * rpi * 4 * qwarps) rpi *= 2;
    p.rows_per_item = rpi;
  }

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, ta, tb, tb64, tsa, tsb, ty, p, ep.kc);
}

}  // namespace

std::atomic<int> g_test_fault{MXFP4_TEST_FAULT_NONE};
std::atomic<int> g_linear_form{MXFP4_LINEAR_AUTO};

cudaError_t launch_gemm(const uint8_t* aq, const uint8_t* asf, const uint8_t* bq,
                        const uint8_t* bsf, int64_t M, int64_t N, int64_t K, void* y,
                        const Epilogue& ep, int64_t ldy, int* status, const GemmScratch& scratch,
                        bool b_early, cudaStream_t stream) {
  // Few activation rows: stream the weights with the swap-AB split-K kernel.
  if (M <= 128)
    return launch_gemm_smallm(aq, asf, bq, bsf, M, N, K, y, ep, ldy, status, scratch, b_early,
                              stream);
  // Otherwise CTA pairs with 256 x 256 tiles.
  if (ep.nvfp4) {
    if (ep.out == kOutF32)
      return launch_pair<5, kOutF32, true>(aq, asf, bq, bsf, M, N, K, y, ep, ldy, status,
                                           stream);
    return launch_pair<5, kOutBf16, true>(aq, asf, bq, bsf, M, N, K, y, ep, ldy, status, stream);
  }
  switch (ep.out) {
    case kOutF32:
      return launch_pair<5, kOutF32, false>(aq, asf, bq, bsf, M, N, K, y, ep, ldy, status, stream);
    case kOutMxfp4:
      return launch_pair<5, kOutMxfp4, false>(aq, asf, bq, bsf, M, N, K, y, ep, ldy, status,
                                              stream);
    default:
      return launch_pair<5, kOutBf16, false>(aq, asf, bq, bsf, M, N, K, y, ep, ldy, status, stream);
  }
}

size_t linear_row_counter_bytes(int64_t M) {
  // one counter per 128 rows, then the quantiser's next work item
  return M > 128 ? (size_t)((M + 127) / 128 + 1) * sizeof(uint32_t) : 0;
}

bool linear_pair_fits(int64_t M, int64_t N, int64_t K, int mode) {
  if (M <= 128 || mode < MXFP4_ROT_NONE || mode > MXFP4_ROT_KRON_4x8) return false;
  const int form = g_linear_form.load(std::memory_order_relaxed);
  if (form != MXFP4_LINEAR_AUTO) return form == MXFP4_LINEAR_ONE_KERNEL;
  // Measured on B200 (DiT-shaped layers, 3584..57344 rows): one kernel is faster once the
  // tiles fill at least 8 rounds of the 74 CTA pairs and x is at least 40 MiB of bf16;
  // below that, quantising the rows the first round needs before it can start costs
  // more than running the quantiser beside the GEMM saves.
  const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
  return tiles >= 8 * 74 && 2 * M * K >= (40ll << 20);
}

cudaError_t launch_linear_pair(const void* x, int mode, const KronCoeffs* kc, uint8_t* xq,
                               uint8_t* xsf, uint32_t* rows_done, const uint8_t* wq,
                               const uint8_t* wsf, int64_t M, int64_t N, int64_t K, void* y,
                               int* status, cudaStream_t stream) {
  if (!linear_pair_fits(M, N, K, mode)) return cudaErrorNotSupported;
  // The counters start at zero in every call (a timed-out call may have left them set).
  cudaError_t e = cudaMemsetAsync(rows_done, 0, linear_row_counter_bytes(M), stream);
  if (e != cudaSuccess) return e;
  Epilogue ep{};
  if (kc) ep.kc = *kc;
  const FusedX fx{x, mode, rows_done};
  return launch_pair<5, kOutBf16, false, true>(xq, xsf, wq, wsf, M, N, K, y, ep, N, status,
                                               stream, &fx);
}

size_t gemm_scratch_bytes(int64_t M, int64_t N, int64_t K) {
  // the CTA-pair kernel needs no scratch
  return M <= 128 ? gemm_smallm_scratch_bytes(M, N, K) : 0;
}

}  // namespace mxfp4
