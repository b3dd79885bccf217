// quantize_norm.cu -- the norm prologue in one pass over x: LayerNorm / RMSNorm
// statistics, normalisation, online rotation and MXFP4 quantisation of bf16 rows.
//
// One CTA per SM (512 threads) works through groups of R whole rows. With groups of 16
// rows a CTA takes a contiguous run of rows (the runs of all CTAs differ by at most one
// row; the last group of a run is partial), so that no CTA works a whole group more
// than another; with smaller groups it takes group blockIdx.x and every gridDim.x-th
// after it (B200, 3584 rows: K = 3072 in runs 17.7 -> 14.8 us, but K = 12288 in runs of
// 4-row groups 64 -> 66 us, so those keep the interleaved order). The groups stream into
// a ring of NB shared-memory buffers, one bulk copy per row, NB - 1 groups ahead of the
// one being worked on. For each group the CTA
// takes every row's statistics from that copy (16 / R warps per row, partial sums
// combined in a fixed order) and then normalises, rotates and quantises all of the
// group's 32-element blocks from the same copy, with the norm's g and b from shared
// memory when they fit beside the ring (staged once per CTA, 16 bytes of padding after
// every 32 values so that the two or more blocks a warp reads at once fall on
// different banks). x is read from HBM once, where a statistics kernel followed by the
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
constexpr uint32_t kNormSmemMax = 232448;   // dynamic shared memory of one CTA
constexpr uint32_t kNormFixed = 1024;       // alignment pad, barriers, statistics
constexpr uint32_t kNormMaxBufs = 16;
constexpr uint32_t kNormInFlight = 96 * 1024;  // row bytes to keep streaming per SM
constexpr uint64_t kNormWaitLimitNs = 2000000000ull;
constexpr int kNormTimeoutCode = 7;  // MXFP4_ERR_TIMEOUT

// Plan of one launch: R rows per group (a power of two <= 16, so that 16 / R warps
// take each row's statistics; the block pass reads the same block of R consecutive rows
// in one warp, and rows 16 bytes apart modulo 128 keep those reads on different banks),
// NB ring buffers, and whether g and b are staged in shared memory.
struct NormPlan {
  uint32_t R = 0, NB = 0;
  bool gb_smem = false;
};

uint32_t norm_pitch(int64_t K) { return (uint32_t)K * 2u + 16u; }
uint32_t norm_gb_bytes(int64_t K) { return (uint32_t)(K / 32) * 144u * 2u; }  // padded g, b

NormPlan norm_plan(int64_t K, bool has_gb) {
  NormPlan pl;
  const uint64_t pitch = norm_pitch(K);
  // The largest group of which two buffers fit; then g and b beside them if they fit
  // too; then as many more buffers (up to kNormMaxBufs) as keep kNormInFlight bytes
  // streaming behind the group being worked on.
  const uint64_t room = kNormSmemMax - kNormFixed;
  uint32_t r = 16;
  while (r > 1 && 2ull * r * pitch > room) r >>= 1;
  if (2ull * r * pitch > room) return pl;  // R = 0: one row does not fit twice
  const uint64_t gb = has_gb ? norm_gb_bytes(K) : 0u;
  const bool use_gb = gb > 0 && 2ull * r * pitch + gb <= room;
  const uint64_t gbytes = (uint64_t)r * pitch;
  uint64_t nb = (room - (use_gb ? gb : 0u)) / gbytes;
  const uint64_t want = (kNormInFlight + gbytes - 1) / gbytes + 1;
  if (nb > want) nb = want;
  if (nb > kNormMaxBufs) nb = kNormMaxBufs;
  pl.R = r;
  pl.NB = (uint32_t)nb;
  pl.gb_smem = use_gb;
  return pl;
}

// Shared memory: [g | b (K floats each, if staged)] [NB row buffers of R rows, `pitch`
// bytes apart: the 16-byte pad puts consecutive rows on different bank groups] [NB
// mbarriers] [abort flag] [per-row (mu, rstd)] [per-warp partial sums].
struct NormSmem {
  uint32_t pitch, gb_bytes, buf_off, buf_bytes, bar, abort_off, st_off, part_off, total;
  __host__ __device__ NormSmem(uint32_t K, uint32_t R, uint32_t NB, bool gb_smem) {
    pitch = K * 2u + 16u;
    gb_bytes = gb_smem ? (K / 32u) * 144u * 2u : 0u;
    buf_off = (gb_bytes + 127u) & ~127u;
    buf_bytes = R * pitch;
    bar = buf_off + NB * buf_bytes;
    abort_off = bar + 8u * NB;
    st_off = abort_off + 16u;
    part_off = st_off + 16u * 8u;
    total = part_off + kNormWarps * 4u;
  }
};

template <int KIND, int MODE, bool GB_SMEM>
__global__ void __launch_bounds__(kNormThreads, 1) norm_rows_kernel(
    const uint16_t* __restrict__ x, uint64_t ldx, uint32_t rows, uint32_t rows_pad, uint32_t K,
    uint32_t R, uint32_t NB, uint32_t n_katoms, float eps,
    const __grid_constant__ KronCoeffs kc, const float* __restrict__ g,
    const float* __restrict__ b, uint8_t* __restrict__ q, uint8_t* __restrict__ sf,
    float* __restrict__ stats, int* status) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_addr(smem_raw) + 127u) & ~127u;
  uint8_t* sptr = smem_raw + (sbase - smem_addr(smem_raw));
  const NormSmem L(K, R, NB, GB_SMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + L.abort_off);
  float2* st_s = reinterpret_cast<float2*>(sptr + L.st_off);
  float* part = reinterpret_cast<float*>(sptr + L.part_off);
  const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
  const uint32_t row_bytes = K * 2u;  // a multiple of 64 (K % 32 == 0)
  const uint32_t chunks = row_bytes / 16u;
  const uint32_t kb_real = K / 32u, kb_pad = n_katoms * 4u;
  // This CTA's groups. Runs (R = 16): a contiguous run [run0, run1) of [0, rows_pad) in
  // groups of R, the last partial. Otherwise groups blockIdx.x + i gridDim.x of R rows.
  const bool runs = R == 16u;
  const uint32_t n_groups = rows_pad / R;
  const uint32_t run0 = runs ? (uint32_t)((uint64_t)rows_pad * blockIdx.x / gridDim.x) : 0u;
  const uint32_t run1 =
      runs ? (uint32_t)((uint64_t)rows_pad * (blockIdx.x + 1u) / gridDim.x) : 0u;
  const uint32_t n_grp = runs ? (run1 - run0 + R - 1u) / R
                         : blockIdx.x < n_groups
                             ? (n_groups - blockIdx.x + gridDim.x - 1u) / gridDim.x
                             : 0u;
  const uint32_t W = kNormWarps / R;  // warps per row in the statistics passes

  if (tid == 0) {
    for (uint32_t i = 0; i < NB; ++i) mbar_init(sbase + L.bar + 8u * i, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Launched with programmatic dependent launch: the kernel before this one may still be
  // writing x or reading q / sf / stats. Wait for it before the first access.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // group i: rows first_row(i) .. + glen(i), of which the first real_rows(i) are < rows
  auto first_row = [&](uint32_t i) -> uint32_t {
    return runs ? run0 + i * R : (blockIdx.x + i * gridDim.x) * R;
  };
  auto glen = [&](uint32_t i) -> uint32_t {
    const uint32_t row0 = first_row(i);
    return runs && run1 - row0 < R ? run1 - row0 : R;
  };
  auto real_rows = [&](uint32_t i) -> uint32_t {
    const uint32_t row0 = first_row(i), n = glen(i);
    return row0 >= rows ? 0u : (rows - row0 < n ? rows - row0 : n);
  };
  uint32_t pending = 0;  // thread 0: bit i set while a copy into buffer i is in flight
  auto issue = [&](uint32_t grp, uint32_t bi) {
    const uint32_t n = real_rows(grp);
    if (n == 0) return;
    const uint32_t bar = sbase + L.bar + 8u * bi;
    mbar_arrive_expect_tx(bar, n * row_bytes);
    for (uint32_t r = 0; r < n; ++r)
      bulk_load(sbase + L.buf_off + bi * L.buf_bytes + r * L.pitch,
                x + (uint64_t)(first_row(grp) + r) * ldx, row_bytes, bar);
    pending |= 1u << bi;
  };
  if (tid == 0)
    for (uint32_t i = 0; i < NB && i < n_grp; ++i) issue(i, i);
  // g and b into shared memory while the first rows stream in
  const float* gs = g;
  const float* bs = b;
  // (staged: the 32 values of block kb at float 36 kb, g first, then b at float 36 K / 32)
  constexpr uint32_t gb_stride = GB_SMEM ? 36u : 32u;
  if constexpr (GB_SMEM) {
    float* gsm = reinterpret_cast<float*>(sptr);
    float* bsm = gsm + 36u * (K / 32u);
    for (uint32_t i = tid; i < K / 4u; i += kNormThreads) {
      const uint32_t at = (i >> 3) * 36u + (i & 7u) * 4u;
      *reinterpret_cast<float4*>(gsm + at) =
          g ? __ldg(reinterpret_cast<const float4*>(g) + i) : make_float4(1.f, 1.f, 1.f, 1.f);
      *reinterpret_cast<float4*>(bsm + at) =
          b ? __ldg(reinterpret_cast<const float4*>(b) + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    gs = g ? gsm : nullptr;
    bs = b ? bsm : nullptr;
    __syncthreads();
  }

  uint32_t phase = 0;  // bit i: parity of buffer i's next completion
  bool aborted = false;
  uint32_t bi = 0;
  for (uint32_t grp = 0; grp < n_grp; ++grp) {
    const uint32_t row0 = first_row(grp);
    const uint32_t nreal = real_rows(grp);
    const uint32_t nrows = glen(grp);
    const uint32_t buf = sbase + L.buf_off + bi * L.buf_bytes;
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
      // (w % W) 32 + l + 32 W i, i = 0, 1, ..., into four paired partial sums by i mod 4
      // (each adds a chunk's 8 elements as 4 pairs), added as
      // ((p0 + p1) + (p2 + p3)) and then the two halves of the pair; the warp's lanes are
      // then added by a butterfly and the W slices of a row in slice order.
      const uint32_t r = warp / W, sl = warp - r * W;
      const uint32_t rbase = buf + r * L.pitch;
      const uint32_t cstep = 32u * W;
      float mu = 0.0f;
      if constexpr (KIND == 0) {
        float2 p4[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
        if (r < nreal)
          for (uint32_t c0 = sl * 32u + lane; c0 < chunks; c0 += 4u * cstep) {
#pragma unroll
            for (uint32_t j = 0; j < 4; ++j) {
              const uint32_t c = c0 + j * cstep;
              if (c < chunks) {
                const uint4 w = ld_shared_v4(rbase + c * 16u);
                float2 t = __fadd2_rn(make_float2(bf16_lo(w.x), bf16_hi(w.x)),
                                      make_float2(bf16_lo(w.y), bf16_hi(w.y)));
                t = __fadd2_rn(t, make_float2(bf16_lo(w.z), bf16_hi(w.z)));
                t = __fadd2_rn(t, make_float2(bf16_lo(w.w), bf16_hi(w.w)));
                p4[j] = __fadd2_rn(p4[j], t);
              }
            }
          }
        const float2 h = __fadd2_rn(__fadd2_rn(p4[0], p4[1]), __fadd2_rn(p4[2], p4[3]));
        float s = h.x + h.y;
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
      float2 q4[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
      const float2 nmu2 = make_float2(-mu, -mu);
      if (r < nreal)
        for (uint32_t c0 = sl * 32u + lane; c0 < chunks; c0 += 4u * cstep) {
#pragma unroll
          for (uint32_t j = 0; j < 4; ++j) {
            const uint32_t c = c0 + j * cstep;
            if (c < chunks) {
              const uint4 w = ld_shared_v4(rbase + c * 16u);
              float2 d0 = make_float2(bf16_lo(w.x), bf16_hi(w.x));
              float2 d1 = make_float2(bf16_lo(w.y), bf16_hi(w.y));
              float2 d2 = make_float2(bf16_lo(w.z), bf16_hi(w.z));
              float2 d3 = make_float2(bf16_lo(w.w), bf16_hi(w.w));
              if constexpr (KIND == 0) {  // RMSNorm: mu = 0, nothing to subtract
                d0 = __fadd2_rn(d0, nmu2);
                d1 = __fadd2_rn(d1, nmu2);
                d2 = __fadd2_rn(d2, nmu2);
                d3 = __fadd2_rn(d3, nmu2);
              }
              q4[j] = __ffma2_rn(d0, d0, q4[j]);
              q4[j] = __ffma2_rn(d1, d1, q4[j]);
              q4[j] = __ffma2_rn(d2, d2, q4[j]);
              q4[j] = __ffma2_rn(d3, d3, q4[j]);
            }
          }
        }
      const float2 hq = __fadd2_rn(__fadd2_rn(q4[0], q4[1]), __fadd2_rn(q4[2], q4[3]));
      float v = hq.x + hq.y;
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
        // g and b: 16-byte aligned, kb 32 floats apart (from shared memory when staged)
        if (gs != nullptr) {
          const float4* gv = reinterpret_cast<const float4*>(gs + kb * gb_stride);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 t = GB_SMEM ? gv[j] : __ldg(gv + j);
            P[2 * j] = __fmul2_rn(P[2 * j], make_float2(t.x, t.y));
            P[2 * j + 1] = __fmul2_rn(P[2 * j + 1], make_float2(t.z, t.w));
          }
        }
        if (bs != nullptr) {
          const float4* bv = reinterpret_cast<const float4*>(bs + kb * gb_stride);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 t = GB_SMEM ? bv[j] : __ldg(bv + j);
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
    for (uint32_t i = tid; i < nreal * pad_real + (nrows - nreal) * kb_pad; i += kNormThreads) {
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
    __syncthreads();  // this buffer is read: the group NB ahead may be copied into it
    if (tid == 0 && grp + NB < n_grp) issue(grp + NB, bi);
    bi = bi + 1u == NB ? 0u : bi + 1u;
  }
  // After an early stop, copies already issued still land in this CTA's shared memory.
  if (aborted && tid == 0) {
    volatile int never = 0;
    uint32_t b2 = bi;
    for (uint32_t n = 0; n < NB; ++n, b2 = b2 + 1u == NB ? 0u : b2 + 1u)
      if ((pending >> b2) & 1u)
        mbar_wait_bounded(sbase + L.bar + 8u * b2, (phase >> b2) & 1u, &never, kNormWaitLimitNs);
  }
}

template <int KIND, int MODE>
cudaError_t launch_kind_mode(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx, float eps,
                             const KronCoeffs& kc, const float* g, const float* b, uint8_t* q,
                             uint8_t* sf, float* stats, int* status, cudaStream_t stream) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  static size_t smem_set[64][2] = {};
  static int sms[64] = {};
  if (!sms[dev]) cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
  const int64_t rows_pad = sf_row_tiles(rows) * 128;
  const NormPlan pl = norm_plan(K, g != nullptr || b != nullptr);
  if (pl.R == 0) return cudaErrorNotSupported;
  const uint32_t R = pl.R;
  auto kern = pl.gb_smem ? norm_rows_kernel<KIND, MODE, true> : norm_rows_kernel<KIND, MODE, false>;
  const size_t smem = 128 + NormSmem((uint32_t)K, R, pl.NB, pl.gb_smem).total;
  if (smem_set[dev][pl.gb_smem ? 1 : 0] < smem) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    smem_set[dev][pl.gb_smem ? 1 : 0] = smem;
  }
  // runs: any number of CTAs up to the rows; groups: up to the groups
  const int64_t units = R == 16 ? rows_pad : rows_pad / R;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(units < sms[dev] ? units : sms[dev]));
  cfg.blockDim = dim3(kNormThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, x, (uint64_t)ldx, (uint32_t)rows, (uint32_t)rows_pad,
                            (uint32_t)K, R, pl.NB, (uint32_t)sf_katoms(K), eps, kc, g, b, q, sf,
                            stats, status);
}

}  // namespace

// One pass while two rows (with their 16-byte pads) fit 200 KB of shared memory.
bool norm_one_pass(int64_t K) { return K > 0 && 2ull * norm_pitch(K) <= 200u * 1024u; }

cudaError_t launch_norm_one_pass(const void* x, int64_t rows, int64_t K, int64_t ldx, int kind,
                                 float eps, const float* g, const float* b, int mode,
                                 const KronCoeffs* kc, uint8_t* q, uint8_t* sf, float* stats,
                                 int* status, cudaStream_t stream) {
  if (!norm_one_pass(K)) return cudaErrorNotSupported;
  KronCoeffs k{};
  if (kc) k = *kc;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
#define MXFP4_NORM_ROWS(KINDV, MODEV)                                                  \
  return launch_kind_mode<KINDV, MODEV>(xb, rows, K, ldx, eps, k, g, b, q, sf, stats, \
                                        status, stream)
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
