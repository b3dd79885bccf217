// internal.h -- declarations shared by the library's translation units (not installed).
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>

#include "../../include/mxfp4.h"

namespace mxfp4 {

// Kronecker factors, passed to the kernel by value (constant bank).
struct KronCoeffs {
  float a[16];  // A, 4x4 row-major
  float b[64];  // B, 8x8 row-major
  // The same numbers laid out for packed (two-lane) FMAs, filled by kron_derive:
  // bt[8 l + k] = B[k][l] (two outputs k, k + 1 per pair), a2[2 q] = a2[2 q + 1] = a[q].
  alignas(8) float bt[64];
  alignas(8) float a2[32];
};

inline void kron_derive(KronCoeffs* kc) {
  for (int k = 0; k < 8; ++k)
    for (int l = 0; l < 8; ++l) kc->bt[8 * l + k] = kc->b[8 * k + l];
  for (int q = 0; q < 16; ++q) kc->a2[2 * q] = kc->a2[2 * q + 1] = kc->a[q];
}

// Rotate (mode 0/1/2) + quantise x[rows, K] (bf16 or fp32) into packed codes q and
// scale bytes sf (tensor-core layout, padding zeroed). Host-validated arguments.
// status: optional device word set to the timeout code if a bounded wait gives up.
cudaError_t launch_rotate_quantize(const void* x, bool x_is_f32, int64_t rows, int64_t K,
                                   int64_t ldx, int mode, const KronCoeffs* kc, uint8_t* q,
                                   uint8_t* sf, int* status, cudaStream_t stream);

// NVFP4 (quantize.cu): tensor scale of x rotated by mode (0 / 1) into scale2[0], and the
// quantiser with that scale: codes as for MXFP4, E4M3 group bytes in atoms of 4 groups of
// 16 (sf_katoms(2K) per row tile). The scale pass is one kernel whose last block writes
// the scale; state: two device words that are zero and that it leaves zero (running
// maximum, block counter), or null: scale2[0..1] are zeroed by a memset and used instead.
cudaError_t launch_nvfp4_tensor_scale(const void* x, bool x_is_f32, int64_t rows, int64_t K,
                                     int64_t ldx, int mode, float* scale2, cudaStream_t stream,
                                     unsigned int* state = nullptr);
cudaError_t launch_nvfp4_quantize(const void* x, bool x_is_f32, int64_t rows, int64_t K,
                                  int64_t ldx, int mode, const float* tensor_scale, uint8_t* q,
                                  uint8_t* sf, int* status, cudaStream_t stream);

// Norm prologue (quantize.cu): per-row statistics of bf16 x into stats [rows][2] (kind 0
// LayerNorm: mean, 1/sqrt(var + eps); kind 1 RMSNorm: 0, 1/sqrt(mean(x^2) + eps)), then
// the quantiser applies v = ((x - mu) * rstd) * g + b before rotating (modes 0, 1, 2).
// One kernel when norm_one_pass(K) (quantize_norm.cu: rows copied whole into shared memory,
// two buffers of at least one row in 200 KB: K <= 51168), else a statistics kernel and
// the quantiser.
bool norm_one_pass(int64_t K);
cudaError_t launch_norm_one_pass(const void* x, int64_t rows, int64_t K, int64_t ldx, int kind,
                                 float eps, const float* g, const float* b, int mode,
                                 const KronCoeffs* kc, uint8_t* q, uint8_t* sf, float* stats,
                                 int* status, cudaStream_t stream);
cudaError_t launch_norm_rotate_quantize(const void* x, int64_t rows, int64_t K, int64_t ldx,
                                       int kind, float eps, const float* g, const float* b,
                                       int mode, const KronCoeffs* kc, uint8_t* q, uint8_t* sf,
                                       float* stats, int* status, cudaStream_t stream);

// Rotation over 64- or 128-element groups (span) + quantisation of fp32 rows
// (quantize_wide.cu); cudaErrorNotSupported for bf16, which the tile quantiser handles.
cudaError_t launch_rotate_quantize_wide(const void* x, bool x_is_f32, int64_t rows, int64_t K,
                                        int64_t ldx, int span, uint8_t* q, uint8_t* sf,
                                        cudaStream_t stream);

// Elements per rotation group of a mode (0, 1, 2: 32; 3: 64; 4: 128).
inline int64_t rotation_span(int mode) { return mode == 3 ? 64 : mode == 4 ? 128 : 32; }

// What the GEMM epilogue writes.
enum OutKind { kOutBf16 = 0, kOutF32 = 1, kOutMxfp4 = 2 };
struct Epilogue {
  int out = kOutBf16;
  const float* bias = nullptr;  // [N] fp32 added to every row before the output step
  // kOutMxfp4 only: each 32-column block of a row is rotated (mode 0/1/2 with kc) and
  // quantised; y holds the packed codes [M, N/2] (ldy bytes per row), ysf the scales in
  // the tensor-core layout of an [M, N] operand.
  int mode = 0;
  KronCoeffs kc{};
  uint8_t* ysf = nullptr;
  // NVFP4 operands (16-element groups, E4M3 group scales in atoms of 4 per 64 K): the
  // result is multiplied by *a_scale * *b_scale (device fp32 tensor scales); bf16 / fp32
  // output only.
  bool nvfp4 = false;
  const float* a_scale = nullptr;
  const float* b_scale = nullptr;
};

// Scratch of the GEMM launchers: data_bytes for the few-row kernel's K-split partials
// (fp32), which every launch writes before it reads them, so their previous contents do
// not matter. It may be absent (null): the few-row kernel then sums its K splits on chip
// (same bits). The CTA-pair kernel needs none.
struct GemmScratch {
  uint8_t* data = nullptr;
  size_t data_bytes = 0;
};

// Block-scaled GEMM y[M, N] = A[M, K] . B[N, K]^T on tcgen05. Host-validated arguments.
// status: device word set to the timeout code if a bounded wait gives up.
// Every kernel of the library is launched with programmatic dependent launch: it waits
// for the previous kernel on the stream before touching memory that kernel may share.
// b_early: the kernel just before this launch on the stream does not write bq / bsf, so
// the few-row kernel may start streaming them before that kernel has finished.
cudaError_t launch_gemm(const uint8_t* aq, const uint8_t* asf, const uint8_t* bq,
                        const uint8_t* bsf, int64_t M, int64_t N, int64_t K, void* y,
                        const Epilogue& ep, int64_t ldy, int* status, const GemmScratch& scratch,
                        bool b_early, cudaStream_t stream);

// Bytes of the data part of the scratch that launch_gemm can use for this problem.
size_t gemm_scratch_bytes(int64_t M, int64_t N, int64_t K);

// Few-row path (M <= 128): swap-AB, K split across the CTAs of a cluster (gemm_smallm.cu).
// For 33..128 rows split 4 or more ways the K-split partials go through the data part of
// the scratch (gemm_smallm_scratch_bytes) when it is large enough, else they are summed
// through distributed shared memory. Either way the bits are the same.
cudaError_t launch_gemm_smallm(const uint8_t* aq, const uint8_t* asf, const uint8_t* bq,
                               const uint8_t* bsf, int64_t M, int64_t N, int64_t K, void* y,
                               const Epilogue& ep, int64_t ldy, int* status,
                               const GemmScratch& scratch, bool b_early, cudaStream_t stream);
size_t gemm_smallm_scratch_bytes(int64_t M, int64_t N, int64_t K);

// Testing only (mxfp4_test_set_fault): a fault the next GEMM launches simulate, read on
// the host when a launch is set up. MXFP4_TEST_FAULT_NONE in every product path.
extern std::atomic<int> g_test_fault;

// The whole layer for 1..8 bf16 activation rows in one launch (gemm_smallm.cu): each
// CTA rotates (mode 0/1/2) and quantises its own K range of x into shared memory while
// it streams W. Returns cudaErrorNotSupported (launching nothing) when the problem is
// outside that kernel's limits (linear_smallm_fits false); the caller then quantises
// and multiplies separately.
bool linear_smallm_fits(int64_t M, int64_t N, int64_t K, int mode);
cudaError_t launch_linear_smallm(const void* x, int64_t ldx, int mode, const KronCoeffs* kc,
                                 const uint8_t* wq, const uint8_t* wsf, int64_t M, int64_t N,
                                 int64_t K, void* y, int64_t ldy, int* status,
                                 cudaStream_t stream);

// The whole layer for more than 128 rows in one launch (gemm.cu): the CTA-pair GEMM with
// six more warps per CTA that rotate (mode 0/1/2) and quantise x into xq / xsf while the
// other warps multiply; the TMA producer of each CTA waits, per 128-row group of A, for
// rows_done[group] to reach the group's row count. rows_done: linear_row_counter_bytes(M)
// bytes, cleared here (one memset) before the launch. Returns cudaErrorNotSupported
// (launching nothing) when linear_pair_fits is false.
// linear_pair_fits: whether the layer takes this form (sizes and mode, or the form set by
// mxfp4_set_linear_form). Host only.
extern std::atomic<int> g_linear_form;
bool linear_pair_fits(int64_t M, int64_t N, int64_t K, int mode);
size_t linear_row_counter_bytes(int64_t M);
cudaError_t launch_linear_pair(const void* x, int mode, const KronCoeffs* kc, uint8_t* xq,
                               uint8_t* xsf, uint32_t* rows_done, const uint8_t* wq,
                               const uint8_t* wsf, int64_t M, int64_t N, int64_t K, void* y,
                               int* status, cudaStream_t stream);

// Scale-factor layout helpers (host side).
inline int64_t sf_katoms(int64_t K) { return (K / 32 + 3) / 4; }
inline int64_t sf_row_tiles(int64_t rows) { return (rows + 127) / 128; }

// ---- argument checks and workspace layouts shared by the entry points (abi.cu, noalloc.cu)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Valid [rows, K] operand description for the scale layout.
inline bool shape_ok(int64_t rows, int64_t K) { return rows >= 0 && K >= 32 && K % 32 == 0; }

// Limits of the kernels' 32-bit index arithmetic.
inline bool within_limits(int64_t rows, int64_t K) {
  const int64_t units = sf_row_tiles(rows) * 128 * sf_katoms(K) * 4;
  return rows < (1ll << 31) && K < (1ll << 31) && units < (1ll << 32);
}

inline bool mode_ok(int mode) { return mode >= MXFP4_ROT_NONE && mode <= MXFP4_ROT_HADAMARD128; }

// A row operand (activations, their codes and scales, the output) may be NULL when it has
// no rows: torch and other frameworks hand out NULL for empty tensors.
inline bool rows_ptr_ok(const void* p, int64_t rows) { return p != nullptr || rows == 0; }

// Kronecker factors from host memory into the kernel-parameter form; false if one is NULL.
inline bool kron_from_host(const float* a, const float* b, KronCoeffs* out) {
  if (!a || !b) return false;
  std::memcpy(out->a, a, sizeof(out->a));
  std::memcpy(out->b, b, sizeof(out->b));
  kron_derive(out);
  return true;
}

// Checks of the layer's arguments (mxfp4_linear and mxfp4_linear_noalloc reject exactly
// the same calls), and the Kronecker coefficients when mode needs them.
mxfp4_status validate_linear(const void* x, int64_t M, int64_t K, mxfp4_rotation mode,
                             const float* kron_a, const float* kron_b, const uint8_t* wq,
                             const uint8_t* wsf, int64_t N, const void* y, KronCoeffs* kc);

// Every workspace starts with the status region: the status word at byte 0, the NVFP4
// layer's tensor scale and its pass's state at 64..79.
constexpr size_t kHeadBytes = 256;

// Layout of the layer's workspace: [status | Xq (M x K/2) | Xsf (sf_k-element operand
// scales) | GEMM data], parts 256-byte aligned. sf_k = K for MXFP4, 2 K for NVFP4. With
// row_counters (the MXFP4 layer), the last part also holds the one-launch layer's row
// counters for more than 128 rows (the pair GEMM needs no data there).
struct LinearLayout {
  size_t q_off, sf_off, g_off, total;
};
LinearLayout linear_layout(int64_t M, int64_t N, int64_t K, int64_t sf_k,
                           bool row_counters = false);

// The GEMM scratch of a workspace laid out as above (data part: from g_off to ws_bytes).
inline GemmScratch workspace_scratch(uint8_t* ws, size_t g_off, size_t ws_bytes) {
  GemmScratch g;
  g.data = ws_bytes > g_off ? ws + g_off : nullptr;
  g.data_bytes = ws_bytes > g_off ? ws_bytes - g_off : 0;
  return g;
}

}  // namespace mxfp4
