// abi.cu -- the extern "C" entry points of libmxfp4 (declared in include/mxfp4.h):
// argument validation, workspace layout and kernel dispatch. No device memory
// is allocated here; every launch is ordered on the caller's stream.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <utility>

#include "internal.h"

using namespace mxfp4;

namespace {

mxfp4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MXFP4_OK : MXFP4_ERR_CUDA; }

// Checks shared by the two NVFP4 layer entry points.
mxfp4_status validate_nvfp4_linear(const void* x, int64_t M, int64_t K, mxfp4_rotation mode,
                                   const uint8_t* wq, const uint8_t* wsf, const float* w_scale,
                                   int64_t N, const void* y, const void* ws, size_t ws_bytes) {
  if (!rows_ptr_ok(x, M) || !wq || !wsf || !w_scale || !rows_ptr_ok(y, M) || !ws)
    return MXFP4_ERR_INVALID_ARG;
  if (mode != MXFP4_ROT_NONE && mode != MXFP4_ROT_HADAMARD32) return MXFP4_ERR_UNSUPPORTED;
  if (!shape_ok(M, K) || N < 16 || N % 16 != 0 || !within_limits(M, 2 * K) ||
      !within_limits(N, 2 * K))
    return MXFP4_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(wq) || !aligned16(wsf) || !aligned16(y) || !aligned16(ws) ||
      (K * 2) % 16 != 0 || (N * 2) % 16 != 0 || (reinterpret_cast<uintptr_t>(w_scale) & 3u))
    return MXFP4_ERR_ALIGN;
  if (ws_bytes < linear_layout(M, N, K, 2 * K).total) return MXFP4_ERR_WORKSPACE;
  return MXFP4_OK;
}

mxfp4_status validate_quantize(const void* x, mxfp4_dtype xdt, int64_t rows, int64_t K,
                               int64_t ldx, const uint8_t* q, const uint8_t* sf) {
  if (!rows_ptr_ok(x, rows) || !rows_ptr_ok(q, rows) || !rows_ptr_ok(sf, rows))
    return MXFP4_ERR_INVALID_ARG;
  if (xdt != MXFP4_DT_BF16 && xdt != MXFP4_DT_F32) return MXFP4_ERR_UNSUPPORTED;
  if (!shape_ok(rows, K) || ldx < K || !within_limits(rows, K)) return MXFP4_ERR_SHAPE;
  const int64_t esize = xdt == MXFP4_DT_F32 ? 4 : 2;
  if (!aligned16(x) || !aligned16(q) || !aligned16(sf) || (ldx * esize) % 16 != 0)
    return MXFP4_ERR_ALIGN;
  return MXFP4_OK;
}

mxfp4_status validate_gemm(const uint8_t* aq, const uint8_t* asf, const uint8_t* bq,
                           const uint8_t* bsf, int64_t M, int64_t N, int64_t K, const void* y,
                           mxfp4_dtype ydt, int64_t ldy) {
  if (!rows_ptr_ok(aq, M) || !rows_ptr_ok(asf, M) || !bq || !bsf || !rows_ptr_ok(y, M))
    return MXFP4_ERR_INVALID_ARG;
  if (ydt != MXFP4_DT_BF16 && ydt != MXFP4_DT_F32) return MXFP4_ERR_UNSUPPORTED;
  if (!shape_ok(M, K) || N < 16 || N % 16 != 0 || ldy < N || !within_limits(M, K) ||
      !within_limits(N, K))
    return MXFP4_ERR_SHAPE;
  const int64_t esize = ydt == MXFP4_DT_F32 ? 4 : 2;
  if (!aligned16(aq) || !aligned16(asf) || !aligned16(bq) || !aligned16(bsf) || !aligned16(y) ||
      (ldy * esize) % 16 != 0)
    return MXFP4_ERR_ALIGN;
  return MXFP4_OK;
}

// The GEMM scratch of a GEMM-only workspace: [status | data].
GemmScratch gemm_workspace_scratch(void* ws, size_t ws_bytes) {
  if (ws_bytes < kHeadBytes) return GemmScratch{};
  return workspace_scratch(static_cast<uint8_t*>(ws), kHeadBytes, ws_bytes);
}

// Workspace of mxfp4_nvfp4_linear: the layer layout with NVFP4 scale bytes; the status
// region holds the X tensor scale at 64 and the scale pass's running maximum and block
// counter at 72 and 76.
constexpr size_t kScaleOff = 64;

// Workspace of mxfp4_norm_linear: [status | Xq | Xsf | row statistics (M x 8
// bytes) | GEMM data].
struct NormWorkspace {
  size_t q_off, sf_off, st_off, g_off, total;
};

NormWorkspace norm_linear_workspace(int64_t M, int64_t N, int64_t K) {
  const LinearLayout l = linear_layout(M, N, K, K);
  NormWorkspace w;
  w.q_off = l.q_off;
  w.sf_off = l.sf_off;
  w.st_off = l.g_off;
  w.g_off = round_up(w.st_off + (size_t)M * 2 * sizeof(float), 256);
  w.total = round_up(w.g_off + gemm_scratch_bytes(M, N, K), 256);
  return w;
}

// Inverse of the n x n row-major matrix a (n <= 8) in double by Gauss-Jordan elimination
// on [a | I], choosing as pivot the largest magnitude in the column at or below the
// diagonal; false if a pivot is zero or a value is not finite.
bool invert_small(const float* a, int n, double* inv) {
  double m[8][16];
  for (int r = 0; r < n; ++r)
    for (int c = 0; c < 2 * n; ++c)
      m[r][c] = c < n ? (double)a[r * n + c] : (c - n == r ? 1.0 : 0.0);
  for (int col = 0; col < n; ++col) {
    int piv = col;
    for (int r = col + 1; r < n; ++r)
      if (std::fabs(m[r][col]) > std::fabs(m[piv][col])) piv = r;
    if (!(std::fabs(m[piv][col]) > 0.0) || !std::isfinite(m[piv][col])) return false;
    if (piv != col)
      for (int c = 0; c < 2 * n; ++c) std::swap(m[piv][c], m[col][c]);
    const double d = m[col][col];
    for (int c = 0; c < 2 * n; ++c) m[col][c] /= d;
    for (int r = 0; r < n; ++r) {
      if (r == col) continue;
      const double f = m[r][col];
      if (f == 0.0) continue;
      for (int c = 0; c < 2 * n; ++c) m[r][c] -= f * m[col][c];
    }
  }
  for (int r = 0; r < n; ++r)
    for (int c = 0; c < n; ++c) {
      inv[r * n + c] = m[r][n + c];
      if (!std::isfinite(inv[r * n + c])) return false;
    }
  return true;
}

}  // namespace

namespace mxfp4 {

LinearLayout linear_layout(int64_t M, int64_t N, int64_t K, int64_t sf_k, bool row_counters) {
  LinearLayout w;
  w.q_off = kHeadBytes;
  w.sf_off = round_up(w.q_off + (size_t)M * (size_t)(K / 2), 256);
  w.g_off = round_up(w.sf_off + mxfp4_sf_bytes(M, sf_k), 256);
  size_t last = gemm_scratch_bytes(M, N, K);  // few-row GEMM data (M <= 128)
  if (row_counters && linear_row_counter_bytes(M) > last) last = linear_row_counter_bytes(M);
  w.total = round_up(w.g_off + last, 256);
  return w;
}

mxfp4_status validate_linear(const void* x, int64_t M, int64_t K, mxfp4_rotation mode,
                             const float* kron_a, const float* kron_b, const uint8_t* wq,
                             const uint8_t* wsf, int64_t N, const void* y, KronCoeffs* kc) {
  if (!rows_ptr_ok(x, M) || !wq || !wsf || !rows_ptr_ok(y, M)) return MXFP4_ERR_INVALID_ARG;
  if (!mode_ok(mode)) return MXFP4_ERR_UNSUPPORTED;
  if (!shape_ok(M, K) || K % rotation_span(mode) != 0 || N < 16 || N % 16 != 0 ||
      !within_limits(M, K) || !within_limits(N, K))
    return MXFP4_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(wq) || !aligned16(wsf) || !aligned16(y) ||
      (K * 2) % 16 != 0 || (N * 2) % 16 != 0)
    return MXFP4_ERR_ALIGN;
  if (mode == MXFP4_ROT_KRON_4x8 && !kron_from_host(kron_a, kron_b, kc))
    return MXFP4_ERR_INVALID_ARG;
  return MXFP4_OK;
}

}  // namespace mxfp4

extern "C" {

size_t mxfp4_sf_bytes(int64_t rows, int64_t K) {
  if (!shape_ok(rows, K)) return 0;
  return (size_t)(sf_row_tiles(rows) * sf_katoms(K) * 512);
}

int64_t mxfp4_sf_offset(int64_t row, int64_t kblock, int64_t K) {
  if (K < 32 || K % 32 != 0 || row < 0 || kblock < 0 || kblock >= K / 32) return -1;
  return ((row / 128) * sf_katoms(K) + kblock / 4) * 512 + (row % 32) * 16 +
         ((row / 32) % 4) * 4 + (kblock % 4);
}

size_t mxfp4_workspace_bytes(int op, int64_t M, int64_t N, int64_t K) {
  (void)N;
  switch (op) {
    case MXFP4_OP_QUANTIZE:
      return 0;
    case MXFP4_OP_GEMM:
      if (!shape_ok(M, K) || N < 0) return kHeadBytes;
      return kHeadBytes + round_up(gemm_scratch_bytes(M, N, K), 256);
    case MXFP4_OP_LINEAR:
      if (!shape_ok(M, K) || N < 0) return 0;
      return linear_layout(M, N, K, K, true).total;
    case MXFP4_OP_NVFP4_LINEAR:
      if (!shape_ok(M, K) || N < 0) return 0;
      return linear_layout(M, N, K, 2 * K).total;
    case MXFP4_OP_NORM_LINEAR:
      if (!shape_ok(M, K) || N < 0) return 0;
      return norm_linear_workspace(M, N, K).total;
    default:
      return 0;
  }
}

const char* mxfp4_status_string(mxfp4_status s) {
  switch (s) {
    case MXFP4_OK: return "ok";
    case MXFP4_ERR_INVALID_ARG: return "invalid argument (null pointer)";
    case MXFP4_ERR_SHAPE: return "unsupported shape";
    case MXFP4_ERR_ALIGN: return "pointer or row stride not 16-byte aligned";
    case MXFP4_ERR_WORKSPACE: return "workspace too small";
    case MXFP4_ERR_UNSUPPORTED: return "unsupported mode or dtype";
    case MXFP4_ERR_CUDA: return "CUDA launch error";
    case MXFP4_ERR_TIMEOUT: return "a kernel's bounded wait expired (output incomplete)";
  }
  return "unknown status";
}

mxfp4_status mxfp4_quantize(const void* x, mxfp4_dtype xdt, int64_t rows, int64_t K, int64_t ldx,
                            uint8_t* q, uint8_t* sf, mxfp4_stream_t stream) {
  return mxfp4_rotate_quantize(x, xdt, rows, K, ldx, MXFP4_ROT_NONE, nullptr, nullptr, q, sf,
                               stream);
}

mxfp4_status mxfp4_rotate_quantize(const void* x, mxfp4_dtype xdt, int64_t rows, int64_t K,
                                   int64_t ldx, mxfp4_rotation mode, const float* kron_a,
                                   const float* kron_b, uint8_t* q, uint8_t* sf,
                                   mxfp4_stream_t stream) {
  mxfp4_status st = validate_quantize(x, xdt, rows, K, ldx, q, sf);
  if (st != MXFP4_OK) return st;
  if (!mode_ok(mode)) return MXFP4_ERR_UNSUPPORTED;
  if (K % rotation_span(mode) != 0) return MXFP4_ERR_SHAPE;
  KronCoeffs kc{};
  if (mode == MXFP4_ROT_KRON_4x8 && !kron_from_host(kron_a, kron_b, &kc))
    return MXFP4_ERR_INVALID_ARG;
  if (rows == 0) return MXFP4_OK;
  return from_cuda(launch_rotate_quantize(x, xdt == MXFP4_DT_F32, rows, K, ldx, (int)mode, &kc, q,
                                          sf, nullptr, static_cast<cudaStream_t>(stream)));
}

mxfp4_status mxfp4_gemm(const uint8_t* aq, const uint8_t* asf, const uint8_t* bq,
                        const uint8_t* bsf, int64_t M, int64_t N, int64_t K, void* y,
                        mxfp4_dtype ydt, int64_t ldy, void* ws, size_t ws_bytes,
                        mxfp4_stream_t stream) {
  mxfp4_status st = validate_gemm(aq, asf, bq, bsf, M, N, K, y, ydt, ldy);
  if (st != MXFP4_OK) return st;
  if (!ws) return MXFP4_ERR_INVALID_ARG;
  if (!aligned16(ws)) return MXFP4_ERR_ALIGN;
  if (ws_bytes < kHeadBytes) return MXFP4_ERR_WORKSPACE;  // scratch: optional, see header
  if (M == 0) return MXFP4_OK;
  // The caller's previous kernel may have written bq / bsf: no early weight loads.
  Epilogue ep;
  ep.out = ydt == MXFP4_DT_F32 ? kOutF32 : kOutBf16;
  return from_cuda(launch_gemm(aq, asf, bq, bsf, M, N, K, y, ep, ldy, static_cast<int*>(ws),
                               gemm_workspace_scratch(ws, ws_bytes), false,
                               static_cast<cudaStream_t>(stream)));
}

mxfp4_status mxfp4_gemm_bias(const uint8_t* aq, const uint8_t* asf, const uint8_t* bq,
                             const uint8_t* bsf, int64_t M, int64_t N, int64_t K,
                             const float* bias, void* y, mxfp4_dtype ydt, int64_t ldy, void* ws,
                             size_t ws_bytes, mxfp4_stream_t stream) {
  mxfp4_status st = validate_gemm(aq, asf, bq, bsf, M, N, K, y, ydt, ldy);
  if (st != MXFP4_OK) return st;
  if (!ws || !bias) return MXFP4_ERR_INVALID_ARG;
  if (!aligned16(ws) || !aligned16(bias)) return MXFP4_ERR_ALIGN;
  if (ws_bytes < kHeadBytes) return MXFP4_ERR_WORKSPACE;  // scratch: optional, see header
  if (M == 0) return MXFP4_OK;
  Epilogue ep;
  ep.out = ydt == MXFP4_DT_F32 ? kOutF32 : kOutBf16;
  ep.bias = bias;
  return from_cuda(launch_gemm(aq, asf, bq, bsf, M, N, K, y, ep, ldy, static_cast<int*>(ws),
                               gemm_workspace_scratch(ws, ws_bytes), false,
                               static_cast<cudaStream_t>(stream)));
}

mxfp4_status mxfp4_gemm_quantize(const uint8_t* aq, const uint8_t* asf, const uint8_t* bq,
                                 const uint8_t* bsf, int64_t M, int64_t N, int64_t K,
                                 const float* bias, mxfp4_rotation mode, const float* kron_a,
                                 const float* kron_b, uint8_t* yq, uint8_t* ysf, void* ws,
                                 size_t ws_bytes, mxfp4_stream_t stream) {
  if (!rows_ptr_ok(aq, M) || !rows_ptr_ok(asf, M) || !bq || !bsf || !rows_ptr_ok(yq, M) ||
      !rows_ptr_ok(ysf, M) || !ws)
    return MXFP4_ERR_INVALID_ARG;
  // the epilogue rotates within one 32-column block: no larger Hadamard groups here
  if (mode != MXFP4_ROT_NONE && mode != MXFP4_ROT_HADAMARD32 && mode != MXFP4_ROT_KRON_4x8)
    return MXFP4_ERR_UNSUPPORTED;
  if (!shape_ok(M, K) || N < 32 || N % 32 != 0 || !within_limits(M, K) || !within_limits(N, K) ||
      !within_limits(M, N))
    return MXFP4_ERR_SHAPE;
  if (!aligned16(aq) || !aligned16(asf) || !aligned16(bq) || !aligned16(bsf) || !aligned16(yq) ||
      !aligned16(ysf) || !aligned16(ws) || (bias && !aligned16(bias)))
    return MXFP4_ERR_ALIGN;
  if (ws_bytes < kHeadBytes) return MXFP4_ERR_WORKSPACE;  // scratch: optional, see header
  Epilogue ep;
  ep.out = kOutMxfp4;
  ep.bias = bias;
  ep.mode = (int)mode;
  ep.ysf = ysf;
  if (mode == MXFP4_ROT_KRON_4x8 && !kron_from_host(kron_a, kron_b, &ep.kc))
    return MXFP4_ERR_INVALID_ARG;
  if (M == 0) return MXFP4_OK;
  return from_cuda(launch_gemm(aq, asf, bq, bsf, M, N, K, yq, ep, N / 2, static_cast<int*>(ws),
                               gemm_workspace_scratch(ws, ws_bytes), false,
                               static_cast<cudaStream_t>(stream)));
}

mxfp4_status mxfp4_linear(const void* x, int64_t M, int64_t K, mxfp4_rotation mode,
                          const float* kron_a, const float* kron_b, const uint8_t* wq,
                          const uint8_t* wsf, int64_t N, void* y, void* ws, size_t ws_bytes,
                          mxfp4_stream_t stream) {
  KronCoeffs kc{};
  const mxfp4_status st = validate_linear(x, M, K, mode, kron_a, kron_b, wq, wsf, N, y, &kc);
  if (st != MXFP4_OK) return st;
  if (!ws) return MXFP4_ERR_INVALID_ARG;
  if (!aligned16(ws)) return MXFP4_ERR_ALIGN;
  const LinearLayout w = linear_layout(M, N, K, K, true);
  if (ws_bytes < w.total) return MXFP4_ERR_WORKSPACE;
  if (M == 0) return MXFP4_OK;
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t* xq = base + w.q_off;
  uint8_t* xsf = base + w.sf_off;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // 1..8 rows: one kernel quantises x inside the GEMM's CTAs.
  cudaError_t e = launch_linear_smallm(x, K, (int)mode, &kc, wq, wsf, M, N, K, y, N,
                                       static_cast<int*>(ws), s);
  if (e != cudaErrorNotSupported) return from_cuda(e);
  // More than 128 rows: one kernel, quantiser warps beside the CTA-pair GEMM.
  e = launch_linear_pair(x, (int)mode, &kc, xq, xsf, reinterpret_cast<uint32_t*>(base + w.g_off),
                         wq, wsf, M, N, K, y, static_cast<int*>(ws), s);
  if (e != cudaErrorNotSupported) return from_cuda(e);
  e = launch_rotate_quantize(x, false, M, K, K, (int)mode, &kc, xq, xsf, static_cast<int*>(ws), s);
  if (e != cudaSuccess) return MXFP4_ERR_CUDA;
  // The kernel just before the GEMM is the quantiser above, which does not write W.
  return from_cuda(launch_gemm(xq, xsf, wq, wsf, M, N, K, y, Epilogue{}, N, static_cast<int*>(ws),
                               workspace_scratch(base, w.g_off, ws_bytes), true, s));
}

int mxfp4_linear_kernel_count(int64_t M, int64_t N, int64_t K, mxfp4_rotation mode) {
  if (!mode_ok(mode)) return -1;
  if (!shape_ok(M, K) || K % rotation_span(mode) != 0 || N < 16 || N % 16 != 0 ||
      !within_limits(M, K) || !within_limits(N, K))
    return -1;
  if (M == 0) return 0;
  return linear_smallm_fits(M, N, K, (int)mode) || linear_pair_fits(M, N, K, (int)mode) ? 1 : 2;
}

int mxfp4_norm_linear_kernel_count(int64_t M, int64_t N, int64_t K, mxfp4_rotation mode) {
  if (mode != MXFP4_ROT_NONE && mode != MXFP4_ROT_HADAMARD32 && mode != MXFP4_ROT_KRON_4x8)
    return -1;
  if (!shape_ok(M, K) || N < 16 || N % 16 != 0 || !within_limits(M, K) || !within_limits(N, K))
    return -1;
  if (M == 0) return 0;
  return norm_one_pass(K) ? 2 : 3;
}

mxfp4_status mxfp4_norm_rotate_quantize(const void* x, int64_t rows, int64_t K, int64_t ldx,
                                        mxfp4_norm kind, float eps, const float* g,
                                        const float* b, mxfp4_rotation mode, const float* kron_a,
                                        const float* kron_b, uint8_t* q, uint8_t* sf,
                                        float* stats, mxfp4_stream_t stream) {
  mxfp4_status st = validate_quantize(x, MXFP4_DT_BF16, rows, K, ldx, q, sf);
  if (st != MXFP4_OK) return st;
  if (!stats) return MXFP4_ERR_INVALID_ARG;
  if (kind != MXFP4_NORM_LAYER && kind != MXFP4_NORM_RMS) return MXFP4_ERR_UNSUPPORTED;
  if (mode != MXFP4_ROT_NONE && mode != MXFP4_ROT_HADAMARD32 && mode != MXFP4_ROT_KRON_4x8)
    return MXFP4_ERR_UNSUPPORTED;
  if (!(eps >= 0.0f)) return MXFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(stats) & 7u) || (g && !aligned16(g)) || (b && !aligned16(b)))
    return MXFP4_ERR_ALIGN;
  KronCoeffs kc{};
  if (mode == MXFP4_ROT_KRON_4x8 && !kron_from_host(kron_a, kron_b, &kc))
    return MXFP4_ERR_INVALID_ARG;
  if (rows == 0) return MXFP4_OK;
  return from_cuda(launch_norm_rotate_quantize(x, rows, K, ldx, (int)kind, eps, g, b, (int)mode,
                                               &kc, q, sf, stats, nullptr,
                                               static_cast<cudaStream_t>(stream)));
}

mxfp4_status mxfp4_norm_linear(const void* x, int64_t M, int64_t K, mxfp4_norm kind, float eps,
                               const float* g, const float* b, mxfp4_rotation mode,
                               const float* kron_a, const float* kron_b, const uint8_t* wq,
                               const uint8_t* wsf, int64_t N, void* y, void* ws,
                               size_t ws_bytes, mxfp4_stream_t stream) {
  if (!rows_ptr_ok(x, M) || !wq || !wsf || !rows_ptr_ok(y, M) || !ws)
    return MXFP4_ERR_INVALID_ARG;
  if (kind != MXFP4_NORM_LAYER && kind != MXFP4_NORM_RMS) return MXFP4_ERR_UNSUPPORTED;
  if (mode != MXFP4_ROT_NONE && mode != MXFP4_ROT_HADAMARD32 && mode != MXFP4_ROT_KRON_4x8)
    return MXFP4_ERR_UNSUPPORTED;
  if (!(eps >= 0.0f)) return MXFP4_ERR_INVALID_ARG;
  if (!shape_ok(M, K) || N < 16 || N % 16 != 0 || !within_limits(M, K) || !within_limits(N, K))
    return MXFP4_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(wq) || !aligned16(wsf) || !aligned16(y) || !aligned16(ws) ||
      (g && !aligned16(g)) || (b && !aligned16(b)) || (K * 2) % 16 != 0 || (N * 2) % 16 != 0)
    return MXFP4_ERR_ALIGN;
  const NormWorkspace w = norm_linear_workspace(M, N, K);
  if (ws_bytes < w.total) return MXFP4_ERR_WORKSPACE;
  KronCoeffs kc{};
  if (mode == MXFP4_ROT_KRON_4x8 && !kron_from_host(kron_a, kron_b, &kc))
    return MXFP4_ERR_INVALID_ARG;
  if (M == 0) return MXFP4_OK;
  uint8_t* base = static_cast<uint8_t*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_norm_rotate_quantize(
      x, M, K, K, (int)kind, eps, g, b, (int)mode, &kc, base + w.q_off, base + w.sf_off,
      reinterpret_cast<float*>(base + w.st_off), static_cast<int*>(ws), s);
  if (e != cudaSuccess) return MXFP4_ERR_CUDA;
  // The kernel just before the GEMM is the quantiser above, which does not write W.
  return from_cuda(launch_gemm(base + w.q_off, base + w.sf_off, wq, wsf, M, N, K, y, Epilogue{},
                               N, static_cast<int*>(ws), workspace_scratch(base, w.g_off, ws_bytes),
                               true, s));
}

size_t mxfp4_nvfp4_sf_bytes(int64_t rows, int64_t K) {
  if (!shape_ok(rows, K)) return 0;
  return mxfp4_sf_bytes(rows, 2 * K);  // atoms of 4 scales per 128 rows, 16-element groups
}

mxfp4_status mxfp4_nvfp4_tensor_scale(const void* x, mxfp4_dtype xdt, int64_t rows, int64_t K,
                                      int64_t ldx, mxfp4_rotation mode, float* scale2,
                                      mxfp4_stream_t stream) {
  if (!rows_ptr_ok(x, rows) || !scale2) return MXFP4_ERR_INVALID_ARG;
  if (xdt != MXFP4_DT_BF16 && xdt != MXFP4_DT_F32) return MXFP4_ERR_UNSUPPORTED;
  if (mode != MXFP4_ROT_NONE && mode != MXFP4_ROT_HADAMARD32) return MXFP4_ERR_UNSUPPORTED;
  if (!shape_ok(rows, K) || ldx < K || !within_limits(rows, K)) return MXFP4_ERR_SHAPE;
  const int64_t esize = xdt == MXFP4_DT_F32 ? 4 : 2;
  if (!aligned16(x) || (ldx * esize) % 16 != 0 || (reinterpret_cast<uintptr_t>(scale2) & 7u))
    return MXFP4_ERR_ALIGN;
  return from_cuda(launch_nvfp4_tensor_scale(x, xdt == MXFP4_DT_F32, rows, K, ldx, (int)mode,
                                             scale2, static_cast<cudaStream_t>(stream)));
}

mxfp4_status mxfp4_nvfp4_quantize(const void* x, mxfp4_dtype xdt, int64_t rows, int64_t K,
                                  int64_t ldx, mxfp4_rotation mode, const float* tensor_scale,
                                  uint8_t* q, uint8_t* sf, mxfp4_stream_t stream) {
  mxfp4_status st = validate_quantize(x, xdt, rows, K, ldx, q, sf);
  if (st != MXFP4_OK) return st;
  if (!tensor_scale) return MXFP4_ERR_INVALID_ARG;
  if (mode != MXFP4_ROT_NONE && mode != MXFP4_ROT_HADAMARD32) return MXFP4_ERR_UNSUPPORTED;
  if (!within_limits(rows, 2 * K)) return MXFP4_ERR_SHAPE;
  if (rows == 0) return MXFP4_OK;
  return from_cuda(launch_nvfp4_quantize(x, xdt == MXFP4_DT_F32, rows, K, ldx, (int)mode,
                                         tensor_scale, q, sf, nullptr,
                                         static_cast<cudaStream_t>(stream)));
}

mxfp4_status mxfp4_nvfp4_gemm(const uint8_t* aq, const uint8_t* asf, const float* a_scale,
                              const uint8_t* bq, const uint8_t* bsf, const float* b_scale,
                              int64_t M, int64_t N, int64_t K, void* y, mxfp4_dtype ydt,
                              int64_t ldy, void* ws, size_t ws_bytes, mxfp4_stream_t stream) {
  mxfp4_status st = validate_gemm(aq, asf, bq, bsf, M, N, K, y, ydt, ldy);
  if (st != MXFP4_OK) return st;
  if (!ws || !a_scale || !b_scale) return MXFP4_ERR_INVALID_ARG;
  if (!within_limits(M, 2 * K) || !within_limits(N, 2 * K)) return MXFP4_ERR_SHAPE;
  if (!aligned16(ws) || (reinterpret_cast<uintptr_t>(a_scale) & 3u) ||
      (reinterpret_cast<uintptr_t>(b_scale) & 3u))
    return MXFP4_ERR_ALIGN;
  if (ws_bytes < kHeadBytes) return MXFP4_ERR_WORKSPACE;  // scratch: optional, see header
  if (M == 0) return MXFP4_OK;
  Epilogue ep;
  ep.out = ydt == MXFP4_DT_F32 ? kOutF32 : kOutBf16;
  ep.nvfp4 = true;
  ep.a_scale = a_scale;
  ep.b_scale = b_scale;
  return from_cuda(launch_gemm(aq, asf, bq, bsf, M, N, K, y, ep, ldy, static_cast<int*>(ws),
                               gemm_workspace_scratch(ws, ws_bytes), false,
                               static_cast<cudaStream_t>(stream)));
}

mxfp4_status mxfp4_nvfp4_linear_static(const void* x, int64_t M, int64_t K,
                                       mxfp4_rotation mode, const float* x_scale,
                                       const uint8_t* wq, const uint8_t* wsf,
                                       const float* w_scale, int64_t N, void* y, void* ws,
                                       size_t ws_bytes, mxfp4_stream_t stream) {
  if (!x_scale) return MXFP4_ERR_INVALID_ARG;
  const mxfp4_status vs = validate_nvfp4_linear(x, M, K, mode, wq, wsf, w_scale, N, y, ws,
                                                ws_bytes);
  if (vs != MXFP4_OK) return vs;
  if (reinterpret_cast<uintptr_t>(x_scale) & 3u) return MXFP4_ERR_ALIGN;
  if (M == 0) return MXFP4_OK;
  const LinearLayout w = linear_layout(M, N, K, 2 * K);
  uint8_t* base = static_cast<uint8_t*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_nvfp4_quantize(x, false, M, K, K, (int)mode, x_scale, base + w.q_off,
                                        base + w.sf_off, static_cast<int*>(ws), s);
  if (e != cudaSuccess) return MXFP4_ERR_CUDA;
  Epilogue ep;
  ep.nvfp4 = true;
  ep.a_scale = x_scale;
  ep.b_scale = w_scale;
  // The kernel just before the GEMM is the quantiser above, which does not write W.
  return from_cuda(launch_gemm(base + w.q_off, base + w.sf_off, wq, wsf, M, N, K, y, ep, N,
                               static_cast<int*>(ws), workspace_scratch(base, w.g_off, ws_bytes),
                               true, s));
}

mxfp4_status mxfp4_nvfp4_linear(const void* x, int64_t M, int64_t K, mxfp4_rotation mode,
                                const uint8_t* wq, const uint8_t* wsf, const float* w_scale,
                                int64_t N, void* y, void* ws, size_t ws_bytes,
                                mxfp4_stream_t stream) {
  const mxfp4_status vs = validate_nvfp4_linear(x, M, K, mode, wq, wsf, w_scale, N, y, ws,
                                                ws_bytes);
  if (vs != MXFP4_OK) return vs;
  const LinearLayout w = linear_layout(M, N, K, 2 * K);
  if (M == 0) return MXFP4_OK;
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* xs = reinterpret_cast<float*>(base + kScaleOff);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the pass's running maximum and block counter: two words after the scale, zero at
  // allocation and left zero by every pass that completes
  cudaError_t e = launch_nvfp4_tensor_scale(x, false, M, K, K, (int)mode, xs, s,
                                            reinterpret_cast<unsigned int*>(xs + 2));
  if (e != cudaSuccess) return MXFP4_ERR_CUDA;
  e = launch_nvfp4_quantize(x, false, M, K, K, (int)mode, xs, base + w.q_off, base + w.sf_off,
                            static_cast<int*>(ws), s);
  if (e != cudaSuccess) return MXFP4_ERR_CUDA;
  Epilogue ep;
  ep.nvfp4 = true;
  ep.a_scale = xs;
  ep.b_scale = w_scale;
  // The kernel just before the GEMM is the quantiser above, which does not write W.
  return from_cuda(launch_gemm(base + w.q_off, base + w.sf_off, wq, wsf, M, N, K, y, ep, N,
                               static_cast<int*>(ws), workspace_scratch(base, w.g_off, ws_bytes),
                               true, s));
}

mxfp4_status mxfp4_kron_weight_factors(const float* A, const float* B, float* At_inv,
                                       float* Bt_inv) {
  if (!A || !B || !At_inv || !Bt_inv) return MXFP4_ERR_INVALID_ARG;
  double ai[16], bi[64];
  if (!invert_small(A, 4, ai) || !invert_small(B, 8, bi)) return MXFP4_ERR_INVALID_ARG;
  // (A^-1)^T and (B^-1)^T, each entry rounded once to fp32
  for (int r = 0; r < 4; ++r)
    for (int c = 0; c < 4; ++c) At_inv[r * 4 + c] = (float)ai[c * 4 + r];
  for (int r = 0; r < 8; ++r)
    for (int c = 0; c < 8; ++c) Bt_inv[r * 8 + c] = (float)bi[c * 8 + r];
  return MXFP4_OK;
}

mxfp4_status mxfp4_set_linear_form(int form) {
  if (form != MXFP4_LINEAR_AUTO && form != MXFP4_LINEAR_ONE_KERNEL &&
      form != MXFP4_LINEAR_TWO_KERNELS)
    return MXFP4_ERR_UNSUPPORTED;
  g_linear_form.store(form);
  return MXFP4_OK;
}

mxfp4_status mxfp4_test_set_fault(int fault) {
  if (fault != MXFP4_TEST_FAULT_NONE && fault != MXFP4_TEST_FAULT_WITHHOLD_ACCUMULATOR)
    return MXFP4_ERR_UNSUPPORTED;
  g_test_fault.store(fault);
  return MXFP4_OK;
}

mxfp4_status mxfp4_poll_status(void* ws, mxfp4_status* out) {
  if (!ws || !out) return MXFP4_ERR_INVALID_ARG;
  int v = 0;
  if (cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MXFP4_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(ws, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return MXFP4_ERR_CUDA;
  *out = static_cast<mxfp4_status>(v);
  return MXFP4_OK;
}

}  // extern "C"
