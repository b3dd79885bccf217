// noalloc.cu -- mxfp4_linear_noalloc: the whole layer with its scratch in a
// fixed, library-owned device array instead of a caller-provided workspace.
//
// Who needs this: code that may not allocate device memory when it runs the
// layer. Examples are an inference engine whose memory plan is fixed at
// start-up, a plugin executing inside another framework's enqueue callback
// where allocation is forbidden, or latency-critical code that cannot afford
// cudaMalloc's implicit device synchronisation. Those callers still own and
// pass their inputs and outputs; only the intermediate quantised activations
// (and the status word) move into the array below.
//
// The array is a file-scope __device__ variable, so every GPU that loads this
// part of the library holds it until the process exits. Its size caps the
// problem: M * K / 2 + the scale bytes of X + 256 must fit in it.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/mxfp4.h"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = MXFP4_NOALLOC_SCRATCH_BYTES;
constexpr size_t kStatusBytes = 256;

// Layout: [status word region (256 B) | Xq (M x K/2) | X scales | GEMM scratch (the rest)],
// parts 256-byte aligned. The array starts zeroed; the GEMM leaves its scratch counters
// zeroed after every call that completes.
static __device__ __align__(256) unsigned char g_linear_scratch[kScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_addr[64] = {};  // device address of g_linear_scratch, per device

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// In host code `g_linear_scratch` names a host-side shadow, not device memory:
// the device address has to be looked up once per device, with that device
// current, and only that address may be handed to a kernel.
mxfp4_status scratch_on_current_device(unsigned char** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MXFP4_ERR_CUDA;
  if (dev < 0 || dev >= 64) return MXFP4_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_linear_scratch) != cudaSuccess || p == nullptr)
      return MXFP4_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_scratch_addr[dev]);
  return MXFP4_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" mxfp4_status mxfp4_linear_noalloc(const void* x, int64_t M, int64_t K,
                                              mxfp4_rotation mode, const float* kron_a,
                                              const float* kron_b, const uint8_t* wq,
                                              const uint8_t* wsf, int64_t N, void* y, int* status,
                                              mxfp4_stream_t stream) {
  using namespace mxfp4;
  if ((!x && M != 0) || !wq || !wsf || (!y && M != 0)) return MXFP4_ERR_INVALID_ARG;
  if (mode < MXFP4_ROT_NONE || mode > MXFP4_ROT_HADAMARD128) return MXFP4_ERR_UNSUPPORTED;
  if (M < 0 || K < 32 || K % rotation_span(mode) != 0 || N < 16 || N % 16 != 0 ||
      M >= (1ll << 31) ||
      K >= (1ll << 31) || N >= (1ll << 31))
    return MXFP4_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(wq) || !aligned16(wsf) || !aligned16(y) ||
      (status && (reinterpret_cast<uintptr_t>(status) & 3u)))
    return MXFP4_ERR_ALIGN;
  KronCoeffs kc{};
  if (mode == MXFP4_ROT_KRON_4x8) {
    if (!kron_a || !kron_b) return MXFP4_ERR_INVALID_ARG;
    for (int i = 0; i < 16; ++i) kc.a[i] = kron_a[i];
    for (int i = 0; i < 64; ++i) kc.b[i] = kron_b[i];
    kron_derive(&kc);
  }
  const size_t q_off = kStatusBytes;
  const size_t sf_off = round_up(q_off + (size_t)M * (size_t)(K / 2), 256);
  const size_t need = round_up(sf_off + mxfp4_sf_bytes(M, K), 256);
  if (need > kScratchBytes) return MXFP4_ERR_WORKSPACE;  // beyond the fixed scratch capacity
  if (M == 0) return MXFP4_OK;

  unsigned char* scratch = nullptr;
  mxfp4_status st = scratch_on_current_device(&scratch);
  if (st != MXFP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status_word = status;
  if (!status_word) {
    // No caller status word: keep one in the scratch and clear the previous call's value.
    status_word = reinterpret_cast<int*>(scratch);
    if (cudaMemsetAsync(status_word, 0, sizeof(int), s) != cudaSuccess) return MXFP4_ERR_CUDA;
  }
  uint8_t* xq = scratch + q_off;
  uint8_t* xsf = scratch + sf_off;
  // Up to 16 rows: one kernel quantises x inside the GEMM's CTAs.
  const cudaError_t fe = launch_linear_smallm(x, K, (int)mode, &kc, wq, wsf, M, N, K, y, N,
                                              status_word, s);
  if (fe != cudaErrorNotSupported) return fe == cudaSuccess ? MXFP4_OK : MXFP4_ERR_CUDA;
  if (launch_rotate_quantize(x, false, M, K, K, (int)mode, &kc, xq, xsf, status_word, s) !=
      cudaSuccess)
    return MXFP4_ERR_CUDA;
  // The kernel just before the GEMM is the quantiser above, which does not write W.
  // GEMM scratch: what is left of the array (the GEMM splits no tile if it is too small).
  if (launch_gemm(xq, xsf, wq, wsf, M, N, K, y, Epilogue{}, N, status_word, scratch + need,
                  kScratchBytes - need, true, s) != cudaSuccess)
    return MXFP4_ERR_CUDA;
  return MXFP4_OK;
}
