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
// problem: 256 bytes (status region) + round256(M * K / 2) + round256(the scale bytes of
// X), plus 4 bytes per 128 rows and 4 more (the one-kernel form's counters) for more than
// 128 rows, must fit in it.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kScratchBytes = MXFP4_NOALLOC_SCRATCH_BYTES;

// Layout: the layer workspace's (status region | Xq | X scales | GEMM data or the
// one-launch layer's row counters = the rest of the array), parts 256-byte aligned. Each
// call clears the status region before its first launch, and the row counters before the
// launch that uses them, so nothing an earlier call left there reaches it; the other parts
// are written before they are read.
static __device__ __align__(256) unsigned char g_linear_scratch[kScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_addr[64] = {};  // device address of g_linear_scratch, per device

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

}  // namespace

extern "C" mxfp4_status mxfp4_linear_noalloc(const void* x, int64_t M, int64_t K,
                                              mxfp4_rotation mode, const float* kron_a,
                                              const float* kron_b, const uint8_t* wq,
                                              const uint8_t* wsf, int64_t N, void* y, int* status,
                                              mxfp4_stream_t stream) {
  using namespace mxfp4;
  KronCoeffs kc{};
  const mxfp4_status vs = validate_linear(x, M, K, mode, kron_a, kron_b, wq, wsf, N, y, &kc);
  if (vs != MXFP4_OK) return vs;
  if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return MXFP4_ERR_ALIGN;
  const LinearLayout w = linear_layout(M, N, K, K);
  if (w.g_off + linear_row_counter_bytes(M) > kScratchBytes)
    return MXFP4_ERR_WORKSPACE;  // beyond the fixed capacity
  if (M == 0) return MXFP4_OK;

  unsigned char* scratch = nullptr;
  mxfp4_status st = scratch_on_current_device(&scratch);
  if (st != MXFP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The status word (used when the caller passes none) starts at zero.
  if (cudaMemsetAsync(scratch, 0, kHeadBytes, s) != cudaSuccess) return MXFP4_ERR_CUDA;
  int* status_word = status ? status : reinterpret_cast<int*>(scratch);
  uint8_t* xq = scratch + w.q_off;
  uint8_t* xsf = scratch + w.sf_off;
  // 1..8 rows: one kernel quantises x inside the GEMM's CTAs.
  const cudaError_t fe = launch_linear_smallm(x, K, (int)mode, &kc, wq, wsf, M, N, K, y, N,
                                              status_word, s);
  if (fe != cudaErrorNotSupported) return fe == cudaSuccess ? MXFP4_OK : MXFP4_ERR_CUDA;
  // More than 128 rows: one kernel, quantiser warps beside the CTA-pair GEMM; its row
  // counters follow the scales.
  const cudaError_t pe =
      launch_linear_pair(x, (int)mode, &kc, xq, xsf, reinterpret_cast<uint32_t*>(scratch + w.g_off),
                         wq, wsf, M, N, K, y, status_word, s);
  if (pe != cudaErrorNotSupported) return pe == cudaSuccess ? MXFP4_OK : MXFP4_ERR_CUDA;
  if (launch_rotate_quantize(x, false, M, K, K, (int)mode, &kc, xq, xsf, status_word, s) !=
      cudaSuccess)
    return MXFP4_ERR_CUDA;
  // The kernel just before the GEMM is the quantiser above, which does not write W.
  // GEMM data: what is left of the array (the GEMM splits no tile if it is too small).
  if (launch_gemm(xq, xsf, wq, wsf, M, N, K, y, Epilogue{}, N, status_word,
                  workspace_scratch(scratch, w.g_off, kScratchBytes), true, s) != cudaSuccess)
    return MXFP4_ERR_CUDA;
  return MXFP4_OK;
}
