/*
 * mxfp4.h -- C ABI of libmxfp4, the MXFP4 W4A4 linear block for NVIDIA B200 (sm_100a).
 *
 * The layer computes Y = X . W^T in three steps:
 *   1. an online block-local rotation of every 32-element block of X
 *      (normalised 32x32 Sylvester Hadamard, "Bridging the Gap Between Promise
 *      and Performance for Microscaling FP4 Quantization", "Methodologie:
 *      MR-GPTQ" item 1 and "GPU Kernel Ondersteuning (QuTLASS)"; or a learned
 *      Kronecker-factored A (x) B transform, "KroQuant: Effiziente Post-
 *      Training-Quantisierung fuer Diffusion Transformers mittels Kronecker-
 *      Produkt-Struktur", "Tiefenanalyse");
 *   2. MXFP4 quantisation: one E8M0 power-of-two scale per 32-element block
 *      and 4-bit E2M1 elements ("AMD Quark delivers MXFP4 quantization for
 *      FLUX.1-dev on Instinct MI350 with 1.92x speedup", "What is MXFP4 and
 *      why does it eliminate dequantization overhead?"; "Bridging the Gap...",
 *      "Probleemstelling" item 2);
 *   3. a block-scaled FP4 x FP4 GEMM against pre-quantised MXFP4 weights with
 *      fp32 accumulation and bf16 (or fp32) output, with no dequantisation to
 *      bf16 in between (AMD Quark page, opening section).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All pointers named x, q, sf, aq, asf, bq, bsf, wq, wsf, y, ws are DEVICE
 *    pointers owned by the caller; the library keeps no reference after the
 *    call returns and allocates no device memory. kron_a / kron_b are HOST
 *    pointers (the transform is passed by value to the kernel).
 *  - Every launch is asynchronous and ordered on `stream` (a cudaStream_t;
 *    NULL = the legacy default stream). Kernels are launched with programmatic
 *    dependent launch: one may be scheduled while the kernel before it on the
 *    stream finishes, and waits for that kernel to complete before it touches
 *    any memory the two could share. The results are those of plain stream
 *    order.
 *  - Argument errors are detected on the host before any launch and launch
 *    nothing: NULL pointer -> MXFP4_ERR_INVALID_ARG; bad sizes ->
 *    MXFP4_ERR_SHAPE; misaligned pointer or row stride -> MXFP4_ERR_ALIGN;
 *    workspace too small -> MXFP4_ERR_WORKSPACE; unknown mode / dtype ->
 *    MXFP4_ERR_UNSUPPORTED. A failed launch returns MXFP4_ERR_CUDA.
 *    rows == 0 (or M == 0) is a valid empty call: nothing is launched (the
 *    NVFP4 tensor-scale pass still writes its scale), and the pointers to
 *    row operands (x, the activation codes and scales, y) may then be NULL.
 *  - Packed E2M1 codes ("q" operands): row-major [rows, K/2] bytes; byte j of a
 *    row holds element 2j in bits 0-3 and element 2j+1 in bits 4-7; bit 3 of a
 *    code is the sign, codes 0..7 are 0, 0.5, 1, 1.5, 2, 3, 4, 6.
 *  - E8M0 scale bytes ("sf" operands), byte b meaning 2^(b-127), 0xFF = NaN,
 *    are stored in the tensor-core scale layout: rows are tiled by 128 and
 *    32-element blocks by 4 into 512-byte atoms, atoms ordered block-group
 *    fastest then row tile, and inside an atom (row r, block kb) sits at byte
 *    (r % 32) * 16 + ((r / 32) % 4) * 4 + kb % 4. The buffer holds
 *    mxfp4_sf_bytes(rows, K) bytes; padding rows/blocks are written as 0 by the
 *    quantisers and must be 0 (or any finite scale) in caller-made buffers.
 *  - Scale rule: e = floor(log2(amax)) - 2 clamped to [-127, 127] (byte
 *    e + 127) where amax is the block's largest magnitude after rotation;
 *    elements are round(y * 2^-e) to the nearest E2M1 value, ties to even,
 *    saturating at +-6; the sign is kept (code 8 for negatives rounding to 0).
 *    An all-zero block gets byte 0; a block with a non-finite value after
 *    rotation gets byte 0xFF and all-zero codes.
 */
#ifndef MXFP4_H_
#define MXFP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MXFP4_OK = 0,
  MXFP4_ERR_INVALID_ARG = 1,
  MXFP4_ERR_SHAPE = 2,
  MXFP4_ERR_ALIGN = 3,
  MXFP4_ERR_WORKSPACE = 4,
  MXFP4_ERR_UNSUPPORTED = 5,
  MXFP4_ERR_CUDA = 6,
  MXFP4_ERR_TIMEOUT = 7
} mxfp4_status;

typedef enum {
  MXFP4_ROT_NONE = 0,       /* plain MXFP4 quantisation */
  MXFP4_ROT_HADAMARD32 = 1, /* y = H32 x, H32 = H2^(x5) / sqrt(32) (Sylvester order) */
  MXFP4_ROT_KRON_4x8 = 2,   /* y = (A (x) B) x, A 4x4, B 8x8 */
  MXFP4_ROT_HADAMARD64 = 3, /* y = H64 x over 64-element groups (2 blocks), K % 64 == 0 */
  MXFP4_ROT_HADAMARD128 = 4 /* y = H128 x over 128-element groups (4 blocks), K % 128 == 0 */
} mxfp4_rotation;

typedef enum { MXFP4_DT_BF16 = 0, MXFP4_DT_F32 = 1 } mxfp4_dtype;

typedef enum {
  MXFP4_OP_QUANTIZE = 0,
  MXFP4_OP_GEMM = 1, /* also mxfp4_gemm_bias, mxfp4_gemm_quantize, mxfp4_nvfp4_gemm */
  MXFP4_OP_LINEAR = 2,
  MXFP4_OP_NVFP4_LINEAR = 3,
  MXFP4_OP_NORM_LINEAR = 4
} mxfp4_op;

typedef enum { MXFP4_NORM_LAYER = 0, MXFP4_NORM_RMS = 1 } mxfp4_norm;

/* A cudaStream_t, passed as an opaque handle so this header needs no CUDA headers. */
typedef void* mxfp4_stream_t;

/* Bytes of the scale-factor buffer for a [rows, K] operand:
 * ceil(rows / 128) * 128 * ceil(K / 128) * 4. K % 32 == 0. Returns 0 on bad sizes. */
size_t mxfp4_sf_bytes(int64_t rows, int64_t K);

/* Byte offset of the scale of (row, 32-element block kblock) in that buffer, or -1 if out of range. */
int64_t mxfp4_sf_offset(int64_t row, int64_t kblock, int64_t K);

/* Device workspace that `op` needs for this problem (0 if none). Every
 * workspace starts with the same 256-byte status region (the status word at
 * byte 0), so one workspace can serve calls of different sizes. After it come,
 * for the layer ops, the quantised activations (and the NORM_LINEAR row
 * statistics), then, for 33..128 activation rows, the few-row GEMM's K-split
 * partials (sized for a 148-SM B200), or, for MXFP4_OP_LINEAR with more than
 * 128 rows, one 4-byte row counter per 128 rows and a 4-byte work-item counter
 * (the one-kernel layer's; each call clears them itself). Allocate it zeroed; every other part is written
 * before it is read. With a smaller partial area than this size the few-row
 * GEMM sums its K splits on chip instead (slower, the same bits). */
size_t mxfp4_workspace_bytes(int op, int64_t M, int64_t N, int64_t K);

/* Static description of a status code. Never NULL. */
const char* mxfp4_status_string(mxfp4_status status);

/*
 * Quantise x[rows, K] (leading dimension ldx elements, bf16 or fp32) to MXFP4
 * with no rotation: q = packed codes [rows, K/2], sf = scale bytes in the
 * tensor-core layout (mxfp4_sf_bytes(rows, K) bytes, padding written as 0).
 * Steps 2 of the layer ("What is MXFP4..." on the AMD Quark page; RTN
 * quantiser of "Bridging the Gap...", "Probleemstelling").
 * Requirements: K % 32 == 0, ldx >= K, x 16-byte aligned and ldx * elemsize a
 * multiple of 16; q and sf 16-byte aligned. The kernel's input pipeline waits
 * on its own copies with a time bound; these two calls have no status word, so
 * an expiry (a copy that never lands) only ends the kernel early, leaving the
 * output incomplete -- mxfp4_linear reports it through its workspace.
 */
mxfp4_status mxfp4_quantize(const void* x, mxfp4_dtype xdt, int64_t rows, int64_t K, int64_t ldx,
                            uint8_t* q, uint8_t* sf, mxfp4_stream_t stream);

/*
 * Rotate each 32-element block of x in fp32 (mode), then quantise as
 * mxfp4_quantize. Hadamard: a five-stage butterfly (strides 1, 2, 4, 8, 16;
 * (a, b) -> (a + b, a - b)) then one multiply by the fp32 value nearest
 * 1/sqrt(32) ("Bridging the Gap...", "Methodologie: MR-GPTQ" item 1).
 * Kronecker: z[8j+k] = sum_l B[k][l] x[8j+l], y[8i+k] = sum_j A[i][j] z[8j+k],
 * each sum in fp32 as the first product followed by fma steps in ascending
 * index order ("KroQuant...",
 * "Tiefenanalyse"). kron_a (16 floats) and kron_b (64 floats) are HOST
 * pointers, row-major, read during the call; NULL for the other modes. To
 * prepare weights for the Kronecker mode pass A^-T and B^-T here
 * (T^-T = A^-T (x) B^-T, "KroQuant...", "Hintergrund": the inverse goes on
 * the weights).
 * Larger Hadamard blocks (modes HADAMARD64 / HADAMARD128; "KroQuant...",
 * "Hintergrund", on the cost of larger Hadamard blocks): each 64- or
 * 128-element group of a row is rotated by the butterfly with strides 1, 2,
 * ..., n/2 and one multiply by the fp32 nearest 1/sqrt(n) (1/8, and half of
 * the 1/sqrt(32) constant); the scales stay per 32 elements. K must be a
 * multiple of the group; weights take the same mode (H_n is symmetric and
 * orthonormal). These two modes have no bounded waits.
 */
mxfp4_status mxfp4_rotate_quantize(const void* x, mxfp4_dtype xdt, int64_t rows, int64_t K,
                                   int64_t ldx, mxfp4_rotation mode, const float* kron_a,
                                   const float* kron_b, uint8_t* q, uint8_t* sf,
                                   mxfp4_stream_t stream);

/*
 * Block-scaled GEMM on the tcgen05 tensor cores (kind::mxf4):
 * y[m][n] = sum_b 2^(asf[m,b] + bsf[n,b] - 254) * sum_{i in b} v(aq[m,i]) v(bq[n,i]),
 * accumulated in fp32, written as bf16 (round to nearest even) or fp32.
 * aq/asf: [M, K] operand (activations), bq/bsf: [N, K] operand (weights),
 * both in the formats above. y: row-major [M, N] with leading dimension ldy
 * elements. Requirements: K % 32 == 0, N % 16 == 0, ldy >= N, y 16-byte aligned
 * and ldy * elemsize a multiple of 16; aq, bq, asf, bsf 16-byte aligned.
 * ws: at least 256 bytes, zeroed when allocated; its first 16 bytes are the
 * device status word (see mxfp4_poll_status). mxfp4_workspace_bytes(
 * MXFP4_OP_GEMM, M, N, K) bytes give the fastest form; with less (too little
 * room for the few-row K-split partials, or a GPU whose SM count needs more)
 * the few-row kernel sums its K splits on chip (slower, the same bits). Fewer
 * than 256 bytes -> MXFP4_ERR_WORKSPACE.
 * ("AMD Quark...", opening section: MXFP4 GEMM with no dequantisation;
 * "Bridging the Gap...", "GPU Kernel Ondersteuning (QuTLASS)".)
 */
mxfp4_status mxfp4_gemm(const uint8_t* aq, const uint8_t* asf, const uint8_t* bq,
                        const uint8_t* bsf, int64_t M, int64_t N, int64_t K, void* y,
                        mxfp4_dtype ydt, int64_t ldy, void* ws, size_t ws_bytes,
                        mxfp4_stream_t stream);

/*
 * Offline weight preparation for the Kronecker mode ("KroQuant...",
 * "Hintergrund": the transform is invertible and its inverse goes on the
 * weights). With activations rotated by T = A (x) B, weights are rotated by
 * T^-T = A^-T (x) B^-T so that (T x) . (T^-T w) = x . w. This computes
 * At_inv = (A^-1)^T (4x4) and Bt_inv = (B^-1)^T (8x8), all row-major HOST
 * float arrays: each inverse by Gauss-Jordan elimination with partial pivoting
 * in double, then every entry rounded once to fp32. Pass them as kron_a /
 * kron_b of mxfp4_rotate_quantize on the fp32 weights. Host only, no GPU.
 * NULL pointer, or a singular or non-finite factor -> MXFP4_ERR_INVALID_ARG.
 */
mxfp4_status mxfp4_kron_weight_factors(const float* A, const float* B, float* At_inv,
                                       float* Bt_inv);

/*
 * mxfp4_gemm with a bias: y[m][n] = (fp32 accumulator) + bias[n], one fp32
 * rounding, then the output conversion. bias: DEVICE fp32 [N], 16-byte
 * aligned, not NULL. Everything else as mxfp4_gemm. (The bias of the step
 * after the contraction: "AMD Quark delivers MXFP4 quantization for FLUX.1-dev
 * on Instinct MI350 with 1.92x speedup", opening section; no formula given.)
 */
mxfp4_status mxfp4_gemm_bias(const uint8_t* aq, const uint8_t* asf, const uint8_t* bq,
                             const uint8_t* bsf, int64_t M, int64_t N, int64_t K,
                             const float* bias, void* y, mxfp4_dtype ydt, int64_t ldy, void* ws,
                             size_t ws_bytes, mxfp4_stream_t stream);

/*
 * mxfp4_gemm whose output is the next layer's MXFP4 activation operand, so no
 * bf16 copy of Y is written or read between layers ("AMD Quark...", opening
 * section and "What is MXFP4 and why does it eliminate dequantization
 * overhead?"): v = (fp32 accumulator) + bias[n] (bias may be NULL), then each
 * 32-column block of every row is rotated like an activation block (mode,
 * with kron_a / kron_b as in mxfp4_rotate_quantize) and quantised with the
 * scale rule and rounding of mxfp4_rotate_quantize, from those fp32 values.
 * yq: packed codes [M, N/2] (row stride N/2 bytes); ysf: mxfp4_sf_bytes(M, N)
 * bytes in the tensor-core layout of an [M, N] operand (padding written 0).
 * Requirements: N % 32 == 0, yq / ysf / bias 16-byte aligned; workspace as
 * mxfp4_gemm. yq / ysf can be passed as aq / asf of the next mxfp4_gemm*.
 */
mxfp4_status mxfp4_gemm_quantize(const uint8_t* aq, const uint8_t* asf, const uint8_t* bq,
                                 const uint8_t* bsf, int64_t M, int64_t N, int64_t K,
                                 const float* bias, mxfp4_rotation mode, const float* kron_a,
                                 const float* kron_b, uint8_t* yq, uint8_t* ysf, void* ws,
                                 size_t ws_bytes, mxfp4_stream_t stream);

/*
 * The whole layer: rotate + quantise x (bf16 [M, K], row stride K) into the
 * workspace, then the block-scaled GEMM with the pre-quantised weights
 * (wq/wsf: [N, K] operand prepared offline with the matching rotation), bf16
 * output y[M, N] (row stride N). ws must hold
 * mxfp4_workspace_bytes(MXFP4_OP_LINEAR, M, N, K) bytes. The two kernels run
 * back to back on `stream`; the GEMM may start loading wq / wsf while the
 * quantiser is still running, so wq / wsf must not overlap the workspace.
 * Two sizes run the layer as one kernel instead (rotation none, Hadamard-32 or
 * Kronecker; see mxfp4_linear_kernel_count):
 *  - 1..8 rows (K splits of at most 12 x 256 elements): each CTA rotates and
 *    quantises its own K range of x into shared memory while it streams the
 *    weights;
 *  - large problems (more than 128 rows, at least 8 x 74 output tiles of
 *    256 x 256, x at least 40 MiB): the CTA-pair GEMM with six more warps per
 *    CTA that rotate and quantise x into the workspace while the other warps
 *    multiply; each CTA's TMA producer waits, per 128-row group of x, for the
 *    group's rows to be published (a GPU-scope release and a counter in the
 *    workspace, cleared by one cudaMemsetAsync before the launch); the quantiser
 *    warps take their rows from a work-item counter there, so whichever CTAs
 *    are resident do all of the quantisation.
 * Codes, scales and the result are the same in every form.
 */
mxfp4_status mxfp4_linear(const void* x, int64_t M, int64_t K, mxfp4_rotation mode,
                          const float* kron_a, const float* kron_b, const uint8_t* wq,
                          const uint8_t* wsf, int64_t N, void* y, void* ws, size_t ws_bytes,
                          mxfp4_stream_t stream);

/*
 * How many kernels mxfp4_linear (and mxfp4_linear_noalloc) launch for these
 * sizes and rotation: 1 when the layer runs as one kernel (mode none /
 * Hadamard-32 / Kronecker, and either 1..8 rows with at most 12 k-tiles of
 * 256 elements per K split of the few-row GEMM, or the large-problem form
 * above), 2 otherwise (quantiser, then GEMM), 0 for M == 0, -1 for sizes or a
 * mode that mxfp4_linear rejects. Follows mxfp4_set_linear_form. Host only;
 * no GPU is touched.
 */
int mxfp4_linear_kernel_count(int64_t M, int64_t N, int64_t K, mxfp4_rotation mode);

/*
 * Which form mxfp4_linear and mxfp4_linear_noalloc take where they have a
 * choice (more than 128 rows, or 1..8 rows within the one-kernel limits; mode
 * none / Hadamard-32 / Kronecker): MXFP4_LINEAR_AUTO (the state at load time)
 * chooses by size as described above; MXFP4_LINEAR_ONE_KERNEL takes the
 * one-kernel form for every problem of more than 128 rows (and keeps the
 * few-row choice); MXFP4_LINEAR_TWO_KERNELS always quantises and multiplies
 * in two kernels. Every form gives the same codes, scales and result; this is
 * for tests that cover both and for measuring them against each other.
 * Process-wide, read when a call is set up. Unknown values ->
 * MXFP4_ERR_UNSUPPORTED.
 */
typedef enum {
  MXFP4_LINEAR_AUTO = 0,
  MXFP4_LINEAR_ONE_KERNEL = 1,
  MXFP4_LINEAR_TWO_KERNELS = 2
} mxfp4_linear_form;

mxfp4_status mxfp4_set_linear_form(int form);

/*
 * Norm prologue: the normalisation that precedes the layer, applied inside the
 * quantiser instead of as a separate pass that writes a normalised bf16 copy
 * of x ("KroQuant...", "Hintergrund": the norms are why the transform runs
 * online). Per-row statistics go to stats (DEVICE, [rows][2] fp32, 8-byte
 * aligned; also an output): LayerNorm mu = mean, rstd = 1 / sqrt(var + eps);
 * RMSNorm mu = 0, rstd = 1 / sqrt(mean(x^2) + eps) (fp32 sums over the row,
 * in an order the library chooses). Then v = ((x - mu) * rstd) * g[c] + b[c]
 * (fp32, in that order; g / b: DEVICE fp32 [K], 16-byte aligned, NULL for
 * 1 / 0 -- for adaLN modulation pass g = 1 + scale and b = shift) is rotated
 * and quantised. For K <= 51168 one kernel does both from whole rows copied
 * into shared memory (x read once); longer rows take a statistics kernel and
 * then the quantiser. x is bf16; modes NONE / HADAMARD32 / KRON_4x8;
 * otherwise as mxfp4_rotate_quantize.
 */
mxfp4_status mxfp4_norm_rotate_quantize(const void* x, int64_t rows, int64_t K, int64_t ldx,
                                        mxfp4_norm kind, float eps, const float* g,
                                        const float* b, mxfp4_rotation mode, const float* kron_a,
                                        const float* kron_b, uint8_t* q, uint8_t* sf,
                                        float* stats, mxfp4_stream_t stream);

/* The layer with the norm prologue: mxfp4_norm_rotate_quantize into the
 * workspace, then the GEMM as in mxfp4_linear. ws: mxfp4_workspace_bytes(
 * MXFP4_OP_NORM_LINEAR, M, N, K) bytes, zeroed at allocation. */
mxfp4_status mxfp4_norm_linear(const void* x, int64_t M, int64_t K, mxfp4_norm kind, float eps,
                               const float* g, const float* b, mxfp4_rotation mode,
                               const float* kron_a, const float* kron_b, const uint8_t* wq,
                               const uint8_t* wsf, int64_t N, void* y, void* ws,
                               size_t ws_bytes, mxfp4_stream_t stream);

/*
 * How many kernels mxfp4_norm_linear launches for these sizes: 2 when the
 * norm, rotation and quantisation run as one kernel that copies whole rows
 * into shared memory (K <= 51168), then the GEMM; 3 otherwise (row
 * statistics, quantiser, GEMM); 0 for M == 0; -1 for arguments it rejects.
 * mxfp4_norm_rotate_quantize launches one kernel fewer. Host only.
 */
int mxfp4_norm_linear_kernel_count(int64_t M, int64_t N, int64_t K, mxfp4_rotation mode);

/*
 * NVFP4, the other FP4 format the pages compare ("Bridging the Gap Between
 * Promise and Performance for Microscaling FP4 Quantization", "Probleemstelling"
 * item 1: 16-element groups; "Format-specifieke Schaaloptimalisatie": tensor and
 * group scales). Codes are packed E2M1 as above; every 16 elements of a row
 * share an unsigned E4M3 scale byte (bias 7, 3 mantissa bits, largest 448) and
 * the tensor has one fp32 scale st. Quantisation of a group of (rotated)
 * values y: g = amax / (6 st), byte = nearest E4M3 of g (ties to even,
 * saturating), S = E4M3(byte) * st, code_i = nearest E2M1 of y_i * (1 / S),
 * each step one fp32 rounding; st = 0 or S = 0 gives byte and codes 0.
 * Scale bytes use the 512-byte atoms of the MXFP4 layout with 16-element groups
 * in place of 32-element blocks: mxfp4_nvfp4_sf_bytes(rows, K) =
 * mxfp4_sf_bytes(rows, 2 K), byte of (row, group g) at mxfp4_sf_offset(row, g,
 * 2 K). Rotation modes: NONE and HADAMARD32 only. K % 32 == 0.
 */
size_t mxfp4_nvfp4_sf_bytes(int64_t rows, int64_t K);

/* Tensor scale st = amax(rotated x) / (6 * 448) (fp32, one rounding) into
 * scale2[0]; scale2: DEVICE pointer to 2 floats, 8-byte aligned, both
 * overwritten ([1] is scratch). Stream-ordered (a memset and one kernel, whose
 * last block to finish writes the scale). */
mxfp4_status mxfp4_nvfp4_tensor_scale(const void* x, mxfp4_dtype xdt, int64_t rows, int64_t K,
                                      int64_t ldx, mxfp4_rotation mode, float* scale2,
                                      mxfp4_stream_t stream);

/* Rotate (mode) and quantise x to NVFP4 with the DEVICE fp32 tensor scale
 * *tensor_scale: q [rows, K/2], sf mxfp4_nvfp4_sf_bytes(rows, K) bytes (padding
 * 0). Requirements as mxfp4_quantize. Weights: quantise them with their own
 * tensor scale (mxfp4_nvfp4_tensor_scale on W). */
mxfp4_status mxfp4_nvfp4_quantize(const void* x, mxfp4_dtype xdt, int64_t rows, int64_t K,
                                  int64_t ldx, mxfp4_rotation mode, const float* tensor_scale,
                                  uint8_t* q, uint8_t* sf, mxfp4_stream_t stream);

/* NVFP4 GEMM on the tcgen05 tensor cores (kind::mxf4nvf4, 16-element UE4M3
 * block scales): y = (*a_scale) (*b_scale) sum_g E4M3(asf) E4M3(bsf) sum v(a) v(b),
 * fp32 accumulation, the tensor scales applied once in fp32 to the sum.
 * a_scale / b_scale: DEVICE fp32 tensor scales. Everything else as mxfp4_gemm
 * (bf16 or fp32 output; workspace mxfp4_workspace_bytes(MXFP4_OP_GEMM, ...)). */
mxfp4_status mxfp4_nvfp4_gemm(const uint8_t* aq, const uint8_t* asf, const float* a_scale,
                              const uint8_t* bq, const uint8_t* bsf, const float* b_scale,
                              int64_t M, int64_t N, int64_t K, void* y, mxfp4_dtype ydt,
                              int64_t ldy, void* ws, size_t ws_bytes, mxfp4_stream_t stream);

/* The NVFP4 layer: tensor scale of the rotated x, quantise x, GEMM with the
 * pre-quantised weights (wq / wsf / *w_scale, from mxfp4_nvfp4_quantize with the
 * same mode), bf16 y [M, N]: three kernels. ws: mxfp4_workspace_bytes(
 * MXFP4_OP_NVFP4_LINEAR, M, N, K) bytes, zeroed at allocation (status word as
 * for mxfp4_linear; the tensor-scale pass keeps two words of its own there and
 * leaves them zero, so zero the workspace again after a timeout). */
mxfp4_status mxfp4_nvfp4_linear(const void* x, int64_t M, int64_t K, mxfp4_rotation mode,
                                const uint8_t* wq, const uint8_t* wsf, const float* w_scale,
                                int64_t N, void* y, void* ws, size_t ws_bytes,
                                mxfp4_stream_t stream);

/* The NVFP4 layer with a static activation tensor scale (one calibrated offline, for
 * instance): x is quantised with *x_scale (DEVICE fp32, 4-byte aligned; the
 * quantisation rule of mxfp4_nvfp4_quantize with st = *x_scale) instead of a scale
 * taken from x, so the layer is two kernels, the quantiser and the GEMM, and x is read
 * once ("Bridging the Gap...", "Methodologie: MR-GPTQ" item 2: tensor and group
 * scales). Groups whose amax / (6 st) exceeds 448 saturate at group scale 448; st = 0
 * gives zero codes. Everything else as mxfp4_nvfp4_linear; x_scale must not be written
 * by the layer's own workspace. */
mxfp4_status mxfp4_nvfp4_linear_static(const void* x, int64_t M, int64_t K,
                                       mxfp4_rotation mode, const float* x_scale,
                                       const uint8_t* wq, const uint8_t* wsf,
                                       const float* w_scale, int64_t N, void* y, void* ws,
                                       size_t ws_bytes, mxfp4_stream_t stream);

/* Size in bytes of the device scratch array that mxfp4_linear_noalloc uses (per GPU). */
#define MXFP4_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/*
 * The same layer as mxfp4_linear, for callers that cannot allocate device
 * memory when they run it -- for instance an inference engine whose memory
 * plan is fixed at start-up, a plugin running inside another framework's
 * enqueue step where allocation is not allowed, or latency-critical code that
 * must avoid cudaMalloc's implicit device synchronisation. (The pages have no
 * counterpart: this is an interface choice of this library.)
 *
 * The caller passes inputs and outputs exactly as for mxfp4_linear but no
 * workspace: the quantised activations live in a static device array of
 * MXFP4_NOALLOC_SCRATCH_BYTES (32 MiB) inside the library, which every GPU
 * that loads the library keeps until the process exits. Nothing is allocated
 * per call (no cudaMalloc / cudaFree, no allocating library routine).
 *  - Arguments are checked exactly as mxfp4_linear checks them.
 *  - Limit: 256 + round256(M * K / 2) + round256(mxfp4_sf_bytes(M, K)), plus
 *    4 bytes per 128 rows and 4 more for more than 128 rows (the one-kernel
 *    form's counters), must not exceed the array (about 62 million activation
 *    elements); larger problems return MXFP4_ERR_WORKSPACE and launch nothing.
 *    The rest of the array holds the few-row GEMM's K-split partials when they
 *    fit (else it sums them on chip: slower, the same bits).
 *  - status: optional DEVICE pointer to a caller-owned, 4-byte aligned int
 *    that the caller zeroes; a bounded-wait timeout sets it to
 *    MXFP4_ERR_TIMEOUT. With NULL the library keeps a status word in its array
 *    (the caller cannot read it).
 *  - Each call first clears the array's status region (one cudaMemsetAsync
 *    of 256 bytes on `stream`), so a status that an earlier call left there
 *    is not seen; every other part it reads it writes first. A call after a
 *    timeout needs no reset.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Every call shares the one array, which keeps the previous call's
 *    contents (see the clearing above). Calls whose
 *    kernels can overlap on the GPU -- different streams, or host threads
 *    without ordering between them -- race on the array and corrupt each
 *    other's results; keep them on one stream or otherwise ordered.
 */
mxfp4_status mxfp4_linear_noalloc(const void* x, int64_t M, int64_t K, mxfp4_rotation mode,
                                  const float* kron_a, const float* kron_b, const uint8_t* wq,
                                  const uint8_t* wsf, int64_t N, void* y, int* status,
                                  mxfp4_stream_t stream);

/*
 * Testing only: the faults that mxfp4_test_set_fault can make the GEMM simulate.
 * MXFP4_TEST_FAULT_WITHHOLD_ACCUMULATOR: in the CTA-pair GEMM (M > 128), the first
 * CTA pair never signals that its first accumulator is complete. Its epilogue
 * waits for that signal at most 1 ms (instead of 2 s), records MXFP4_ERR_TIMEOUT
 * in the status word and stops; the pair's other roles see the stop at their
 * next bounded wait, drain their copies, release tensor memory and return, so
 * the kernel ends normally. The tiles of that pair are not written; every other
 * pair's tiles are right.
 */
typedef enum {
  MXFP4_TEST_FAULT_NONE = 0,
  MXFP4_TEST_FAULT_WITHHOLD_ACCUMULATOR = 1
} mxfp4_test_fault;

/*
 * Testing only: make the GEMM launches set up after this call simulate `fault`
 * (MXFP4_TEST_FAULT_NONE restores normal operation, the state at load time).
 * It lets a test drive a bounded device wait to its limit -- the path that
 * reports MXFP4_ERR_TIMEOUT -- with no GPU fault and no hang. Process-wide
 * and read when a launch is set up; never call it in production code.
 * Unknown values -> MXFP4_ERR_UNSUPPORTED.
 */
mxfp4_status mxfp4_test_set_fault(int fault);

/*
 * Read the device status word at the start of a workspace (synchronises with
 * the device): MXFP4_OK, or MXFP4_ERR_TIMEOUT if a kernel's bounded wait on a
 * pipeline barrier ran out (the kernel then stopped early, released its
 * tensor memory and returned; its output is incomplete). The word is sticky:
 * kernels only ever set it, this call clears it. Zero the whole workspace once
 * when it is allocated, and again after a timeout (a kernel that stopped early
 * can leave the NVFP4 tensor-scale pass's words set). mxfp4_linear_noalloc
 * needs no such reset: it clears its own at each call.
 */
mxfp4_status mxfp4_poll_status(void* ws, mxfp4_status* out);

#ifdef __cplusplus
}
#endif

#endif /* MXFP4_H_ */
