/*
 * MXFP4 W4A4 linear block -- plain CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY. This file defines what the CUDA path must compute
 * and is used by the tests, by the smoke check and by the benchmark's CPU
 * baseline leg. Nothing in the product path may link, load or call it. It
 * shares no code, header, table or constant with the CUDA sources.
 *
 * Sources (pages, by title and section):
 *  [AMD]  "AMD Quark delivers MXFP4 quantization for FLUX.1-dev on Instinct
 *         MI350 with 1.92x speedup", section "What is MXFP4 and why does it
 *         eliminate dequantization overhead?": 4 bits per element, blocks of
 *         32 elements sharing one higher-precision scale, part of the
 *         Microscaling (MX) specification; the GEMM consumes MXFP4 directly
 *         with no dequantisation to FP16/BF16 (opening section).
 *  [MRG]  "Bridging the Gap Between Promise and Performance for Microscaling
 *         FP4 Quantization", "Probleemstelling" item 2 (MXFP4: group of 32,
 *         power-of-two scales in E8M0 format), "Methodologie: MR-GPTQ" item 1
 *         (block-wise Hadamard rotation of weights and activations before
 *         quantisation; RTN baseline) and "GPU Kernel Ondersteuning (QuTLASS)"
 *         (the activation rotation runs online, fused with quantisation).
 *  [KRQ]  "KroQuant: Effiziente Post-Training-Quantisierung fuer Diffusion
 *         Transformers mittels Kronecker-Produkt-Struktur", abstract,
 *         "Hintergrund" (invertible transform on activations, inverse on the
 *         weights, run online) and "Tiefenanalyse" (a learned Kronecker-
 *         structured transform applied to every 32-element activation block).
 *
 * Where the pages leave a step open, the reading taken is stated beside it:
 *  - E2M1 element values {0, 0.5, 1, 1.5, 2, 3, 4, 6} with a sign bit (bit 3):
 *    the MX format's FP4 element, which the pages name but do not spell out.
 *  - Scale rule: e = floor(log2(amax)) - 2 (2 = exponent of the largest E2M1
 *    magnitude, 6 = 1.5 * 2^2), clamped to [-127, 127], stored as e + 127.
 *    floor(log2) is read exactly from the fp32 bit pattern.
 *    All-zero block -> byte 0. Any non-finite value in the (rotated) block ->
 *    byte 0xFF (the E8M0 NaN) and all codes 0.
 *  - Element rounding: nearest E2M1 magnitude of |y| * 2^-e, ties to the even
 *    code, saturating at 6; the sign is kept, so negatives that round to zero
 *    give code 8 (-0).
 *  - Hadamard: H = H2^(x5) / sqrt(32) (Sylvester order), evaluated as a
 *    five-stage butterfly (strides 1, 2, 4, 8, 16; (a, b) -> (a + b, a - b))
 *    in fp32, then one fp32 multiply by the fp32 value nearest 1/sqrt(32).
 *  - Kronecker: T = A (x) B, A 4x4, B 8x8, one T shared by every block;
 *    y[8i+k] = sum_j A[i][j] * z[8j+k], z[8j+k] = sum_l B[k][l] * x[8j+l],
 *    each sum in fp32 as the first product (one rounding) followed by fmaf
 *    steps in ascending index order.
 *    Weights take T^-T = A^-T (x) B^-T (inverses in double, rounded to fp32).
 *  - Packing: byte j of a row holds element 2j in bits 0-3 and element 2j+1
 *    in bits 4-7.
 *  - GEMM: Y[m][n] = sum over blocks b of 2^(sx + sw - 254) *
 *    sum_{i in b} v(qx_i) * v(qw_i): exact integer block sums (values are
 *    multiples of 1/2, so products are multiples of 1/4), then a double sum
 *    over blocks. S[m][n] = sum |v(qx_i) v(qw_i)| * scale is returned as the
 *    magnitude for the tolerance rule.
 *
 * Built with -O2 -ffp-contract=off and no fast-math, so every fp32 operation
 * below is one IEEE round-to-nearest-even operation, subnormals included.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- formats */

/* E2M1 magnitudes for codes 0..7 (bit 3 of a code is the sign). */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* Twice the signed E2M1 value of each code: an integer in [-12, 12]. */
static int e2m1_twice(int code) {
  int m = (int)(2.0 * E2M1_MAG[code & 7]);
  return (code & 8) ? -m : m;
}

double oracle_e2m1_value(int code) {
  double m = E2M1_MAG[code & 7];
  return (code & 8) ? -m : m;
}

double oracle_e8m0_value(int byte) {
  if (byte == 255) return NAN;
  return ldexp(1.0, byte - 127);
}

/* Nearest E2M1 magnitude code for a >= 0, ties to the even code; above 6 the
 * nearest grid point is 6 itself, which is the saturation. */
static int e2m1_magnitude_code(double a) {
  int best = 0;
  double best_d = fabs(a - E2M1_MAG[0]);
  for (int c = 1; c < 8; ++c) {
    double d = fabs(a - E2M1_MAG[c]);
    if (d < best_d || (d == best_d && (c % 2) == 0)) {
      best = c;
      best_d = d;
    }
  }
  return best;
}

/* Signed E2M1 code of s (round to nearest, ties to even, saturating). */
int oracle_e2m1_code(double s) {
  int c = e2m1_magnitude_code(fabs(s));
  return signbit(s) ? (c | 8) : c;
}

void oracle_e2m1_code_array(const double* s, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)oracle_e2m1_code(s[i]);
}

/* floor(log2(a)) for finite a > 0, from the fp32 bits. */
int oracle_floor_log2_f32(float a) {
  uint32_t u;
  memcpy(&u, &a, 4);
  int biased = (int)((u >> 23) & 0xFF);
  if (biased != 0) return biased - 127;
  uint32_t mant = u & 0x7FFFFF; /* subnormal: value = mant * 2^-149 */
  int top = 31;
  while (!((mant >> top) & 1u)) --top;
  return top - 149;
}

/* Shared-scale exponent of a block whose largest magnitude is amax (finite). */
int oracle_scale_exponent(float amax) {
  if (amax == 0.0f) return -127;
  int e = oracle_floor_log2_f32(amax) - 2;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

/* Quantise one block of 32 fp32 values: codes (unpacked, 32 bytes) + E8M0 byte. */
void oracle_quantize_block(const float* y, uint8_t* codes, uint8_t* scale_byte) {
  float amax = 0.0f;
  int finite = 1;
  for (int i = 0; i < 32; ++i) {
    if (!isfinite(y[i])) finite = 0;
    else if (fabsf(y[i]) > amax) amax = fabsf(y[i]);
  }
  if (!finite) {
    *scale_byte = 0xFF;
    memset(codes, 0, 32);
    return;
  }
  int e = oracle_scale_exponent(amax);
  *scale_byte = (uint8_t)(e + 127);
  for (int i = 0; i < 32; ++i) codes[i] = (uint8_t)oracle_e2m1_code(ldexp((double)y[i], -e));
}

/* -------------------------------------------------------------- rotations */

/* The fp32 value nearest 1/sqrt(32) = 0.17677669529663688... */
static const float INV_SQRT32 = 0x1.6a09e6p-3f;

float oracle_inv_sqrt32(void) { return INV_SQRT32; }

/* Unnormalised five-stage Walsh-Hadamard butterfly, fp32. */
void oracle_fwht32_unnormalised(const float* x, float* v) {
  for (int i = 0; i < 32; ++i) v[i] = x[i];
  for (int s = 0; s < 5; ++s) {
    int h = 1 << s;
    for (int i = 0; i < 32; ++i) {
      if (i & h) continue;
      float a = v[i], b = v[i + h];
      v[i] = a + b;
      v[i + h] = a - b;
    }
  }
}

/* y = H32 x with H32 = H2^(x5)/sqrt(32): butterfly, then one multiply each. */
void oracle_hadamard32(const float* x, float* y) {
  oracle_fwht32_unnormalised(x, y);
  for (int i = 0; i < 32; ++i) y[i] = y[i] * INV_SQRT32;
}

/* Larger rotation blocks (n = 64 or 128 elements, i.e. 2 or 4 MX blocks), the contrast
 * "KroQuant..." ("Hintergrund") draws with block-wise Hadamard of larger blocks: Sylvester
 * H_n = H2^(x log2 n) / sqrt(n), butterfly strides 1, 2, ..., n/2 in fp32, then one
 * multiply by the fp32 nearest 1/sqrt(n). The scales stay per 32 elements. */
static const float INV_SQRT64 = 0.125f;          /* exact */
static const float INV_SQRT128 = 0x1.6a09e6p-4f; /* = fp32(1/sqrt(32)) / 2, exact halving */

void oracle_fwht_unnormalised(const float* x, int n, float* v) {
  for (int i = 0; i < n; ++i) v[i] = x[i];
  for (int h = 1; h < n; h <<= 1)
    for (int i = 0; i < n; ++i) {
      if (i & h) continue;
      float a = v[i], b = v[i + h];
      v[i] = a + b;
      v[i + h] = a - b;
    }
}

void oracle_hadamard_n(const float* x, int n, float* y) {
  const float c = n == 32 ? INV_SQRT32 : n == 64 ? INV_SQRT64 : INV_SQRT128;
  oracle_fwht_unnormalised(x, n, y);
  for (int i = 0; i < n; ++i) y[i] = y[i] * c;
}

/* Elements per rotation group of a mode: 32, or 64 / 128 for modes 3 / 4. */
int oracle_rotation_span(int mode) { return mode == 3 ? 64 : mode == 4 ? 128 : 32; }

/* y = (A (x) B) x for one 32-block; A 4x4, B 8x8 row-major fp32. */
void oracle_kron32(const float* A, const float* B, const float* x, float* y) {
  float z[32];
  for (int j = 0; j < 4; ++j)
    for (int k = 0; k < 8; ++k) {
      float acc = B[k * 8 + 0] * x[8 * j + 0];
      for (int l = 1; l < 8; ++l) acc = fmaf(B[k * 8 + l], x[8 * j + l], acc);
      z[8 * j + k] = acc;
    }
  for (int i = 0; i < 4; ++i)
    for (int k = 0; k < 8; ++k) {
      float acc = A[i * 4 + 0] * z[8 * 0 + k];
      for (int j = 1; j < 4; ++j) acc = fmaf(A[i * 4 + j], z[8 * j + k], acc);
      y[8 * i + k] = acc;
    }
}

/* Rotate n blocks (n x 32 fp32) in mode 0 (none), 1 (Hadamard), 2 (Kronecker). */
void oracle_rotate_blocks(const float* x, int64_t n, int mode, const float* A, const float* B,
                          float* y) {
  for (int64_t i = 0; i < n; ++i) {
    if (mode == 1) oracle_hadamard32(x + 32 * i, y + 32 * i);
    else if (mode == 2) oracle_kron32(A, B, x + 32 * i, y + 32 * i);
    else memcpy(y + 32 * i, x + 32 * i, 32 * sizeof(float));
  }
}

void oracle_quantize_blocks(const float* y, int64_t n, uint8_t* codes, uint8_t* scales) {
  for (int64_t i = 0; i < n; ++i) oracle_quantize_block(y + 32 * i, codes + 32 * i, scales + i);
}

/* bf16 bits -> fp32 (exact). */
static float bf16_to_f32(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/*
 * Rotate-and-quantise a row-major matrix x[rows, K] (leading dimension ldx
 * elements; xdt 0 = bf16 bits, 1 = fp32). Outputs, in the LOGICAL layout:
 * q[rows, K/2] packed codes and s[rows, K/32] E8M0 bytes. K % 32 == 0.
 */
void oracle_rotate_quantize(const void* x, int xdt, int64_t rows, int64_t K, int64_t ldx, int mode,
                            const float* A, const float* B, uint8_t* q, uint8_t* s) {
  const int64_t nb = K / 32;
  const int span = oracle_rotation_span(mode); /* K % span == 0 */
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    float xin[128], y[128];
    uint8_t codes[32];
    for (int64_t g = 0; g < K / span; ++g) {
      for (int i = 0; i < span; ++i) {
        int64_t idx = r * ldx + (int64_t)span * g + i;
        xin[i] = xdt == 0 ? bf16_to_f32(((const uint16_t*)x)[idx]) : ((const float*)x)[idx];
      }
      if (mode == 3 || mode == 4) oracle_hadamard_n(xin, span, y);
      else oracle_rotate_blocks(xin, 1, mode, A, B, y);
      for (int c = 0; c < span / 32; ++c) {
        const int64_t b = (int64_t)(span / 32) * g + c;
        oracle_quantize_block(y + 32 * c, codes, s + r * nb + b);
        for (int j = 0; j < 16; ++j)
          q[r * (K / 2) + 16 * b + j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
      }
    }
  }
}

/* Dequantise the logical MXFP4 matrix back to double (codes * 2^(s-127)). */
void oracle_dequantize(const uint8_t* q, const uint8_t* s, int64_t rows, int64_t K, double* out) {
  int64_t nb = K / 32;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = q[r * (K / 2) + k / 2];
      int code = (k & 1) ? (byte >> 4) : (byte & 15);
      out[r * K + k] = oracle_e2m1_value(code) * oracle_e8m0_value(s[r * nb + k / 32]);
    }
}

/* ------------------------------------------------------------------- GEMM */

static int code_at(const uint8_t* q, int64_t K, int64_t row, int64_t k) {
  uint8_t byte = q[row * (K / 2) + k / 2];
  return (k & 1) ? (byte >> 4) : (byte & 15);
}

/*
 * Exact block-scaled contraction for a list of (m, n) pairs:
 * ref = sum_b 2^(sa[m,b] + sb[n,b] - 254) * sum_{i in b} v(qa) v(qb), and
 * S   = sum_b 2^(...) * sum_{i in b} |v(qa) v(qb)|.
 * Operands in the logical layout (q: rows x K/2, s: rows x K/32).
 */
void oracle_gemm_pairs(const uint8_t* aq, const uint8_t* as, const uint8_t* bq, const uint8_t* bs,
                       int64_t K, const int64_t* mi, const int64_t* ni, int64_t npairs, double* ref,
                       double* S) {
  int64_t nb = K / 32;
#pragma omp parallel for schedule(dynamic, 64)
  for (int64_t p = 0; p < npairs; ++p) {
    int64_t m = mi[p], n = ni[p];
    double acc = 0.0, mag = 0.0;
    for (int64_t b = 0; b < nb; ++b) {
      int64_t quarters = 0, quarters_abs = 0; /* products of 2v(.) pairs: units of 1/4 */
      for (int64_t i = 32 * b; i < 32 * b + 32; ++i) {
        int prod = e2m1_twice(code_at(aq, K, m, i)) * e2m1_twice(code_at(bq, K, n, i));
        quarters += prod;
        quarters_abs += prod < 0 ? -prod : prod;
      }
      int sa = as[m * nb + b], sb = bs[n * nb + b];
      double w = (sa == 255 || sb == 255) ? NAN : ldexp(1.0, sa + sb - 254 - 2);
      acc += (double)quarters * w;
      mag += (double)quarters_abs * w;
    }
    ref[p] = acc;
    S[p] = mag;
  }
}

/* Full product for all rows of a and b: ref[M][N], S[M][N]. */
void oracle_gemm(const uint8_t* aq, const uint8_t* as, const uint8_t* bq, const uint8_t* bs,
                 int64_t M, int64_t N, int64_t K, double* ref, double* S) {
  int64_t np = M * N;
  int64_t* mi = (int64_t*)malloc(sizeof(int64_t) * (size_t)np);
  int64_t* ni = (int64_t*)malloc(sizeof(int64_t) * (size_t)np);
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      mi[m * N + n] = m;
      ni[m * N + n] = n;
    }
  oracle_gemm_pairs(aq, as, bq, bs, K, mi, ni, np, ref, S);
  free(mi);
  free(ni);
}

/* ------------------------------------------------------------ helpers */

/* Round a double to the nearest bf16 value (ties to even), returned as double. */
double oracle_bf16_round(double x) {
  if (x == 0.0 || !isfinite(x)) return x;
  int e;
  frexp(fabs(x), &e);             /* |x| = f * 2^e, f in [0.5, 1) */
  int lsb_exp = (e - 1) - 7;      /* 8 significant bits */
  if (lsb_exp < -133) lsb_exp = -133; /* bf16 subnormal spacing */
  double scaled = ldexp(x, -lsb_exp);
  double r = nearbyint(scaled);   /* default rounding mode: nearest, ties to even */
  double out = ldexp(r, lsb_exp);
  if (fabs(out) >= 0x1.0p128) return x > 0 ? INFINITY : -INFINITY;
  return out;
}

void oracle_bf16_round_array(const double* x, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_round(x[i]);
}

/* Gauss-Jordan inverse with partial pivoting in double. Returns 0, or -1 if singular. */
int oracle_inverse(const double* A, int n, double* inv) {
  double a[64 * 128];
  if (n > 64) return -1;
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < 2 * n; ++j) a[i * 2 * n + j] = j < n ? A[i * n + j] : (j - n == i ? 1.0 : 0.0);
  for (int c = 0; c < n; ++c) {
    int piv = c;
    for (int r = c + 1; r < n; ++r)
      if (fabs(a[r * 2 * n + c]) > fabs(a[piv * 2 * n + c])) piv = r;
    if (fabs(a[piv * 2 * n + c]) < 1e-300) return -1;
    if (piv != c)
      for (int j = 0; j < 2 * n; ++j) {
        double t = a[c * 2 * n + j];
        a[c * 2 * n + j] = a[piv * 2 * n + j];
        a[piv * 2 * n + j] = t;
      }
    double d = a[c * 2 * n + c];
    for (int j = 0; j < 2 * n; ++j) a[c * 2 * n + j] /= d;
    for (int r = 0; r < n; ++r) {
      if (r == c) continue;
      double f = a[r * 2 * n + c];
      if (f == 0.0) continue;
      for (int j = 0; j < 2 * n; ++j) a[r * 2 * n + j] -= f * a[c * 2 * n + j];
    }
  }
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < n; ++j) inv[i * n + j] = a[i * 2 * n + n + j];
  return 0;
}

/* Weight-side factors for the Kronecker mode: A^-T and B^-T, inverted in double, rounded to fp32. */
int oracle_kron_weight_factors(const float* A, const float* B, float* At_inv, float* Bt_inv) {
  double a[16], b[64], ai[16], bi[64];
  for (int i = 0; i < 16; ++i) a[i] = A[i];
  for (int i = 0; i < 64; ++i) b[i] = B[i];
  if (oracle_inverse(a, 4, ai) || oracle_inverse(b, 8, bi)) return -1;
  for (int i = 0; i < 4; ++i)
    for (int j = 0; j < 4; ++j) At_inv[i * 4 + j] = (float)ai[j * 4 + i];
  for (int i = 0; i < 8; ++i)
    for (int j = 0; j < 8; ++j) Bt_inv[i * 8 + j] = (float)bi[j * 8 + i];
  return 0;
}

/*
 * Physical scale-factor layout (the tensor-core operand layout the library
 * writes): rows tiled by 128 and 32-blocks by 4 into 512-byte atoms, atoms
 * ordered block-group fastest then row tile; inside an atom the byte of
 * (row r, block kb) sits at (r % 32) * 16 + ((r / 32) % 4) * 4 + kb % 4.
 * Rows pad to a multiple of 128 and blocks to a multiple of 4, padding 0.
 */
int64_t oracle_sf_bytes(int64_t rows, int64_t K) {
  int64_t rt = (rows + 127) / 128, ka = (K / 32 + 3) / 4;
  return rt * ka * 512;
}

int64_t oracle_sf_offset(int64_t row, int64_t kb, int64_t K) {
  int64_t ka = (K / 32 + 3) / 4;
  return ((row / 128) * ka + kb / 4) * 512 + (row % 32) * 16 + ((row / 32) % 4) * 4 + (kb % 4);
}

/* Logical [rows, K/32] scales -> physical buffer (padding zero). */
void oracle_sf_to_physical(const uint8_t* s, int64_t rows, int64_t K, uint8_t* phys) {
  memset(phys, 0, (size_t)oracle_sf_bytes(rows, K));
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < K / 32; ++b) phys[oracle_sf_offset(r, b, K)] = s[r * (K / 32) + b];
}

/* Physical buffer -> logical [rows, K/32]. */
void oracle_sf_from_physical(const uint8_t* phys, int64_t rows, int64_t K, uint8_t* s) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < K / 32; ++b) s[r * (K / 32) + b] = phys[oracle_sf_offset(r, b, K)];
}

/* ------------------------------------------------------------------ NVFP4
 *
 * The other FP4 format the pages compare ("Bridging the Gap Between Promise and
 * Performance for Microscaling FP4 Quantization", "Probleemstelling" item 1 and
 * "Format-specifieke Schaaloptimalisatie"): E2M1 elements in groups of 16, each group
 * with its own scale, plus one scale for the whole tensor. Read as NVIDIA's NVFP4: the
 * group scale is an unsigned E4M3 byte (4 exponent bits, bias 7, 3 mantissa bits, no
 * infinities; finite codes 0..126, largest 448), the tensor scale an fp32 number.
 */
double oracle_e4m3_value(int b) {
  int e = (b >> 3) & 15, m = b & 7;
  if (e == 0) return ldexp((double)m, -9); /* subnormal: m/8 * 2^(1-7) */
  return ldexp(1.0 + m / 8.0, e - 7);
}

/* Nearest finite E4M3 code to v >= 0, ties to the even code, above 448 -> 448. */
int oracle_e4m3_code(double v) {
  int best = 0;
  double bd = fabs(v - oracle_e4m3_value(0));
  for (int c = 1; c <= 126; ++c) {
    double d = fabs(v - oracle_e4m3_value(c));
    if (d < bd || (d == bd && (c & 1) == 0 && (best & 1) == 1)) {
      best = c;
      bd = d;
    }
  }
  return best;
}

/* One group of 16 fp32 values with tensor scale st (> 0, or 0 for an all-zero tensor):
 * g = amax / (6 st) in two fp32 roundings, group byte = nearest E4M3 of g, element scale
 * S = E4M3(byte) * st (one fp32 rounding), r = 1 / S (one rounding), code_i = nearest
 * E2M1 of y_i * r (one rounding; ties to even, saturating at 6, sign kept). */
void oracle_nvfp4_quantize_group(const float* y, float st, uint8_t* codes, uint8_t* sbyte) {
  float amax = 0.0f;
  for (int i = 0; i < 16; ++i) {
    float a = fabsf(y[i]);
    if (a > amax) amax = a;
  }
  if (!(st > 0.0f)) {
    *sbyte = 0;
    memset(codes, 0, 16);
    return;
  }
  float den = 6.0f * st;
  float g = amax / den;
  int sb = oracle_e4m3_code((double)g);
  *sbyte = (uint8_t)sb;
  float S = (float)oracle_e4m3_value(sb) * st;
  if (S == 0.0f) {
    memset(codes, 0, 16);
    return;
  }
  float r = 1.0f / S;
  for (int i = 0; i < 16; ++i) {
    float v = y[i] * r;
    codes[i] = (uint8_t)oracle_e2m1_code((double)v);
  }
}

static void load_block(const void* x, int xdt, int64_t idx, float* out) {
  for (int i = 0; i < 32; ++i)
    out[i] = xdt == 0 ? bf16_to_f32(((const uint16_t*)x)[idx + i]) : ((const float*)x)[idx + i];
}

/* Tensor scale of x rotated by mode (0 none, 1 Hadamard-32): amax / (6 * 448), one
 * fp32 rounding; 0 for an all-zero tensor. K % 32 == 0. */
float oracle_nvfp4_tensor_scale(const void* x, int xdt, int64_t rows, int64_t K, int64_t ldx,
                                int mode) {
  float amax = 0.0f;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < K / 32; ++b) {
      float xin[32], y[32];
      load_block(x, xdt, r * ldx + 32 * b, xin);
      if (mode == 1) oracle_hadamard32(xin, y);
      else memcpy(y, xin, sizeof(y));
      for (int i = 0; i < 32; ++i)
        if (fabsf(y[i]) > amax) amax = fabsf(y[i]);
    }
  return amax / 2688.0f;
}

/* Rotate (mode 0 / 1) and quantise x[rows, K] to NVFP4 with tensor scale st: q[rows, K/2]
 * packed codes (element 2j low nibble of byte j), s[rows, K/16] E4M3 group bytes. */
void oracle_nvfp4_rotate_quantize(const void* x, int xdt, int64_t rows, int64_t K, int64_t ldx,
                                  int mode, float st, uint8_t* q, uint8_t* s) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < K / 32; ++b) {
      float xin[32], y[32];
      uint8_t codes[32];
      load_block(x, xdt, r * ldx + 32 * b, xin);
      if (mode == 1) oracle_hadamard32(xin, y);
      else memcpy(y, xin, sizeof(y));
      oracle_nvfp4_quantize_group(y, st, codes, s + r * (K / 16) + 2 * b);
      oracle_nvfp4_quantize_group(y + 16, st, codes + 16, s + r * (K / 16) + 2 * b + 1);
      for (int j = 0; j < 16; ++j)
        q[r * (K / 2) + 16 * b + j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
    }
  }
}

/* Exact NVFP4 product: ref[m][n] = alpha * sum_g E4M3(as[m,g]) E4M3(bs[n,g])
 * sum_{i in g} v(a_i) v(b_i) (per-group integer sums in units of 1/4, then double),
 * S[m][n] = |alpha| * sum_i |a_i b_i| with the group scales. */
void oracle_nvfp4_gemm(const uint8_t* aq, const uint8_t* as, const uint8_t* bq,
                       const uint8_t* bs, int64_t M, int64_t N, int64_t K, double alpha,
                       double* ref, double* S) {
  const int64_t ng = K / 16;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0, mag = 0.0;
      for (int64_t g = 0; g < ng; ++g) {
        int64_t isum = 0, iabs = 0;
        for (int64_t i = 16 * g; i < 16 * g + 16; ++i) {
          int64_t p = (int64_t)e2m1_twice(code_at(aq, K, m, i)) * e2m1_twice(code_at(bq, K, n, i));
          isum += p;
          iabs += p < 0 ? -p : p;
        }
        const double sc = oracle_e4m3_value(as[m * ng + g]) * oracle_e4m3_value(bs[n * ng + g]);
        acc += (double)isum * 0.25 * sc;
        mag += (double)iabs * 0.25 * sc;
      }
      ref[m * N + n] = alpha * acc;
      S[m * N + n] = fabs(alpha) * mag;
    }
}

/* ------------------------------------------------------- norm prologue (row f3)
 *
 * The step right before the rotation ("KroQuant: Effiziente Post-Training-Quantisierung
 * fuer Diffusion Transformers mittels Kronecker-Produkt-Struktur", "Hintergrund": the
 * normalisation layers are why the transform has to run online). Two norms:
 *   kind 0 (LayerNorm): mu = mean(x), var = mean((x - mu)^2), rstd = 1 / sqrt(var + eps);
 *   kind 1 (RMSNorm):   mu = 0, rstd = 1 / sqrt(mean(x^2) + eps);
 * then, per element, v = ((x - mu) * rstd) * g[c] + b[c] (g = 1 and b = 0 when absent),
 * before the rotation and quantisation. The statistics are defined in exact arithmetic
 * and computed here in double; the per-element steps are fp32 operations in the order
 * written (sub, mul, mul, add), so that given the fp32 statistics a GPU used, the codes
 * follow bit for bit. */
void oracle_row_stats(const void* x, int xdt, int64_t rows, int64_t K, int64_t ldx, int kind,
                      double eps, double* mu, double* rstd) {
  for (int64_t r = 0; r < rows; ++r) {
    double s = 0.0, m = 0.0, v = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      const int64_t idx = r * ldx + k;
      s += xdt == 0 ? bf16_to_f32(((const uint16_t*)x)[idx]) : ((const float*)x)[idx];
    }
    if (kind == 0) m = s / (double)K;
    for (int64_t k = 0; k < K; ++k) {
      const int64_t idx = r * ldx + k;
      const double d = (xdt == 0 ? bf16_to_f32(((const uint16_t*)x)[idx])
                                 : ((const float*)x)[idx]) - m;
      v += d * d;
    }
    mu[r] = m;
    rstd[r] = 1.0 / sqrt(v / (double)K + eps);
  }
}

/* Normalise with the given fp32 statistics (mu_f, rstd_f per row), then rotate-quantise
 * (modes 0, 1, 2) into q[rows, K/2], s[rows, K/32] (logical layout). */
void oracle_norm_rotate_quantize(const void* x, int xdt, int64_t rows, int64_t K, int64_t ldx,
                                 const float* mu_f, const float* rstd_f, const float* g,
                                 const float* bvec, int mode, const float* A, const float* B,
                                 uint8_t* q, uint8_t* s) {
  const int64_t nb = K / 32;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    float xin[32], y[32];
    uint8_t codes[32];
    for (int64_t b = 0; b < nb; ++b) {
      for (int i = 0; i < 32; ++i) {
        const int64_t c = 32 * b + i, idx = r * ldx + c;
        const float xv = xdt == 0 ? bf16_to_f32(((const uint16_t*)x)[idx]) : ((const float*)x)[idx];
        float v = (xv - mu_f[r]) * rstd_f[r];
        if (g) v = v * g[c];
        if (bvec) v = v + bvec[c];
        xin[i] = v;
      }
      oracle_rotate_blocks(xin, 1, mode, A, B, y);
      oracle_quantize_block(y, codes, s + r * nb + b);
      for (int j = 0; j < 16; ++j)
        q[r * (K / 2) + 16 * b + j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
    }
  }
}
