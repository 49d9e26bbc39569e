/*
 * sixbit_oracle.c -- plain, slow, CPU reference for the 6Bit-Diffusion hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and the CPU-baseline leg of
 * bench.py may load this library. The product path (the CUDA library) never calls it, shares
 * no source, header, table or helper with it, and fails loudly when its own build is missing.
 *
 * Source pages (cited by title and section):
 *   [VU]  "6Bit-Diffusion: dynamic quantization ..." popular write-up of arXiv:2603.18742
 *         (vetunion.cn), sections 一 (DMPQ, block Hadamard), 二 (Temporal Delta Cache),
 *         三 (Purified Delta Refresh, INT8 after restart), 四 (W4A6, fused kernel).
 *   [GS]  "6Bit-Diffusion: Inference-Time Mixed-Precision Quantization for Video Diffusion
 *         Models" (gist.science explainer), sections 2 (DMPQ), 3 (TDC), 4 (PDR).
 * The pages name NVFP4 and INT8 but give no encoding recipe, no Hadamard normalisation, no
 * thresholds and no reduction order. Every such gap is filled by a stated reading (R-*), written
 * once here as plain loops so a reader can check it by eye:
 *   R-H     unnormalised Sylvester Hadamard over consecutive blocks of B channels, butterfly
 *           stages h = 1, 2, 4, ... B/2, (a, b) -> (a + b, a - b), FP32 round-to-nearest-even.
 *   R-RED   per-row sums: pairwise FP32 tree over the row zero-padded to a power of two;
 *           across rows: the same pairwise tree in FP64 over the row partials.
 *   R-D     d = sqrt(sum (y - x)^2) / sqrt(sum x^2), FP64.
 *   R-PDR   ratio = max|x| / (sum|x| / numel) on the raw (unrotated) layer input, FP64.
 *   R-INT8  symmetric per-token: s = a / 127, q = clamp(rne(y * (127 / a)), -127, 127), FP32;
 *           when 127 / a overflows, y = 0 gives 0 (its exact product) instead of 0 * inf.
 *   R-FP4   NVFP4: E2M1 codes, one E4M3 scale per 16 elements, FP32 tensor scale A / (6 * 448).
 *   R-RULE  INT8 iff a * d_prev + b > tau (FP64, no fused multiply-add); restart -> INT8.
 *   R-TDC   delta = sum|y_new - y_last| / sum|y_last|; acc += delta each later step;
 *           skip iff acc <= threshold; a computed step resets acc to 0.
 *   R-REUSE the cache keeps the module's residual D = y - x of its last computed step (bf16: the
 *           FP32 difference of the bf16 values, rounded to nearest even); a skipped step
 *           returns y = x + D (FP32 sum of the bf16 values, rounded to nearest even).
 *   R-REUSE-FP8 the same residual kept in FP8: E4M3 codes with one FP32 scale per token
 *           (s = max|d| / 448, the recipe of R-DQ-FP8); a skipped step returns bf16(x + E4M3 * s).
 * Parity of R-RULE constants, R-TDC accumulator semantics and R-PDR granularity is pinned only
 * to these definitions ("parity unpinned" against the pages, which print no constants).
 *
 * Build: gcc -O2 -fno-fast-math -ffp-contract=off -fopenmp -shared -fPIC (x86-64 SSE, default
 * round-to-nearest-even). OpenMP only splits independent rows; results do not depend on it.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#include <float.h>

#define ORC_NVFP4 0
#define ORC_INT8 1
#define ORC_BF16 2
#define ORC_SKIP 3

/* ------------------------------------------------------------------------------------------ */
/* bf16 and helpers                                                                            */
/* ------------------------------------------------------------------------------------------ */

static float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* round-to-nearest-even FP32 -> bf16 (used only to compare against bf16 GPU outputs) */
uint16_t orc_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u); /* NaN */
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

static int64_t pow2_ceil(int64_t n) {
  int64_t p = 1;
  while (p < n) p <<= 1;
  return p;
}

/* ------------------------------------------------------------------------------------------ */
/* R-H: Hadamard                                                                               */
/* ------------------------------------------------------------------------------------------ */

/* Closed form of the Sylvester matrix entry: H[i][j] = (-1)^popcount(i & j). */
int orc_hadamard_entry(int i, int j) {
  return (__builtin_popcount((unsigned)(i & j)) & 1) ? -1 : 1;
}

/* In-place fast Walsh-Hadamard transform of one block of B values (B a power of two),
 * unnormalised, stages h = 1, 2, 4, ..., B/2 ascending, FP32 round-to-nearest-even. */
void orc_fwht_f32(float* v, int B) {
  for (int h = 1; h < B; h <<= 1) {
    for (int j0 = 0; j0 < B; j0 += 2 * h) {
      for (int j = j0; j < j0 + h; ++j) {
        float a = v[j];
        float b = v[j + h];
        v[j] = a + b;
        v[j + h] = a - b;
      }
    }
  }
}

/* y[m][k] = (H_B x[m][block])[k]: bf16 -> FP32 (exact), then the block FWHT along each row. */
void orc_rotate_rows(const uint16_t* x, int64_t M, int64_t K, int B, float* y) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    float* row = y + m * K;
    for (int64_t k = 0; k < K; ++k) row[k] = bf16_to_f32(x[m * K + k]);
    for (int64_t j = 0; j < K; j += B) orc_fwht_f32(row + j, B);
  }
}

/* ------------------------------------------------------------------------------------------ */
/* R-RED: deterministic pairwise sums                                                          */
/* ------------------------------------------------------------------------------------------ */

/* S(lo, n) = S(lo, n/2) + S(lo + n/2, n/2) over the n terms zero-padded to a power of two,
 * evaluated level by level (adjacent pairs first), in FP32. */
float orc_pairwise_f32(const float* t, int64_t n) {
  if (n <= 0) return 0.0f;
  int64_t p = pow2_ceil(n);
  float* buf = (float*)calloc((size_t)p, sizeof(float));
  memcpy(buf, t, (size_t)n * sizeof(float));
  for (int64_t len = p; len > 1; len >>= 1)
    for (int64_t i = 0; i < len / 2; ++i) buf[i] = buf[2 * i] + buf[2 * i + 1];
  float r = buf[0];
  free(buf);
  return r;
}

double orc_pairwise_f64(const double* t, int64_t n) {
  if (n <= 0) return 0.0;
  int64_t p = pow2_ceil(n);
  double* buf = (double*)calloc((size_t)p, sizeof(double));
  memcpy(buf, t, (size_t)n * sizeof(double));
  for (int64_t len = p; len > 1; len >>= 1)
    for (int64_t i = 0; i < len / 2; ++i) buf[i] = buf[2 * i] + buf[2 * i + 1];
  double r = buf[0];
  free(buf);
  return r;
}

/* ------------------------------------------------------------------------------------------ */
/* Pre-pass: rotation, per-token amax, PDR ratio, difference statistic                         */
/* ------------------------------------------------------------------------------------------ */

/* Statistics record written by orc_prepass (indices of `out`):
 *   0 sum|x|   1 sum (x - x_ref)^2   2 sum x_ref^2   3 max|x|   4 max_m a_m (rotated amax)
 *   5 ratio = max|x| / (sum|x| / numel)   6 d = sqrt(out[1]) / sqrt(out[2])   7 numel
 * The rotation is of X (the layer input); statistics 0, 3 and 5 are of the raw X
 * ([VU] section 三: outlier ratio of the input data, maximum over mean); 1, 2 and 6 compare
 * X (module output y) with X_ref (module input x) ([VU] section 一: difference between a
 * module's input and output). Without X_ref, out[1], out[2] and out[6] are 0. */
void orc_prepass(const uint16_t* X, const uint16_t* Xref, int64_t M, int64_t K, int B,
                 float* y_rot /* nullable, M*K */, float* row_amax /* M */,
                 float* row_part /* nullable, M*3: sum|x|, sum d^2, sum r^2 per row */,
                 double* out /* 8 */) {
  float* rp = row_part ? row_part : (float*)malloc((size_t)M * 3 * sizeof(float));
  float maxabs_all = 0.0f;
#pragma omp parallel
  {
    float* t0 = (float*)malloc((size_t)K * sizeof(float));
    float* t1 = (float*)malloc((size_t)K * sizeof(float));
    float* t2 = (float*)malloc((size_t)K * sizeof(float));
    float* yr = (float*)malloc((size_t)K * sizeof(float));
    float local_max = 0.0f;
#pragma omp for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
      for (int64_t k = 0; k < K; ++k) {
        float xv = bf16_to_f32(X[m * K + k]);
        float ax = fabsf(xv);
        t0[k] = ax;
        if (ax > local_max) local_max = ax;
        if (Xref) {
          float rv = bf16_to_f32(Xref[m * K + k]);
          float dv = xv - rv;
          t1[k] = dv * dv;
          t2[k] = rv * rv;
        } else {
          t1[k] = 0.0f;
          t2[k] = 0.0f;
        }
        yr[k] = xv;
      }
      rp[m * 3 + 0] = orc_pairwise_f32(t0, K);
      rp[m * 3 + 1] = orc_pairwise_f32(t1, K);
      rp[m * 3 + 2] = orc_pairwise_f32(t2, K);
      for (int64_t j = 0; j < K; j += B) orc_fwht_f32(yr + j, B);
      float am = 0.0f;
      for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(yr[k]);
        if (a > am) am = a;
      }
      row_amax[m] = am;
      if (y_rot) memcpy(y_rot + m * K, yr, (size_t)K * sizeof(float));
    }
#pragma omp critical
    {
      if (local_max > maxabs_all) maxabs_all = local_max;
    }
    free(t0);
    free(t1);
    free(t2);
    free(yr);
  }
  double* col = (double*)malloc((size_t)(M > 0 ? M : 1) * sizeof(double));
  for (int s = 0; s < 3; ++s) {
    for (int64_t m = 0; m < M; ++m) col[m] = (double)rp[m * 3 + s];
    out[s] = orc_pairwise_f64(col, M);
  }
  free(col);
  float amax_rot = 0.0f;
  for (int64_t m = 0; m < M; ++m)
    if (row_amax[m] > amax_rot) amax_rot = row_amax[m];
  double numel = (double)M * (double)K;
  out[3] = (double)maxabs_all;
  out[4] = (double)amax_rot;
  if (out[0] == 0.0) {
    out[5] = INFINITY;
  } else {
    double mean = out[0] / numel;
    out[5] = out[3] / mean;
  }
  if (Xref) {
    double num = sqrt(out[1]);
    double den = sqrt(out[2]);
    out[6] = (den == 0.0) ? (num == 0.0 ? 0.0 : INFINITY) : num / den;
  } else {
    out[6] = 0.0;
  }
  out[7] = numel;
  if (!row_part) free(rp);
}

/* Statistics of every aligned 128-channel chunk of every row (K a multiple of 128, B | 128):
 * out[(m * (K / 128) + c) * 3 + i] for chunk c of row m is
 *   i = 0: max over the chunk of |H_B x| (its B-blocks rotated as in R-H),
 *   i = 1: sum of |x| over the chunk's 128 values in the canonical pairwise order (R-RED),
 *   i = 2: max |x|.
 * A chunk is an aligned subtree of its row's sum tree, so these records carry everything the
 * pre-pass needs from the row; they are what the first FFN layer's epilogue produces for the
 * second layer's pre-pass ("write-up" section 四: quantization work fused into the layers). */
void orc_chunk_stats(const uint16_t* x, int64_t M, int64_t K, int B, float* out) {
  const int64_t NC = K / 128;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t c = 0; c < NC; ++c) {
      float v[128], a[128];
      float mx = 0.0f;
      for (int i = 0; i < 128; ++i) {
        v[i] = bf16_to_f32(x[m * K + c * 128 + i]);
        a[i] = fabsf(v[i]);
        if (a[i] > mx) mx = a[i];
      }
      for (int len = 128; len > 1; len >>= 1)
        for (int i = 0; i < len / 2; ++i) a[i] = a[2 * i] + a[2 * i + 1];
      for (int j = 0; j < 128; j += B) orc_fwht_f32(v + j, B);
      float am = 0.0f;
      for (int i = 0; i < 128; ++i)
        if (fabsf(v[i]) > am) am = fabsf(v[i]);
      float* o = out + (m * NC + c) * 3;
      o[0] = am;
      o[1] = a[0];
      o[2] = mx;
    }
  }
}

/* ------------------------------------------------------------------------------------------ */
/* R-INT8                                                                                      */
/* ------------------------------------------------------------------------------------------ */

/* Symmetric per-row INT8 of the rotated rows: s_m = a_m / 127, q = clamp(rne(y * (127/a_m))).
 * a_m = 0 gives s_m = 0 and all codes 0; when 127/a_m overflows, nonzero y clamp to +-127 and
 * y = 0 gives 0. */
void orc_quant_int8(const float* y, int64_t M, int64_t K, const float* row_amax, int8_t* q,
                    float* s) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    float a = row_amax[m];
    if (a == 0.0f) {
      s[m] = 0.0f;
      for (int64_t k = 0; k < K; ++k) q[m * K + k] = 0;
      continue;
    }
    s[m] = a / 127.0f;
    float inv = 127.0f / a;
    for (int64_t k = 0; k < K; ++k) {
      float v = y[m * K + k] * inv;
      float r = nearbyintf(v); /* default rounding mode: nearest, ties to even */
      if (r > 127.0f) r = 127.0f;
      if (r < -127.0f) r = -127.0f;
      /* 127/a overflows to +inf for a below 127/FLT_MAX: y = 0 then gives 0 * inf = NaN, whose
       * exact value y * (127/a) is 0 */
      if (r != r) r = 0.0f;
      q[m * K + k] = (int8_t)r;
    }
  }
}

/* ------------------------------------------------------------------------------------------ */
/* Number formats (OCP Microscaling v1.0 element types; NVFP4 scale = E4M3)                   */
/* ------------------------------------------------------------------------------------------ */

/* E2M1: sign | 2-bit exponent (bias 1) | 1-bit mantissa. Magnitudes by code 0..7. */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

float orc_e2m1_decode(uint8_t c) {
  double v = E2M1_MAG[c & 7];
  return (float)((c & 8) ? -v : v);
}

/* Nearest representable magnitude, ties to the even code (mantissa bit 0), saturating at 6;
 * the sign bit is kept, so a negative value that rounds to zero gives code 0x8. */
uint8_t orc_e2m1_encode(float v) {
  uint8_t sign = signbit(v) ? 8 : 0;
  double a = fabs((double)v);
  if (a >= 6.0) return sign | 7;
  int best = 0;
  double bestd = a;
  for (int c = 1; c < 8; ++c) {
    double d = fabs(a - E2M1_MAG[c]);
    if (d < bestd || (d == bestd && (c & 1) == 0)) {
      best = c;
      bestd = d;
    }
  }
  return (uint8_t)(sign | best);
}

/* E4M3 (the "FN" variant): sign | 4-bit exponent (bias 7) | 3-bit mantissa; no infinities;
 * S.1111.111 is NaN; largest finite 448; subnormals m/8 * 2^-6. */
float orc_e4m3_decode(uint8_t c) {
  int s = c >> 7;
  int e = (c >> 3) & 15;
  int m = c & 7;
  if (e == 15 && m == 7) return NAN;
  double v = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
  return (float)(s ? -v : v);
}

/* Round to nearest, ties to even code, saturate to +-448 (satfinite): a search over every
 * finite non-negative code (their values cached once from orc_e4m3_decode). */
static double E4M3_POS[127];
static int E4M3_POS_READY = 0;

uint8_t orc_e4m3_encode(float v) {
  if (!E4M3_POS_READY) {
#pragma omp critical(orc_e4m3_table)
    {
      if (!E4M3_POS_READY) {
        for (int c = 0; c < 127; ++c) E4M3_POS[c] = (double)orc_e4m3_decode((uint8_t)c);
#pragma omp flush
        E4M3_POS_READY = 1;
      }
    }
  }
  uint8_t sign = signbit(v) ? 0x80 : 0;
  double a = fabs((double)v);
  if (a >= 448.0) return sign | 0x7e;
  int best = 0;
  double bestd = a;
  for (int c = 1; c <= 0x7e; ++c) {
    double d = fabs(a - E4M3_POS[c]);
    if (d < bestd || (d == bestd && (c & 1) == 0)) {
      best = c;
      bestd = d;
    }
  }
  return (uint8_t)(sign | best);
}

/* ------------------------------------------------------------------------------------------ */
/* R-FP4: NVFP4 encode                                                                         */
/* ------------------------------------------------------------------------------------------ */

/* Byte offset of the scale of (row m, 16-element group g) in the tensor-core tiled layout:
 * 512-byte atoms of 128 rows x 4 groups, atom (m/128, g/4) at ((m/128)*(K/64) + g/4)*512,
 * inside the atom row m%32 owns 16 bytes, then the 32-row quarter (m%128)/32, then g%4. */
int64_t orc_sf_tiled_offset(int64_t m, int64_t g, int64_t K) {
  return ((m / 128) * (K / 64) + g / 4) * 512 + (m % 32) * 16 + ((m % 128) / 32) * 4 + (g % 4);
}

int64_t orc_sf_tiled_bytes(int64_t M, int64_t K) { return ((M + 127) / 128) * 128 * (K / 16); }

float orc_nvfp4_tensor_scale(float A) { return (A == 0.0f) ? 1.0f : A / 2688.0f; }

/* Encode rotated rows y [M][K] with tensor amax A:
 *   s_g = A / 2688 (2688 = 6 * 448); per 16-element group along K:
 *   sb = E4M3((amax_g / 6) / s_g), den = dec(sb) * s_g, codes = E2M1(y * (1 / den));
 *   den = 0 or 1/den not finite -> all codes of the group 0.
 * codes: [M][K/2] bytes, element 2i in the low nibble. sf_logical: [M][K/16].
 * sf_tiled (nullable): orc_sf_tiled_bytes(M, K) bytes, padding rows zero. */
void orc_quant_nvfp4(const float* y, int64_t M, int64_t K, float A, uint8_t* codes,
                     uint8_t* sf_logical, uint8_t* sf_tiled, float* s_g_out) {
  float s_g = orc_nvfp4_tensor_scale(A);
  *s_g_out = s_g;
  int64_t G = K / 16;
  if (sf_tiled) memset(sf_tiled, 0, (size_t)orc_sf_tiled_bytes(M, K));
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t g = 0; g < G; ++g) {
      const float* v = y + m * K + g * 16;
      float amax = 0.0f;
      for (int i = 0; i < 16; ++i) {
        float a = fabsf(v[i]);
        if (a > amax) amax = a;
      }
      float sfv = (amax / 6.0f) / s_g;
      uint8_t sb = orc_e4m3_encode(sfv);
      float den = orc_e4m3_decode(sb) * s_g;
      uint8_t q[16];
      float inv = (den == 0.0f) ? 0.0f : 1.0f / den;
      if (den == 0.0f || !(inv <= FLT_MAX)) {
        for (int i = 0; i < 16; ++i) q[i] = 0;
      } else {
        for (int i = 0; i < 16; ++i) q[i] = orc_e2m1_encode(v[i] * inv);
      }
      for (int i = 0; i < 8; ++i)
        codes[m * (K / 2) + g * 8 + i] = (uint8_t)(q[2 * i] | (q[2 * i + 1] << 4));
      sf_logical[m * G + g] = sb;
      if (sf_tiled) sf_tiled[orc_sf_tiled_offset(m, g, K)] = sb;
    }
  }
}

/* ------------------------------------------------------------------------------------------ */
/* GEMM references, FP64                                                                       */
/* ------------------------------------------------------------------------------------------ */

double orc_gelu_tanh(double v) {
  const double c = sqrt(2.0 / 3.14159265358979323846);
  return 0.5 * v * (1.0 + tanh(c * (v + 0.044715 * v * v * v)));
}

static double bias_at(const uint16_t* bias, int64_t n) {
  return bias ? (double)bf16_to_f32(bias[n]) : 0.0;
}

/* Y[r][n] = (s_gx * s_gw / B) * sum_k dec(x[m][k]) * dec(w[n][k]) + bias[n]  (optional GELU),
 * dec(.) = E2M1 value times its group's E4M3 scale; m = rows[r]. Y is FP64 [nrows][N].
 * acc (nullable): the raw sum before the epilogue. */
void orc_gemm_nvfp4(const uint8_t* xc, const uint8_t* xsf, float sgx, const uint8_t* wc,
                    const uint8_t* wsf, float sgw, const uint16_t* bias, int64_t M, int64_t N,
                    int64_t K, int B, int gelu, const int64_t* rows, int64_t nrows, double* Y,
                    double* acc) {
  (void)M;
  int64_t G = K / 16;
  double alpha = ((double)sgx * (double)sgw) / (double)B;
  double* wdec = (double*)malloc((size_t)N * K * sizeof(double));
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = wc[n * (K / 2) + k / 2];
      uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
      wdec[n * K + k] = (double)orc_e2m1_decode(c) * (double)orc_e4m3_decode(wsf[n * G + k / 16]);
    }
#pragma omp parallel
  {
    double* xd = (double*)malloc((size_t)K * sizeof(double));
#pragma omp for schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
      int64_t m = rows[r];
      for (int64_t k = 0; k < K; ++k) {
        uint8_t byte = xc[m * (K / 2) + k / 2];
        uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
        xd[k] = (double)orc_e2m1_decode(c) * (double)orc_e4m3_decode(xsf[m * G + k / 16]);
      }
      for (int64_t n = 0; n < N; ++n) {
        double s = 0.0;
        const double* w = wdec + n * K;
        for (int64_t k = 0; k < K; ++k) s += xd[k] * w[k];
        if (acc) acc[r * N + n] = s;
        double v = s * alpha + bias_at(bias, n);
        Y[r * N + n] = gelu ? orc_gelu_tanh(v) : v;
      }
    }
    free(xd);
  }
  free(wdec);
}

/* acc[r][n] = sum_k qx[m][k] * qw[n][k] (exact, int64);
 * Y[r][n] = acc * s_x[m] * s_w[n] / B + bias[n] (optional GELU), FP64. */
void orc_gemm_int8(const int8_t* qx, const float* sx, const int8_t* qw, const float* sw,
                   const uint16_t* bias, int64_t M, int64_t N, int64_t K, int B, int gelu,
                   const int64_t* rows, int64_t nrows, double* Y, int64_t* acc) {
  (void)M;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t m = rows[r];
    for (int64_t n = 0; n < N; ++n) {
      int64_t s = 0;
      for (int64_t k = 0; k < K; ++k) s += (int64_t)qx[m * K + k] * (int64_t)qw[n * K + k];
      if (acc) acc[r * N + n] = s;
      double v = (double)s * (double)sx[m] * (double)sw[n] / (double)B + bias_at(bias, n);
      Y[r * N + n] = gelu ? orc_gelu_tanh(v) : v;
    }
  }
}

/* Y[r][n] = sum_k x[m][k] * w[n][k] + bias[n] (optional GELU), FP64, raw bf16 operands. */
void orc_gemm_bf16(const uint16_t* X, const uint16_t* W, const uint16_t* bias, int64_t M,
                   int64_t N, int64_t K, int gelu, const int64_t* rows, int64_t nrows, double* Y) {
  (void)M;
  double* wd = (double*)malloc((size_t)N * K * sizeof(double));
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < N * K; ++i) wd[i] = (double)bf16_to_f32(W[i]);
#pragma omp parallel
  {
    double* xd = (double*)malloc((size_t)K * sizeof(double));
#pragma omp for schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
      int64_t m = rows[r];
      for (int64_t k = 0; k < K; ++k) xd[k] = (double)bf16_to_f32(X[m * K + k]);
      for (int64_t n = 0; n < N; ++n) {
        double s = 0.0;
        const double* w = wd + n * K;
        for (int64_t k = 0; k < K; ++k) s += xd[k] * w[k];
        double v = s + bias_at(bias, n);
        Y[r * N + n] = gelu ? orc_gelu_tanh(v) : v;
      }
    }
    free(xd);
  }
  free(wd);
}

/* ------------------------------------------------------------------------------------------ */
/* R-TDC and decisions                                                                         */
/* ------------------------------------------------------------------------------------------ */

/* delta = sum|y_new - y_last| / sum|y_last| with R-RED sums; the difference is taken in FP32
 * from the bf16 values. sum|y_last| = 0 gives +inf (recompute). out[0] = S1, out[1] = S2. */
double orc_tdc_delta(const uint16_t* ynew, const uint16_t* ylast, int64_t M, int64_t C,
                     double* out) {
  float* rp = (float*)malloc((size_t)(M > 0 ? M : 1) * 2 * sizeof(float));
#pragma omp parallel
  {
    float* t0 = (float*)malloc((size_t)C * sizeof(float));
    float* t1 = (float*)malloc((size_t)C * sizeof(float));
#pragma omp for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
      for (int64_t c = 0; c < C; ++c) {
        float a = bf16_to_f32(ynew[m * C + c]);
        float b = bf16_to_f32(ylast[m * C + c]);
        t0[c] = fabsf(a - b);
        t1[c] = fabsf(b);
      }
      rp[m * 2 + 0] = orc_pairwise_f32(t0, C);
      rp[m * 2 + 1] = orc_pairwise_f32(t1, C);
    }
    free(t0);
    free(t1);
  }
  double* col = (double*)malloc((size_t)(M > 0 ? M : 1) * sizeof(double));
  double S[2];
  for (int s = 0; s < 2; ++s) {
    for (int64_t m = 0; m < M; ++m) col[m] = (double)rp[m * 2 + s];
    S[s] = orc_pairwise_f64(col, M);
  }
  free(col);
  free(rp);
  if (out) {
    out[0] = S[0];
    out[1] = S[1];
  }
  return (S[1] == 0.0) ? INFINITY : S[0] / S[1];
}

/* R-REUSE ([VU] 二: a skipped module reuses the cached result; [GS] 3: the old outcome is used
 * and adjusted very slightly; [VU] 七: the cache holds historical results). At a computed step
 * the module's residual is kept, D = bf16(y - x); at a skipped step y = bf16(x + D). n elements,
 * all bf16 bit patterns. */
void orc_tdc_refresh(const uint16_t* x, const uint16_t* y, int64_t n, uint16_t* d) {
  for (int64_t i = 0; i < n; ++i) d[i] = orc_f32_to_bf16(bf16_to_f32(y[i]) - bf16_to_f32(x[i]));
}

void orc_tdc_reuse(const uint16_t* x, const uint16_t* d, int64_t n, uint16_t* y) {
  for (int64_t i = 0; i < n; ++i) y[i] = orc_f32_to_bf16(bf16_to_f32(x[i]) + bf16_to_f32(d[i]));
}

/* R-REUSE-FP8 ([VU] 七: the cache's historical results may be kept in low-precision formats):
 * the residual of a computed step kept in FP8, one E4M3 code per element and one FP32 scale per
 * row (token), with the per-token recipe of R-DQ-FP8: d = RN(y - x) in FP32 from the bf16 values,
 * a = max |d| over the row, s = a / 448, codes E4M3(RN(d * (448 / a))) (round to nearest even,
 * saturating); a = 0 gives s = 0 and zero codes; 448 / a overflowing gives +-448 (0x7e) for every
 * nonzero d and 0 for zeros. At a skipped step y = bf16(x + dec) with dec = RN(E4M3(code) * s).
 * x, y: bf16 [M][C]; codes [M][C]; scale [M]. */
void orc_tdc_refresh_fp8(const uint16_t* x, const uint16_t* y, int64_t M, int64_t C, uint8_t* codes,
                         float* scale) {
#pragma omp parallel
  {
    float* d = (float*)malloc((size_t)C * sizeof(float));
#pragma omp for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
      float a = 0.0f;
      for (int64_t c = 0; c < C; ++c) {
        d[c] = bf16_to_f32(y[m * C + c]) - bf16_to_f32(x[m * C + c]);
        if (fabsf(d[c]) > a) a = fabsf(d[c]);
      }
      const float s = (a == 0.0f) ? 0.0f : a / 448.0f;
      const float inv = (a == 0.0f) ? 0.0f : 448.0f / a;
      scale[m] = s;
      for (int64_t c = 0; c < C; ++c) {
        uint8_t q;
        if (a == 0.0f) q = 0;
        else if (!(inv <= FLT_MAX)) q = (d[c] == 0.0f) ? 0 : (uint8_t)((d[c] < 0.0f ? 0x80 : 0) | 0x7e);
        else q = orc_e4m3_encode(d[c] * inv);
        codes[m * C + c] = q;
      }
    }
    free(d);
  }
}

void orc_tdc_reuse_fp8(const uint16_t* x, const uint8_t* codes, const float* scale, int64_t M, int64_t C,
                       uint16_t* y) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t c = 0; c < C; ++c) {
      const float dec = orc_e4m3_decode(codes[m * C + c]) * scale[m];
      y[m * C + c] = orc_f32_to_bf16(bf16_to_f32(x[m * C + c]) + dec);
    }
}

/* Per-module state of the Temporal Delta Cache and of the precision rule. */
typedef struct {
  double prev_d; /* d of the last computed step */
  double acc;    /* accumulated delta since the last computed step */
  double delta;  /* delta between the last two computed outputs */
  int32_t have_d;       /* prev_d belongs to the step just before this one */
  int32_t n_out;        /* computed outputs so far */
  int32_t last_skipped; /* the previous step was skipped */
  int32_t skip;         /* decision of the current step */
} orc_state;

void orc_state_init(orc_state* s) { memset(s, 0, sizeof(*s)); }

/* [VU] section 二: the first two steps are computed (two outputs are needed for delta); later,
 * acc += delta and the module is skipped while acc <= threshold. A skipped step leaves no
 * difference statistic for the next one ([VU] section 三), so have_d is cleared. */
void orc_tdc_step(orc_state* s, double thr) {
  if (s->n_out < 2) {
    s->skip = 0;
  } else {
    s->acc = s->acc + s->delta;
    s->skip = (s->acc <= thr) ? 1 : 0;
  }
  if (s->skip) {
    s->have_d = 0;
    s->last_skipped = 1;
  }
}

/* [VU] sections 一 and 三, [GS] section 2: INT8 when the rule says the module is changing
 * (a * d + b > tau), NVFP4 otherwise; INT8 when no difference of the previous step exists
 * (first step, or restart after skips). force >= 0 overrides (benchmarks). */
int orc_select_precision(const orc_state* s, double a, double b, double tau, int force) {
  if (s->skip) return ORC_SKIP;
  if (force >= 0) return force;
  if (!s->have_d) return ORC_INT8;
  double v = a * s->prev_d;
  v = v + b;
  return (v > tau) ? ORC_INT8 : ORC_NVFP4;
}

/* [VU] section 三: a quantized layer whose input outlier ratio exceeds rho computes in full
 * precision (BF16 here) so that what enters the cache is not quantized. */
int orc_apply_pdr(int prec, double ratio, double rho, int force) {
  if (force >= 0) return prec;
  if ((prec == ORC_NVFP4 || prec == ORC_INT8) && ratio > rho) return ORC_BF16;
  return prec;
}

/* A computed step: store delta (when two outputs exist), d (when measured), reset acc. */
void orc_tdc_record(orc_state* s, int have_delta, double delta, int have_d, double d) {
  if (s->skip) return;
  if (have_delta) s->delta = delta;
  s->n_out += 1;
  s->acc = 0.0;
  s->last_skipped = 0;
  if (have_d) {
    s->prev_d = d;
    s->have_d = 1;
  } else {
    s->have_d = 0;
  }
}

/* ------------------------------------------------------------------------------------------ */
/* Delta tokens ("DeltaQuant: 4-bit Video Diffusion Models with Spatiotemporal Delta          */
/* Smoothing", abstract): the activations of the latent video grid are grouped into local 3D   */
/* spatiotemporal cubes; each cube's mean token is its core token, kept in FP8; only the      */
/* differences of the cube's tokens from it (delta tokens) go through the 4-bit path.          */
/*   R-DQ-CUBE  tokens [0, T) are text tokens, one cube each; token T + (f H + h) W + w is the */
/*              grid position (f, h, w) of an F x H x W grid, in cube (f / ct, h / ch, w / cw) */
/*              (edge cubes are smaller). Cubes are numbered text first, then grid cubes in    */
/*              (f, h, w) order of their first position.                                        */
/*   R-DQ-MEAN  the core before FP8, per channel: the pairwise FP32 sum over the cube's tokens */
/*              in index order (zero-padded to a power of two), divided by the token count.    */
/*   R-DQ-FP8   per core token: a = max |mean| over its channels, inv = 448 / a, s = a / 448   */
/*              (FP32); codes E4M3(RN(mean * inv)); dec = E4M3 value * s. a = 0 gives s = 0 and */
/*              zero codes; when 448 / a overflows, nonzero means take +-448 and zeros 0.      */
/*   R-DQ-DELTA delta token = bf16(x - dec of its cube's core): the FP32 difference of the     */
/*              bf16 input and the FP32 core, rounded to nearest even, so the delta tensor is  */
/*              an ordinary bf16 activation for the 4-bit path (rotation, NVFP4, GEMM).        */
/*   R-DQ-GEMM  Y = GEMM(delta) + bf16(dec) W^T + bias (then the optional GELU): the core      */
/*              product is computed once per cube, on the dequantized core rounded to bf16 (the */
/*              operand format of the full-precision tensor path; the page keeps cores in FP8   */
/*              but names no FP8 weight format), and added to each of the cube's tokens.        */
/* ------------------------------------------------------------------------------------------ */

static int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }

/* Number of cubes, or -1 when M != T + F H W or a size is not positive (T may be 0). */
int64_t orc_cube_count(int64_t M, int64_t T, int64_t F, int64_t H, int64_t W, int64_t ct, int64_t ch,
                       int64_t cw) {
  if (T < 0 || F < 1 || H < 1 || W < 1 || ct < 1 || ch < 1 || cw < 1 || M != T + F * H * W) return -1;
  return T + cdiv64(F, ct) * cdiv64(H, ch) * cdiv64(W, cw);
}

/* Cube of token t (R-DQ-CUBE). */
int64_t orc_cube_of_token(int64_t t, int64_t T, int64_t F, int64_t H, int64_t W, int64_t ct,
                          int64_t ch, int64_t cw) {
  if (t < T) return t;
  int64_t g = t - T;
  int64_t f = g / (H * W), h = (g / W) % H, w = g % W;
  return T + ((f / ct) * cdiv64(H, ch) + h / ch) * cdiv64(W, cw) + w / cw;
}

/* The tokens of cube k in index order; returns their count (at most ct ch cw). */
int64_t orc_cube_tokens(int64_t k, int64_t T, int64_t F, int64_t H, int64_t W, int64_t ct,
                        int64_t ch, int64_t cw, int64_t* tok) {
  if (k < T) {
    tok[0] = k;
    return 1;
  }
  int64_t g = k - T;
  int64_t nh = cdiv64(H, ch), nw = cdiv64(W, cw);
  int64_t a = g / (nh * nw), b = (g / nw) % nh, c = g % nw;
  int64_t n = 0;
  for (int64_t f = a * ct; f < F && f < (a + 1) * ct; ++f)
    for (int64_t h = b * ch; h < H && h < (b + 1) * ch; ++h)
      for (int64_t w = c * cw; w < W && w < (c + 1) * cw; ++w) tok[n++] = T + (f * H + h) * W + w;
  return n;
}

/* R-DQ-MEAN, R-DQ-FP8, R-DQ-DELTA for every cube of X [M][K] (bf16):
 * codes [ncube][K] E4M3, scale [ncube] (s), dec [ncube][K] FP32, delta [M][K] bf16. */
void orc_delta_split(const uint16_t* X, int64_t M, int64_t K, int64_t T, int64_t F, int64_t H,
                     int64_t W, int64_t ct, int64_t ch, int64_t cw, uint8_t* codes, float* scale,
                     float* dec, uint16_t* delta) {
  int64_t ncube = orc_cube_count(M, T, F, H, W, ct, ch, cw);
  if (ncube < 0) return;
#pragma omp parallel
  {
    int64_t* tok = (int64_t*)malloc((size_t)(ct * ch * cw) * sizeof(int64_t));
    float* col = (float*)malloc((size_t)(ct * ch * cw) * sizeof(float));
    float* mean = (float*)malloc((size_t)K * sizeof(float));
#pragma omp for schedule(static)
    for (int64_t k = 0; k < ncube; ++k) {
      int64_t n = orc_cube_tokens(k, T, F, H, W, ct, ch, cw, tok);
      float a = 0.0f;
      for (int64_t c = 0; c < K; ++c) {
        for (int64_t j = 0; j < n; ++j) col[j] = bf16_to_f32(X[tok[j] * K + c]);
        mean[c] = orc_pairwise_f32(col, n) / (float)n;
        float m = fabsf(mean[c]);
        if (m > a) a = m;
      }
      float s = (a == 0.0f) ? 0.0f : a / 448.0f;
      float inv = (a == 0.0f) ? 0.0f : 448.0f / a;
      scale[k] = s;
      for (int64_t c = 0; c < K; ++c) {
        uint8_t q;
        if (a == 0.0f) q = 0;
        else if (!(inv <= FLT_MAX)) q = (mean[c] == 0.0f) ? 0 : (uint8_t)((mean[c] < 0.0f ? 0x80 : 0) | 0x7e);
        else q = orc_e4m3_encode(mean[c] * inv);
        codes[k * K + c] = q;
        dec[k * K + c] = orc_e4m3_decode(q) * s;
      }
      for (int64_t j = 0; j < n; ++j)
        for (int64_t c = 0; c < K; ++c)
          delta[tok[j] * K + c] = orc_f32_to_bf16(bf16_to_f32(X[tok[j] * K + c]) - dec[k * K + c]);
    }
    free(tok);
    free(col);
    free(mean);
  }
}

/* R-DQ-GEMM for the token rows `rows`: Y[r][n] = Yd[r][n] + sum_k bf16(dec[cube(m)][k]) w[n][k]
 * + bias[n] (optional GELU), FP64; Yd: the delta GEMM's rows without bias or GELU (FP64). */
void orc_delta_linear(const double* Yd, const float* dec, const uint16_t* Wt, const uint16_t* bias,
                      int64_t M, int64_t N, int64_t K, int64_t T, int64_t F, int64_t H, int64_t W,
                      int64_t ct, int64_t ch, int64_t cw, int gelu, const int64_t* rows, int64_t nrows,
                      double* Y) {
  (void)M;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t cube = orc_cube_of_token(rows[r], T, F, H, W, ct, ch, cw);
    const float* d = dec + cube * K;
    for (int64_t n = 0; n < N; ++n) {
      double s = 0.0;
      for (int64_t k = 0; k < K; ++k)
        s += (double)bf16_to_f32(orc_f32_to_bf16(d[k])) * (double)bf16_to_f32(Wt[n * K + k]);
      double v = Yd[r * N + n] + s + bias_at(bias, n);
      Y[r * N + n] = gelu ? orc_gelu_tanh(v) : v;
    }
  }
}
