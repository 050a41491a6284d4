/*
 * lqq_oracle.c -- plain, slow CPU oracle for the block-quantized W4A8 GEMM
 * (LiquidQuant "LQQ" weights, per-token INT8 activations, INT32 GEMM, FP64
 * epilogue to bf16).
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library under bit_block_quantized_w4a8_b200/csrc) never calls
 * it, and the two share no source, header, table or helper.
 *
 * Source of the method: the review page "LiquidGEMM" (pith.science verdict
 * on arXiv 2509.01229).  Citations below name the field of that page and
 * the paper section / equation the field discusses:
 *   key_machinery   -- the dequantization identity (q_u4 * s_u8 + a) XOR 0x80
 *                      with a = 2^7 + min(Q_i8), precomputed offline.
 *   referee major 3 -- paper Sec. 4, Eq. (7): protective range [-119, 119],
 *                      s_u8 <= 16 from (119 - (-119)) / 15, s_u8 an integer.
 *   referee minor 2 -- paper Sec. 4, Eq. (10): UINT4 codes are q_u8 / s_u8
 *                      rounded to the nearest integer.
 *   referee summary -- shift INT8 weights into UINT8 before quantizing to
 *                      UINT4; dequantization stays inside UINT8.
 *   skeptic concrete_test -- default group size 64.
 *   supporting_citations [29] -- per-token INT8 activations (SmoothQuant).
 *
 * Readings taken where the page leaves a step open (each is listed, with its
 * reason, in the design notes of the repository):
 *   R1 s_u8 = ceil((max - min) / 15), at least 1 ("ceil" rule).  The
 *      alternative "round" rule (round half up, codes clamped to 15) is kept
 *      selectable so that the overflow sweep can check both.
 *   R2 Q_u4 = floor((2 (q - min) + s) / (2 s)): round to nearest, ties up.
 *   R3 FP -> INT8 steps divide in IEEE fp32 (x / s, no reciprocal) and round
 *      half to even (nearbyintf under the default rounding mode).
 *   R4 weight level 1: s_w = absmax / 119, Q_i8 = clamp(rint(W / s_w), +-119);
 *      activations: s_x = absmax / 127, Q = clamp(rint(X / s_x), +-127).
 *      An all-zero row has scale 0 and all-zero codes.
 *   R5 groups run along K inside one output channel: k in [g*G, g*G + G).
 *   R6 epilogue: y = s_x[m] * s_w[n] * acc[m][n] in FP64, rounded once to
 *      bf16 (round to nearest, ties to even).
 *
 * Build: gcc -O2 -std=c11 -fopenmp -ffp-contract=off -shared -fPIC.
 * The OpenMP loops only split independent output rows across threads; no
 * arithmetic is reordered.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define LQQ_W_RANGE 119 /* protective range, referee major 3 (Sec. 4, Eq. 7) */
#define LQQ_X_RANGE 127 /* symmetric INT8 activations (reading R4) */

enum { LQQ_RULE_CEIL = 0, LQQ_RULE_ROUND = 1 };

int lqq_oracle_version(void) { return 1; }

int lqq_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ---- level 1: per-row symmetric INT8 (weights: per output channel,
 *      activations: per token).  Readings R3, R4. ---------------------- */
static void quantize_rows_sym(const float* X, int64_t rows, int64_t cols,
                              int range, int8_t* Q, float* scale) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const float* x = X + r * cols;
    float amax = 0.0f;
    for (int64_t c = 0; c < cols; ++c) {
      float v = fabsf(x[c]);
      if (v > amax) amax = v;
    }
    float s = amax / (float)range;
    scale[r] = s;
    int8_t* q = Q + r * cols;
    for (int64_t c = 0; c < cols; ++c) {
      if (s == 0.0f) {
        q[c] = 0;
        continue;
      }
      float t = nearbyintf(x[c] / s);
      if (t > (float)range) t = (float)range;
      if (t < -(float)range) t = -(float)range;
      q[c] = (int8_t)t;
    }
  }
}

void lqq_quantize_act(const float* X, int64_t M, int64_t K, int8_t* Xq,
                      float* s_x) {
  quantize_rows_sym(X, M, K, LQQ_X_RANGE, Xq, s_x);
}

void lqq_quantize_weights_i8(const float* W, int64_t N, int64_t K,
                             int8_t* Qi8, float* s_w) {
  quantize_rows_sym(W, N, K, LQQ_W_RANGE, Qi8, s_w);
}

/* ---- level 2: per group, shift by the minimum into UINT8 and quantize to
 *      UINT4 with an integer scale.  Referee summary; referee major 3
 *      (Sec. 4, Eq. 7); referee minor 2 (Sec. 4, Eq. 10); key_machinery. -- */

/* Integer group scale s_u8 from the group's min and max of Q_i8 (R1). */
int lqq_group_scale(int mn, int mx, int rule) {
  int d = mx - mn; /* the group's range in the UINT8 domain, q_u8 max */
  int s;
  if (rule == LQQ_RULE_ROUND)
    s = (2 * d + 15) / 30; /* round(d / 15), ties up */
  else
    s = (d + 14) / 15; /* ceil(d / 15) */
  return s < 1 ? 1 : s;
}

/* UINT4 code of one INT8 weight q in a group with minimum mn and scale s
 * (R2): q_u8 = q - mn, code = round(q_u8 / s), ties up. */
int lqq_group_code(int q, int mn, int s, int rule) {
  int u = q - mn;
  int c = (2 * u + s) / (2 * s);
  if (rule == LQQ_RULE_ROUND && c > 15) c = 15;
  return c;
}

/* Offset a = 2^7 + min(Q_i8) (key_machinery). */
int lqq_group_offset(int mn) { return 128 + mn; }

/* Canonical (unpacked) LQQ weights: codes[N*K] one code per byte,
 * s_u8[N*G], a[N*G] with G = K / group. */
void lqq_quantize_weights_u4(const int8_t* Qi8, int64_t N, int64_t K,
                             int group, int rule, uint8_t* codes,
                             uint8_t* s_u8, uint8_t* a) {
  int64_t G = K / group;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < G; ++g) {
      const int8_t* q = Qi8 + n * K + g * group;
      int mn = q[0], mx = q[0];
      for (int i = 1; i < group; ++i) {
        if (q[i] < mn) mn = q[i];
        if (q[i] > mx) mx = q[i];
      }
      int s = lqq_group_scale(mn, mx, rule);
      s_u8[n * G + g] = (uint8_t)s;
      a[n * G + g] = (uint8_t)lqq_group_offset(mn);
      uint8_t* c = codes + n * K + g * group;
      for (int i = 0; i < group; ++i)
        c[i] = (uint8_t)lqq_group_code(q[i], mn, s, rule);
    }
  }
}

/* Both levels.  Qi8 may be NULL (the INT8 weights are then not returned). */
int lqq_quantize_weights(const float* W, int64_t N, int64_t K, int group,
                         int rule, int8_t* Qi8, float* s_w, uint8_t* codes,
                         uint8_t* s_u8, uint8_t* a) {
  if (group <= 0 || K % group != 0) return -1;
  int8_t* q = Qi8 ? Qi8 : (int8_t*)malloc((size_t)(N * K));
  if (!q) return -2;
  lqq_quantize_weights_i8(W, N, K, q, s_w);
  lqq_quantize_weights_u4(q, N, K, group, rule, codes, s_u8, a);
  if (!Qi8) free(q);
  return 0;
}

/* ---- dequantization ------------------------------------------------- */

/* Plain signed dequantization: Q^_i8 = code * s_u8 + min, with
 * min = a - 128.  This is what the identity of key_machinery computes;
 * it is written here without the XOR so that the two can be compared. */
int lqq_dequant_signed(int code, int s, int a) { return code * s + (a - 128); }

/* The key_machinery identity itself on one byte: (q_u4 * s_u8 + a) XOR 0x80,
 * read back as a two's-complement INT8.  Returns the UINT8 intermediate in
 * *u8 so callers can check it never leaves [0, 255]. */
int lqq_dequant_xor(int code, int s, int a, int* u8) {
  int u = code * s + a;
  if (u8) *u8 = u;
  int b = (u ^ 0x80) & 0xFF;
  return b >= 128 ? b - 256 : b;
}

void lqq_dequant_weights(const uint8_t* codes, const uint8_t* s_u8,
                         const uint8_t* a, int64_t N, int64_t K, int group,
                         int8_t* W8) {
  int64_t G = K / group;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      int64_t g = k / group;
      W8[n * K + k] = (int8_t)lqq_dequant_signed(codes[n * K + k],
                                                 s_u8[n * G + g], a[n * G + g]);
    }
}

/* ---- integer GEMM: acc[m][n] = sum_k Xq[m][k] * W8[n][k] ---------------
 * A textbook triple loop accumulating in int64.  Returns -1 if any result
 * does not fit in int32 (the GPU accumulates in INT32). */
int lqq_gemm_i32(const int8_t* Xq, const int8_t* W8, int64_t M, int64_t N,
                 int64_t K, int32_t* acc) {
  int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
  for (int64_t m = 0; m < M; ++m) {
    const int8_t* x = Xq + m * K;
    for (int64_t n = 0; n < N; ++n) {
      const int8_t* w = W8 + n * K;
      int64_t s = 0;
      for (int64_t k = 0; k < K; ++k) s += (int64_t)x[k] * (int64_t)w[k];
      if (s > INT32_MAX || s < INT32_MIN) bad = 1;
      acc[m * N + n] = (int32_t)s;
    }
  }
  return bad ? -1 : 0;
}

/* ---- bf16 rounding of a double, once, to nearest with ties to even ----
 * bf16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
uint16_t lqq_bf16_from_double(double x) {
  uint16_t sign = 0;
  if (isnan(x)) return 0x7FC0;
  if (signbit(x)) {
    sign = 0x8000;
    x = -x;
  }
  if (x == 0.0) return sign;
  if (isinf(x)) return (uint16_t)(sign | 0x7F80);
  int e;
  double f = frexp(x, &e); /* x = f * 2^e, f in [0.5, 1) */
  /* normal bf16 values are r * 2^(e - 8) with r in [128, 256) */
  if (e - 1 >= -126) {
    double r = nearbyint(ldexp(f, 8)); /* exact scaling; RNE to integer */
    if (r >= 256.0) {
      r = 128.0;
      e += 1;
    }
    int ef = e - 1 + 127; /* biased exponent of r/128 * 2^(e-1) */
    if (ef >= 255) return (uint16_t)(sign | 0x7F80);
    return (uint16_t)(sign | (ef << 7) | ((int)r - 128));
  }
  /* subnormal: x = r * 2^-133, r in [0, 128]; r == 128 is the smallest
   * normal, whose encoding is also 128 */
  double r = nearbyint(ldexp(x, 133));
  return (uint16_t)(sign | (int)r);
}

/* Epilogue (R6): Y[m][n] = bf16(s_x[m] * s_w[n] * acc[m][n]) in FP64. */
void lqq_epilogue_bf16(const int32_t* acc, const float* s_x, const float* s_w,
                       int64_t M, int64_t N, uint16_t* Y) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double y = (double)s_x[m] * (double)s_w[n] * (double)acc[m * N + n];
      Y[m * N + n] = lqq_bf16_from_double(y);
    }
}

/* Whole forward from quantized operands: dequantize (plain signed form),
 * integer GEMM, FP64 epilogue.  acc may be NULL. */
int lqq_w4a8_gemm(const int8_t* Xq, const float* s_x, const uint8_t* codes,
                  const uint8_t* s_u8, const uint8_t* a, const float* s_w,
                  int64_t M, int64_t N, int64_t K, int group, int32_t* acc,
                  uint16_t* Y) {
  int8_t* W8 = (int8_t*)malloc((size_t)(N * K));
  int32_t* A = acc ? acc : (int32_t*)malloc((size_t)(M * N) * sizeof(int32_t));
  if (!W8 || !A) {
    free(W8);
    if (!acc) free(A);
    return -2;
  }
  lqq_dequant_weights(codes, s_u8, a, N, K, group, W8);
  int rc = lqq_gemm_i32(Xq, W8, M, N, K, A);
  if (Y) lqq_epilogue_bf16(A, s_x, s_w, M, N, Y);
  free(W8);
  if (!acc) free(A);
  return rc;
}

/* Selected outputs only, computed one by one straight from the codes
 * (for full-size checks where the whole product is too slow on the CPU). */
int lqq_w4a8_gemm_sampled(const int8_t* Xq, const float* s_x,
                          const uint8_t* codes, const uint8_t* s_u8,
                          const uint8_t* a, const float* s_w, int64_t M,
                          int64_t N, int64_t K, int group, const int64_t* ms,
                          const int64_t* ns, int64_t count, int32_t* acc,
                          uint16_t* Y) {
  int64_t G = K / group;
  int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
  for (int64_t i = 0; i < count; ++i) {
    int64_t m = ms[i], n = ns[i];
    if (m < 0 || m >= M || n < 0 || n >= N) {
      bad = 1;
      continue;
    }
    int64_t s = 0;
    for (int64_t k = 0; k < K; ++k) {
      int64_t g = k / group;
      int w = lqq_dequant_signed(codes[n * K + k], s_u8[n * G + g],
                                 a[n * G + g]);
      s += (int64_t)Xq[m * K + k] * (int64_t)w;
    }
    if (s > INT32_MAX || s < INT32_MIN) bad = 1;
    acc[i] = (int32_t)s;
    if (Y)
      Y[i] = lqq_bf16_from_double((double)s_x[m] * (double)s_w[n] * (double)s);
  }
  return bad ? -1 : 0;
}
