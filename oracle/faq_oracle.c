/*
 * faq_oracle.c -- the oracle for FA quantization (see faq_oracle.h).
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the tests, the smoke check and the
 * benchmark's CPU-baseline leg, never by the product path.  Plain C99 with
 * fp64 arithmetic wherever the method leaves the precision open; the fp32
 * steps (scale = amax / qmax and x / scale) are the ones the pages' scale
 * definitions imply and are written as single IEEE fp32 divisions.  Build
 * without -ffast-math (oracle/build.py does).
 *
 * Each codec works from the number format's definition: find the spacing of
 * the representable values around |v|, round |v| to a multiple of that
 * spacing with round-half-to-even (C99 rint in the default rounding mode),
 * saturate, then pack the fields.  The tests pin every codec against a
 * brute-force nearest-value search over all codes and against ml_dtypes.
 */
#include "faq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Flat index of element (b, h, s, d) in the data layout ([SD] 注意事项). */
static size_t elem_index(int layout, int H, int S, int D, int b, int h, int s,
                         int d) {
  if (layout == ORC_LAYOUT_BNSD) return (((size_t)b * H + h) * S + s) * D + d;
  return (((size_t)b * S + s) * H + h) * D + d;
}

/* Index of the token row (b, h, s) in the data layout (rows of packed codes). */
static size_t row_index(int layout, int H, int S, int b, int h, int s) {
  if (layout == ORC_LAYOUT_BNSD) return ((size_t)b * H + h) * S + s;
  return ((size_t)b * S + s) * H + h;
}

/* ------------------------------------------------------------------------ */
/* Scalar codecs                                                             */
/* ------------------------------------------------------------------------ */

float orc_bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* bf16: 1 sign, 8 exponent bits (bias 127), 7 stored mantissa bits. */
uint16_t orc_f64_to_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  const int neg = signbit(x) ? 1 : 0;
  const double a = fabs(x);
  double quantum;
  if (a < 0x1p-126) {
    quantum = 0x1p-133; /* subnormal spacing 2^-126 * 2^-7 */
  } else {
    int e;
    frexp(a, &e);                /* a in [2^(e-1), 2^e) */
    quantum = ldexp(1.0, e - 8); /* 8 significant bits */
  }
  const double r = rint(a / quantum) * quantum;
  uint16_t bits;
  if (r >= 0x1p128) {
    bits = 0x7F80; /* rounded past the largest finite value: infinity */
  } else {
    const float f = (float)r; /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    bits = (uint16_t)(u >> 16);
  }
  return (uint16_t)(bits | (neg ? 0x8000u : 0u));
}

/* float8_e4m3fn ([FA] 组合2: E4M3, max 448): 1 sign, 4 exponent bits with
 * bias 7, 3 mantissa bits; no infinity; S.1111.111 is NaN; largest finite
 * 1.75 * 2^8 = 448; smallest normal 2^-6; subnormal spacing 2^-9.
 * Saturating: every finite |v| above 448 encodes as 448. */
uint8_t orc_e4m3_encode(float v) {
  if (isnan(v)) return 0x7F;
  const int neg = signbit(v) ? 1 : 0;
  double a = fabs((double)v);
  if (isinf(a)) a = 448.0;
  double quantum;
  if (a < 0x1p-6) {
    quantum = 0x1p-9;
  } else {
    int e;
    frexp(a, &e);                /* a in [2^(e-1), 2^e) */
    quantum = ldexp(1.0, e - 4); /* 4 significant bits */
  }
  double r = rint(a / quantum) * quantum;
  if (r > 448.0) r = 448.0;
  uint8_t code;
  if (r < 0x1p-6) {
    code = (uint8_t)(r / 0x1p-9); /* exponent field 0, mantissa r / 2^-9 */
  } else {
    int e;
    const double m = frexp(r, &e); /* r = m 2^e, m in [0.5, 1) */
    const int E = e - 1;           /* r = 1.mmm * 2^E */
    const int mant = (int)(m * 16.0) - 8;
    code = (uint8_t)(((E + 7) << 3) | mant);
  }
  return (uint8_t)(code | (neg ? 0x80u : 0u));
}

double orc_e4m3_decode(uint8_t c) {
  const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  double val;
  if (e == 15 && m == 7)
    val = NAN;
  else if (e == 0)
    val = ldexp((double)m, -9); /* 0.mmm * 2^-6 */
  else
    val = ldexp((double)(8 + m), e - 7 - 3); /* 1.mmm * 2^(e-7) */
  return s ? -val : val;
}

/* E2M1 ([FA] 组合3: emax 2, max 6): 1 sign, 2 exponent bits with bias 1,
 * 1 mantissa bit.  Magnitudes by code 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6.
 * Spacing 0.5 below 2, 1 in [2, 4), 2 in [4, 8); saturating at 6. */
uint8_t orc_e2m1_encode(float v) {
  static const double grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  const int neg = signbit(v) ? 1 : 0;
  double a = fabs((double)v);
  if (isnan(a) || isinf(a)) a = 6.0;
  double quantum;
  if (a < 2.0)
    quantum = 0.5;
  else if (a < 4.0)
    quantum = 1.0;
  else
    quantum = 2.0;
  double r = rint(a / quantum) * quantum;
  if (r > 6.0) r = 6.0;
  int code = 0;
  for (int i = 0; i < 8; ++i)
    if (grid[i] == r) code = i;
  return (uint8_t)(code | (neg ? 8 : 0));
}

double orc_e2m1_decode(uint8_t c) {
  static const double grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  const double val = grid[c & 7];
  return (c & 8) ? -val : val;
}

/* INT8 symmetric ([SD] Linear 量化 通用原理: [-max, max] -> [-128, 127]):
 * nearest integer, ties to even, clamped to [-128, 127]. */
int8_t orc_int8_encode(float v) {
  if (isnan(v)) return 0;
  double r = rint((double)v);
  if (r > 127.0) r = 127.0;
  if (r < -128.0) r = -128.0;
  return (int8_t)r;
}

/* MX shared exponent ([FA] 组合3): the OCP-MX rule floor(log2 amax) - emax
 * with emax = 2, read exactly from the binary exponent, clamped to the E8M0
 * range [-127, 127].  amax == 0 gives -127 (E8M0 byte 0). */
int orc_mx_exponent(float amax) {
  if (!(amax > 0.0f)) return -127;
  int e;
  frexp((double)amax, &e); /* amax in [2^(e-1), 2^e): floor(log2) = e - 1 */
  int x = (e - 1) - 2;
  if (x < -127) x = -127;
  if (x > 127) x = 127;
  return x;
}

/* The same rule for E4M3 elements ([FA] 模式清单, FA PerBlock with MXFP8):
 * floor(log2 amax) - 8, E4M3's largest exponent (max 448 = 1.75 * 2^8). */
int orc_mx_exponent_e4m3(float amax) {
  if (!(amax > 0.0f)) return -127;
  int e;
  frexp((double)amax, &e);
  int x = (e - 1) - 8;
  if (x < -127) x = -127;
  if (x > 127) x = 127;
  return x;
}

/* ------------------------------------------------------------------------ */
/* Quantizers                                                                */
/* ------------------------------------------------------------------------ */

/* [FA] 组合1: static per-head minmax calibration -- the running maximum of
 * |x| over every (b, s, d) of head h. */
void orc_calibrate_per_head(const uint16_t* x, int B, int H, int S, int D,
                            int layout, float* amax) {
  for (int h = 0; h < H; ++h) {
    float m = amax[h];
    for (int b = 0; b < B; ++b)
      for (int s = 0; s < S; ++s)
        for (int d = 0; d < D; ++d) {
          const float a = fabsf(orc_bf16_to_f32(x[elem_index(layout, H, S, D, b, h, s, d)]));
          if (a > m) m = a;
        }
    amax[h] = m;
  }
}

/* [FA] 组合1: scale s_h = amax_h / 127 (one per head, symmetric, no offset);
 * code = int8(x / s_h).  A zero scale gives code 0. */
void orc_quantize_int8_per_head(const uint16_t* x, int B, int H, int S, int D,
                                int layout, const float* amax, int8_t* codes,
                                float* scales) {
  for (int h = 0; h < H; ++h) {
    const float sh = amax[h] / 127.0f;
    scales[h] = sh;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
      for (int s = 0; s < S; ++s)
        for (int d = 0; d < D; ++d) {
          const size_t i = elem_index(layout, H, S, D, b, h, s, d);
          const float xf = orc_bf16_to_f32(x[i]);
          codes[i] = (sh > 0.0f) ? orc_int8_encode(xf / sh) : (int8_t)0;
        }
  }
}

/* [FA] 组合2: per (b, h, token) amax over D, scale = amax / 448,
 * code = e4m3(x / scale).  A zero scale gives code 0x00. */
void orc_quantize_fp8_per_token(const uint16_t* x, int B, int H, int S, int D,
                                int layout, uint8_t* codes, float* scales) {
#pragma omp parallel for collapse(3) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int s = 0; s < S; ++s) {
        float amax = 0.0f;
        for (int d = 0; d < D; ++d) {
          const float a = fabsf(orc_bf16_to_f32(x[elem_index(layout, H, S, D, b, h, s, d)]));
          if (a > amax) amax = a;
        }
        const float sc = amax / 448.0f;
        scales[((size_t)b * H + h) * S + s] = sc;
        for (int d = 0; d < D; ++d) {
          const size_t i = elem_index(layout, H, S, D, b, h, s, d);
          const float xf = orc_bf16_to_f32(x[i]);
          codes[i] = (sc > 0.0f) ? orc_e4m3_encode(xf / sc) : (uint8_t)0;
        }
      }
}

/* [FA] 模式清单, FA PerHead with FP8: 组合1's static per-head calibration with
 * the E4M3 range, s_h = amax_h / 448, code = e4m3(x / s_h) (values beyond the
 * calibrated range saturate to +-448).  A zero scale gives code 0x00. */
void orc_quantize_fp8_per_head(const uint16_t* x, int B, int H, int S, int D,
                               int layout, const float* amax, uint8_t* codes,
                               float* scales) {
  for (int h = 0; h < H; ++h) {
    const float sh = amax[h] / 448.0f;
    scales[h] = sh;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
      for (int s = 0; s < S; ++s)
        for (int d = 0; d < D; ++d) {
          const size_t i = elem_index(layout, H, S, D, b, h, s, d);
          const float xf = orc_bf16_to_f32(x[i]);
          codes[i] = (sh > 0.0f) ? orc_e4m3_encode(xf / sh) : (uint8_t)0;
        }
  }
}

/* [FA] 模式清单, FA PerToken with INT8: 组合2's dynamic per-token amax with the
 * INT8 range, s = amax / 127 per (b, h, token), code = int8(x / s).  A zero
 * scale gives code 0. */
void orc_quantize_int8_per_token(const uint16_t* x, int B, int H, int S, int D,
                                 int layout, int8_t* codes, float* scales) {
#pragma omp parallel for collapse(3) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int s = 0; s < S; ++s) {
        float amax = 0.0f;
        for (int d = 0; d < D; ++d) {
          const float a = fabsf(orc_bf16_to_f32(x[elem_index(layout, H, S, D, b, h, s, d)]));
          if (a > amax) amax = a;
        }
        const float sc = amax / 127.0f;
        scales[((size_t)b * H + h) * S + s] = sc;
        for (int d = 0; d < D; ++d) {
          const size_t i = elem_index(layout, H, S, D, b, h, s, d);
          const float xf = orc_bf16_to_f32(x[i]);
          codes[i] = (sc > 0.0f) ? orc_int8_encode(xf / sc) : (int8_t)0;
        }
      }
}

/* [FA] 组合3: blocks of 32 consecutive elements along head_dim share one
 * E8M0 exponent X = 2^e, e = floor(log2 amax) - 2; values are E2M1 of x / X. */
void orc_quantize_mxfp4(const uint16_t* x, int B, int H, int S, int D,
                        int layout, uint8_t* codes, uint8_t* e8m0) {
  const int G = D / 32;
#pragma omp parallel for collapse(3) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int s = 0; s < S; ++s) {
        const size_t row = row_index(layout, H, S, b, h, s);
        for (int g = 0; g < G; ++g) {
          float amax = 0.0f;
          for (int j = 0; j < 32; ++j) {
            const float a = fabsf(orc_bf16_to_f32(x[elem_index(layout, H, S, D, b, h, s, g * 32 + j)]));
            if (a > amax) amax = a;
          }
          const int e = orc_mx_exponent(amax);
          e8m0[(((size_t)b * H + h) * S + s) * G + g] = (uint8_t)(e + 127);
          const float X = ldexpf(1.0f, e);
          for (int j = 0; j < 32; j += 2) {
            const int d = g * 32 + j;
            const uint8_t lo = orc_e2m1_encode(orc_bf16_to_f32(x[elem_index(layout, H, S, D, b, h, s, d)]) / X);
            const uint8_t hi = orc_e2m1_encode(orc_bf16_to_f32(x[elem_index(layout, H, S, D, b, h, s, d + 1)]) / X);
            codes[row * (size_t)(D / 2) + d / 2] = (uint8_t)(lo | (hi << 4));
          }
        }
      }
}

/* [SD] FA量化 旋转: x' = x * R (R applied on the right, [D, D] row-major),
 * summed in fp64. */
void orc_rotate_f64(const uint16_t* x, int B, int H, int S, int D, int layout,
                    const uint16_t* R, double* out) {
#pragma omp parallel for collapse(3) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int s = 0; s < S; ++s)
        for (int j = 0; j < D; ++j) {
          double acc = 0.0;
          for (int d = 0; d < D; ++d)
            acc += (double)orc_bf16_to_f32(x[elem_index(layout, H, S, D, b, h, s, d)]) *
                   (double)orc_bf16_to_f32(R[(size_t)d * D + j]);
          out[elem_index(layout, H, S, D, b, h, s, j)] = acc;
        }
}

/* The rotated operand stays in the input precision (bf16), rounded once,
 * before the block quantization step that follows it. */
void orc_rotate(const uint16_t* x, int B, int H, int S, int D, int layout,
                const uint16_t* R, uint16_t* out) {
  const size_t n = (size_t)B * H * S * D;
  double* tmp = (double*)malloc(n * sizeof(double));
  if (!tmp) return;
  orc_rotate_f64(x, B, H, S, D, layout, R, tmp);
#pragma omp parallel for schedule(static)
  for (size_t i = 0; i < n; ++i) out[i] = orc_f64_to_bf16(tmp[i]);
  free(tmp);
}

/* [SD] FA量化 块量化: one E4M3 scale = amax / 448 per (b, h, block of `blk`
 * consecutive tokens) over all of D; a last partial block uses its own
 * amax. */
void orc_quantize_fp8_block(const uint16_t* x, int B, int H, int S, int D,
                            int layout, int blk, uint8_t* codes,
                            float* scales) {
  const int nblk = (S + blk - 1) / blk;
#pragma omp parallel for collapse(3) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int g = 0; g < nblk; ++g) {
        const int s0 = g * blk;
        const int s1 = (s0 + blk < S) ? s0 + blk : S;
        float amax = 0.0f;
        for (int s = s0; s < s1; ++s)
          for (int d = 0; d < D; ++d) {
            const float a = fabsf(orc_bf16_to_f32(x[elem_index(layout, H, S, D, b, h, s, d)]));
            if (a > amax) amax = a;
          }
        const float sc = amax / 448.0f;
        scales[((size_t)b * H + h) * nblk + g] = sc;
        for (int s = s0; s < s1; ++s)
          for (int d = 0; d < D; ++d) {
            const size_t i = elem_index(layout, H, S, D, b, h, s, d);
            const float xf = orc_bf16_to_f32(x[i]);
            codes[i] = (sc > 0.0f) ? orc_e4m3_encode(xf / sc) : (uint8_t)0;
          }
      }
}

/* [FA] 模式清单, FA PerBlock with MXFP8: as 组合3, 32 consecutive elements of
 * head_dim share X = 2^e, e = floor(log2 amax) - 8, with E4M3 elements
 * e4m3(x / X) (x / X < 512; values above 448 saturate). */
void orc_quantize_mxfp8(const uint16_t* x, int B, int H, int S, int D,
                        int layout, uint8_t* codes, uint8_t* e8m0) {
  const int G = D / 32;
#pragma omp parallel for collapse(3) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int s = 0; s < S; ++s)
        for (int g = 0; g < G; ++g) {
          float amax = 0.0f;
          for (int j = 0; j < 32; ++j) {
            const float a = fabsf(orc_bf16_to_f32(x[elem_index(layout, H, S, D, b, h, s, g * 32 + j)]));
            if (a > amax) amax = a;
          }
          const int e = orc_mx_exponent_e4m3(amax);
          e8m0[(((size_t)b * H + h) * S + s) * G + g] = (uint8_t)(e + 127);
          const float X = ldexpf(1.0f, e);
          for (int j = 0; j < 32; ++j) {
            const size_t i = elem_index(layout, H, S, D, b, h, s, g * 32 + j);
            codes[i] = orc_e4m3_encode(orc_bf16_to_f32(x[i]) / X);
          }
        }
}

/* ------------------------------------------------------------------------ */
/* FakeQuant dequantization ([MODE] 模式索引: quantize, then dequantize)      */
/* ------------------------------------------------------------------------ */

double orc_dequant_elem(const orc_qt* t, int b, int h, int s, int d) {
  const size_t i = elem_index(t->layout, t->H, t->S, t->D, b, h, s, d);
  switch (t->mode) {
    case ORC_MODE_FLOAT:
      return (double)orc_bf16_to_f32(((const uint16_t*)t->codes)[i]);
    case ORC_MODE_INT8_PER_HEAD:
      return (double)((const int8_t*)t->codes)[i] * (double)((const float*)t->scales)[h];
    case ORC_MODE_FP8_PER_TOKEN:
      return orc_e4m3_decode(((const uint8_t*)t->codes)[i]) *
             (double)((const float*)t->scales)[((size_t)b * t->H + h) * t->S + s];
    case ORC_MODE_MXFP8: {
      const int G = t->D / 32;
      const int e = (int)((const uint8_t*)t->scales)[(((size_t)b * t->H + h) * t->S + s) * G + d / 32] - 127;
      return ldexp(orc_e4m3_decode(((const uint8_t*)t->codes)[i]), e);
    }
    case ORC_MODE_FP8_PER_HEAD:
      return orc_e4m3_decode(((const uint8_t*)t->codes)[i]) * (double)((const float*)t->scales)[h];
    case ORC_MODE_INT8_PER_TOKEN:
      return (double)((const int8_t*)t->codes)[i] *
             (double)((const float*)t->scales)[((size_t)b * t->H + h) * t->S + s];
    case ORC_MODE_FP8_BLOCK: {
      const int nblk = (t->S + t->blk - 1) / t->blk;
      return orc_e4m3_decode(((const uint8_t*)t->codes)[i]) *
             (double)((const float*)t->scales)[((size_t)b * t->H + h) * nblk + s / t->blk];
    }
    case ORC_MODE_MXFP4: {
      const size_t row = row_index(t->layout, t->H, t->S, b, h, s);
      const uint8_t byte = ((const uint8_t*)t->codes)[row * (size_t)(t->D / 2) + d / 2];
      const uint8_t nib = (d & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
      const int G = t->D / 32;
      const int e = (int)((const uint8_t*)t->scales)[(((size_t)b * t->H + h) * t->S + s) * G + d / 32] - 127;
      return ldexp(orc_e2m1_decode(nib), e);
    }
    default:
      return NAN;
  }
}

void orc_dequant_head(const orc_qt* t, int b, int h, double* out) {
#pragma omp parallel for schedule(static)
  for (int s = 0; s < t->S; ++s)
    for (int d = 0; d < t->D; ++d) out[(size_t)s * t->D + d] = orc_dequant_elem(t, b, h, s, d);
}

/* ------------------------------------------------------------------------ */
/* Attention (FlashAttention's exact result, computed directly)              */
/* ------------------------------------------------------------------------ */

void orc_attention(const orc_qt* q, const orc_qt* k, const orc_qt* v,
                   int causal, double scale, const int* rows, int nrows,
                   double* out, double* lse) {
  const int B = q->B, Hq = q->H, Sq = q->S, D = q->D;
  const int Hkv = k->H, Sk = k->S;
  const int group = Hq / Hkv;
  if (rows == NULL) nrows = Sq;
  if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
  double* kd = (double*)malloc((size_t)Sk * D * sizeof(double));
  double* vd = (double*)malloc((size_t)Sk * D * sizeof(double));
  if (!kd || !vd) {
    free(kd);
    free(vd);
    return;
  }
  for (int b = 0; b < B; ++b)
    for (int hk = 0; hk < Hkv; ++hk) {
      orc_dequant_head(k, b, hk, kd);
      orc_dequant_head(v, b, hk, vd);
#pragma omp parallel
      {
        double* sc = (double*)malloc((size_t)Sk * sizeof(double));
        double* qr = (double*)malloc((size_t)D * sizeof(double));
#pragma omp for collapse(2) schedule(dynamic, 4)
        for (int g = 0; g < group; ++g)
          for (int r = 0; r < nrows; ++r) {
            const int h = hk * group + g;
            const int i = rows ? rows[r] : r;
            double* o = out + (((size_t)b * Hq + h) * nrows + r) * D;
            for (int d = 0; d < D; ++d) qr[d] = orc_dequant_elem(q, b, h, i, d);
            const int last = causal ? i + (Sk - Sq) : Sk - 1; /* last visible key */
            const int nvis = (last + 1 < Sk) ? last + 1 : Sk;
            if (nvis <= 0) {
              for (int d = 0; d < D; ++d) o[d] = 0.0;
              if (lse) lse[((size_t)b * Hq + h) * nrows + r] = -INFINITY;
              continue;
            }
            double m = -INFINITY;
            for (int j = 0; j < nvis; ++j) {
              double acc = 0.0;
              for (int d = 0; d < D; ++d) acc += qr[d] * kd[(size_t)j * D + d];
              sc[j] = acc * scale;
              if (sc[j] > m) m = sc[j];
            }
            double l = 0.0;
            for (int j = 0; j < nvis; ++j) {
              sc[j] = exp(sc[j] - m);
              l += sc[j];
            }
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            for (int j = 0; j < nvis; ++j) {
              const double p = sc[j];
              const double* vr = vd + (size_t)j * D;
              for (int d = 0; d < D; ++d) o[d] += p * vr[d];
            }
            for (int d = 0; d < D; ++d) o[d] /= l;
            if (lse) lse[((size_t)b * Hq + h) * nrows + r] = m + log(l);
          }
        free(sc);
        free(qr);
      }
    }
  free(kd);
  free(vd);
}

/* ------------------------------------------------------------------------ */
/* Array forms of the scalar codecs (for exhaustive tests)                   */
/* ------------------------------------------------------------------------ */

void orc_e4m3_encode_n(const float* v, uint8_t* out, size_t n) {
  for (size_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}
void orc_e2m1_encode_n(const float* v, uint8_t* out, size_t n) {
  for (size_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(v[i]);
}
void orc_int8_encode_n(const float* v, int8_t* out, size_t n) {
  for (size_t i = 0; i < n; ++i) out[i] = orc_int8_encode(v[i]);
}
void orc_mx_exponent_e4m3_n(const float* v, int* out, size_t n) {
  for (size_t i = 0; i < n; ++i) out[i] = orc_mx_exponent_e4m3(v[i]);
}
void orc_mx_exponent_n(const float* v, int* out, size_t n) {
  for (size_t i = 0; i < n; ++i) out[i] = orc_mx_exponent(v[i]);
}
void orc_f64_to_bf16_n(const double* v, uint16_t* out, size_t n) {
  for (size_t i = 0; i < n; ++i) out[i] = orc_f64_to_bf16(v[i]);
}
