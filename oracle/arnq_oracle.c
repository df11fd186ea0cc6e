/*
 * arnq_oracle.c -- plain, slow, obviously-correct CPU oracle for the fused
 * residual-add + RMSNorm + per-row symmetric dynamic quantization operator.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or
 * calls this file; it shares no header, helper, table or constant with the CUDA
 * path.  Only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg load it.
 *
 * What it follows:
 *   [V2]  "aclnnAddRmsNormDynamicQuantV2" (Huawei CANN operator docs),
 *         section "Formula" (x = x1 + x2; Rms; RmsNorm with gamma and beta;
 *         input1/input2 smooth scaling; scale1Out/y1Out/scale2Out/y2Out cases;
 *         row_max = per-row maximum) and section "Constraints" (outputMask /
 *         smoothScale rules, ND format, deterministic compute).
 *   [P5]  "aclnnRmsNormDynamicQuant" (same docs), section "计算公式" (formula:
 *         RmsNorm with gamma + beta, optional smoothScales, scaleOut =
 *         row_max(abs(input))/max_val, yOut = round(input/scaleOut), max_val =
 *         127 for INT8) and section "约束说明" (empty tensors not supported).
 *
 * Readings where the pages are silent (each one is listed in the design doc):
 *   - x = x1 + x2 is an IEEE binary32 add (round to nearest even) of the two
 *     16-bit inputs, rounded once more (RNE) to the input dtype; that rounded
 *     x is both the xOut output and the x that is normalised.
 *   - y, input1 and input2 are never rounded to a 16-bit type (kept in fp64).
 *   - scaleOut is rounded (RNE) to binary32 and the codes divide by that
 *     stored value; round() is round-half-to-even; codes are clamped to
 *     [-Q, Q] as a guard that the arithmetic never needs (hits are counted).
 *   - Q = 127 for INT8, 7 for INT4; INT4 codes are packed two per byte,
 *     two's-complement nibbles, the even index in the low nibble.  The
 *     alternate INT4 container (the page names no container) holds eight
 *     codes per 32-bit word: code 8w + k of a row in bits 4k .. 4k+3 of word
 *     w (two's-complement nibbles), for rows whose length is a multiple of 8.
 *   - a row whose scale is 0 (all inputs 0) yields scale 0 and all codes 0.
 *   - y2 is produced with the mask absent only when both smooth scales are
 *     given.
 *
 * Arithmetic: fp64 everywhere the definition does arithmetic, except the add
 * itself, which the reading above fixes to binary32.  Sums run sequentially
 * over the row.  Build with -ffp-contract=off and without -ffast-math so that
 * every operation below is the IEEE operation written.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#if !defined(FLT_EVAL_METHOD) || FLT_EVAL_METHOD != 0
#error "the oracle needs float arithmetic evaluated in binary32 (FLT_EVAL_METHOD == 0)"
#endif

/* ---- the oracle's own codes (independent of the library's enums) ---------- */
#define ORC_OK 0
#define ORC_BAD_MASK 1  /* a Constraints-section rule on outputMask / smooth scales */
#define ORC_EMPTY 2     /* empty tensor: not supported (aclnnRmsNormDynamicQuant) */
#define ORC_BAD_SHAPE 3 /* INT4 with a row length its container cannot pack */
#define ORC_NULL 4      /* a required input or a selected output is missing */
#define ORC_BAD_ARG 5   /* unknown dtype / qdtype, negative or non-finite eps */

#define ORC_BF16 0
#define ORC_FP16 1
#define ORC_INT8 0
#define ORC_INT4 1
#define ORC_INT4_WORDS 2 /* INT4 codes, eight per 32-bit word */

/* ------------------------------------------------------------------------- */
/* 16-bit floating-point formats, written from their definitions.            */
/*   bfloat16: 1 sign, 8 exponent (bias 127), 7 fraction bits.               */
/*   binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits.               */
/* ------------------------------------------------------------------------- */

/* Exact value of a bfloat16 bit pattern: it is the top half of a binary32. */
static double decode_bf16(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Exact value of a binary16 bit pattern. */
static double decode_fp16(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int m = h & 0x3FF;
  double v;
  if (e == 0x1F) {
    v = m ? NAN : INFINITY;
  } else if (e == 0) {
    v = ldexp((double)m, -24); /* subnormal: m * 2^-24 */
  } else {
    v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

static double decode16(uint16_t h, int dtype) {
  return dtype == ORC_BF16 ? decode_bf16(h) : decode_fp16(h);
}

/* Round-to-nearest-even decision when `drop` low bits are removed from `sig`:
 * returns the kept part, incremented when the removed part is above one half,
 * or exactly one half with the kept part odd. */
static uint32_t rne_shift(uint32_t sig, int drop) {
  if (drop <= 0) return sig;
  if (drop >= 32) return 0; /* sig < 2^24 here, so the removed part is < 1/2 */
  uint32_t kept = sig >> drop;
  uint32_t rem = sig & ((1u << drop) - 1u);
  uint32_t half = 1u << (drop - 1);
  if (rem > half || (rem == half && (kept & 1u))) kept += 1u;
  return kept;
}

/* binary32 -> bfloat16, round to nearest even.  Keeps the top 16 bits of the
 * pattern; rounding up carries into the exponent (and to infinity) naturally. */
static uint16_t encode_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) {
    return (uint16_t)((u >> 16) | 0x0040u); /* NaN stays a (quiet) NaN */
  }
  uint32_t sign = u & 0x80000000u;
  uint32_t mag = u & 0x7FFFFFFFu;
  uint32_t kept = rne_shift(mag, 16); /* <= 0x7F80 (infinity) for finite input */
  return (uint16_t)((sign >> 16) | kept);
}

/* binary32 -> binary16, round to nearest even, overflow to infinity,
 * gradual underflow to subnormals and zero. */
static uint16_t encode_fp16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  int exp = (int)((u >> 23) & 0xFF);
  uint32_t frac = u & 0x7FFFFFu;
  if (exp == 0xFF) return (uint16_t)(sign | (frac ? 0x7E00u : 0x7C00u));
  if (exp == 0) return sign; /* |f| < 2^-126: far below half of 2^-24 */
  int e = exp - 127;                /* value = sig * 2^(e - 23) */
  uint32_t sig = frac | 0x800000u;  /* 24-bit significand */
  if (e >= -14) {
    /* normal binary16: keep 11 significant bits */
    uint32_t kept = rne_shift(sig, 13);
    if (kept == 0x800u) { /* rounding carried out of the significand */
      kept = 0x400u;
      e += 1;
    }
    if (e > 15) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)(kept & 0x3FFu));
  }
  /* subnormal binary16: value = k * 2^-24, k = sig * 2^(e - 23 + 24) */
  uint32_t k = rne_shift(sig, 13 + (-14 - e));
  /* k == 0x400 is the smallest normal, whose encoding is exactly 0x400 */
  return (uint16_t)(sign | (uint16_t)k);
}

static uint16_t encode16(float f, int dtype) {
  return dtype == ORC_BF16 ? encode_bf16(f) : encode_fp16(f);
}

/* Round half to even, to an integer-valued double (the definition). */
static double round_half_even(double v) {
  double fl = floor(v);
  double d = v - fl; /* exact */
  if (d > 0.5) return fl + 1.0;
  if (d < 0.5) return fl;
  return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* ------------------------------------------------------------------------- */
/* Output selection and the Constraints section's rules ([V2]).              */
/* mask < 0: outputMaskOptional absent; otherwise bit 0 = outputMask[0],     */
/* bit 1 = outputMask[1].                                                    */
/* ------------------------------------------------------------------------- */
int orc_selected_outputs(int mask, int has_s1, int has_s2, int *y1_on, int *y2_on) {
  int present = mask >= 0;
  int m0 = present && (mask & 1);
  int m1 = present && (mask & 2);
  /* "When outputMaskOptional is not empty and smoothScale1Optional has a value,
   *  outputMaskOptional[0] must be True.  When smoothScale2Optional has a value,
   *  outputMaskOptional[1] must be True." */
  if (present && has_s1 && !m0) return ORC_BAD_MASK;
  if (present && has_s2 && !m1) return ORC_BAD_MASK;
  /* "outputMaskOptional[0] and outputMaskOptional[1] cannot both be False." */
  if (present && !m0 && !m1) return ORC_BAD_MASK;
  /* "When outputMaskOptional is empty and smoothScale2Optional has a value,
   *  smoothScale1Optional must also have a value." */
  if (!present && has_s2 && !has_s1) return ORC_BAD_MASK;
  /* Formula: y1Out/scale1Out valid when outputMask[0] = True or no mask. */
  int on1 = m0 || !present;
  /* Formula: y2Out/scale2Out valid when outputMask[1] = True, or no mask with
   * both smooth scales given. */
  int on2 = m1 || (!present && has_s1 && has_s2);
  if (y1_on) *y1_on = on1;
  if (y2_on) *y2_on = on2;
  return ORC_OK;
}

/* Dynamic per-row symmetric quantization of one row of fp64 inputs:
 * scale = row_max(abs(input)) / Q rounded to binary32, code = round(input /
 * scale) with round-half-even, clamped to [-Q, Q] (guard; hits counted).
 * Writes n int8 codes, n/2 packed INT4 bytes (even index in the low nibble),
 * or n/8 32-bit words of eight INT4 codes (code k of a word in bits 4k..4k+3). */
static void quantize_row(const double *in, int64_t n, int qdtype, uint8_t *codes_out,
                         float *scale_out, int64_t *clamp_hits) {
  double qmax = (qdtype == ORC_INT8) ? 127.0 : 7.0;
  uint32_t *words = (uint32_t *)codes_out;
  double amax = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    double a = fabs(in[j]);
    if (a > amax) amax = a;
  }
  float scale = (float)(amax / qmax); /* binary32, round to nearest even */
  *scale_out = scale;
  for (int64_t j = 0; j < n; ++j) {
    double q = 0.0;
    if (scale != 0.0f) {
      q = round_half_even(in[j] / (double)scale);
      if (q > qmax) { q = qmax; ++*clamp_hits; }
      if (q < -qmax) { q = -qmax; ++*clamp_hits; }
    }
    int code = (int)q;
    if (qdtype == ORC_INT8) {
      codes_out[j] = (uint8_t)(int8_t)code;
    } else if (qdtype == ORC_INT4_WORDS) {
      uint32_t nib = (uint32_t)code & 0xFu; /* two's-complement nibble */
      if ((j % 8) == 0) words[j / 8] = 0u;
      words[j / 8] |= nib << (4 * (j % 8));
    } else {
      uint8_t nib = (uint8_t)(code & 0xF); /* two's-complement nibble */
      if ((j & 1) == 0) {
        codes_out[j / 2] = nib;
      } else {
        codes_out[j / 2] = (uint8_t)(codes_out[j / 2] | (uint8_t)(nib << 4));
      }
    }
  }
}

static int check_common(int64_t rows, int64_t n, int dtype, float eps, int qdtype) {
  if (dtype != ORC_BF16 && dtype != ORC_FP16) return ORC_BAD_ARG;
  if (qdtype != ORC_INT8 && qdtype != ORC_INT4 && qdtype != ORC_INT4_WORDS) return ORC_BAD_ARG;
  if (!(eps >= 0.0f) || !isfinite(eps)) return ORC_BAD_ARG;
  if (rows <= 0 || n <= 0) return ORC_EMPTY;
  if (qdtype == ORC_INT4 && (n % 2) != 0) return ORC_BAD_SHAPE;
  if (qdtype == ORC_INT4_WORDS && (n % 8) != 0) return ORC_BAD_SHAPE;
  return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* [V2] aclnnAddRmsNormDynamicQuantV2, "Formula" section, row by row.        */
/* All tensors row-major ("ND"): x1, x2, x_out, in1_dbg, in2_dbg are         */
/* [rows, n]; gamma, beta, smooth1, smooth2 are [n]; scale1/scale2 are       */
/* [rows]; y1/y2 are [rows, n] int8, [rows, n/2] packed INT4 bytes, or      */
/* [rows, n/8] 32-bit words of eight INT4 codes (4-byte aligned).            */
/* in1_dbg / in2_dbg (optional) receive the fp64 input1 / input2 values.     */
/* ------------------------------------------------------------------------- */
int orc_add_rms_norm_dynamic_quant_v2(
    const uint16_t *x1, const uint16_t *x2, const uint16_t *gamma, const uint16_t *beta,
    const uint16_t *smooth1, const uint16_t *smooth2, int64_t rows, int64_t n, int dtype,
    float eps, int mask, int qdtype, uint8_t *y1, float *scale1, uint8_t *y2, float *scale2,
    uint16_t *x_out, double *in1_dbg, double *in2_dbg, int64_t *clamp_hits) {
  int on1 = 0, on2 = 0;
  int st = orc_selected_outputs(mask, smooth1 != NULL, smooth2 != NULL, &on1, &on2);
  if (st != ORC_OK) return st;
  st = check_common(rows, n, dtype, eps, qdtype);
  if (st != ORC_OK) return st;
  if (!x1 || !x2 || !gamma) return ORC_NULL;
  if (on1 && (!y1 || !scale1)) return ORC_NULL;
  if (on2 && (!y2 || !scale2)) return ORC_NULL;

  int64_t code_bytes = (qdtype == ORC_INT8) ? n : n / 2;
  double *x = (double *)malloc(sizeof(double) * (size_t)n);
  double *in1 = (double *)malloc(sizeof(double) * (size_t)n);
  double *in2 = (double *)malloc(sizeof(double) * (size_t)n);
  if (!x || !in1 || !in2) {
    free(x); free(in1); free(in2);
    return ORC_BAD_ARG;
  }
  int64_t hits = 0;
  for (int64_t r = 0; r < rows; ++r) {
    const uint16_t *a = x1 + r * n;
    const uint16_t *b = x2 + r * n;
    /* x = x1 + x2: binary32 add, then rounded to the input dtype. */
    for (int64_t j = 0; j < n; ++j) {
      float fa = (float)decode16(a[j], dtype); /* exact */
      float fb = (float)decode16(b[j], dtype); /* exact */
      float s = fa + fb;                       /* IEEE binary32 add, RNE */
      uint16_t xr = encode16(s, dtype);
      if (x_out) x_out[r * n + j] = xr;
      x[j] = decode16(xr, dtype);
    }
    /* Rms(x) = sqrt( (1/n) * sum_i x_i^2 + epsilon ) */
    double ss = 0.0;
    for (int64_t j = 0; j < n; ++j) ss += x[j] * x[j];
    double rms = sqrt(ss / (double)n + (double)eps);
    /* y = x / Rms(x) * gamma + beta; input_k = y * smoothScale_k if given. */
    for (int64_t j = 0; j < n; ++j) {
      double y = x[j] / rms * decode16(gamma[j], dtype);
      if (beta) y += decode16(beta[j], dtype);
      in1[j] = smooth1 ? y * decode16(smooth1[j], dtype) : y;
      in2[j] = smooth2 ? y * decode16(smooth2[j], dtype) : y;
    }
    if (in1_dbg) memcpy(in1_dbg + r * n, in1, sizeof(double) * (size_t)n);
    if (in2_dbg) memcpy(in2_dbg + r * n, in2, sizeof(double) * (size_t)n);
    /* scale_k = row_max(abs(input_k)) / Q; y_k = round(input_k / scale_k). */
    if (on1) quantize_row(in1, n, qdtype, y1 + r * code_bytes, scale1 + r, &hits);
    if (on2) quantize_row(in2, n, qdtype, y2 + r * code_bytes, scale2 + r, &hits);
  }
  free(x); free(in1); free(in2);
  if (clamp_hits) *clamp_hits = hits;
  return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* [P5] aclnnRmsNormDynamicQuant, "计算公式" (formula) section: the same     */
/* normalisation on a given x (no add), one optional smoothScales, one       */
/* output.  max_val = 127 for INT8 (page) and 7 for INT4 (from [V2]).        */
/* ------------------------------------------------------------------------- */
int orc_rms_norm_dynamic_quant(const uint16_t *x, const uint16_t *gamma, const uint16_t *beta,
                               const uint16_t *smooth, int64_t rows, int64_t n, int dtype,
                               float eps, int qdtype, uint8_t *y, float *scale,
                               double *in_dbg, int64_t *clamp_hits) {
  int st = check_common(rows, n, dtype, eps, qdtype);
  if (st != ORC_OK) return st;
  if (!x || !gamma || !y || !scale) return ORC_NULL;
  int64_t code_bytes = (qdtype == ORC_INT8) ? n : n / 2;
  double *in = (double *)malloc(sizeof(double) * (size_t)n);
  if (!in) return ORC_BAD_ARG;
  int64_t hits = 0;
  for (int64_t r = 0; r < rows; ++r) {
    const uint16_t *xr = x + r * n;
    double ss = 0.0;
    for (int64_t j = 0; j < n; ++j) {
      double v = decode16(xr[j], dtype);
      ss += v * v;
    }
    double rms = sqrt(ss / (double)n + (double)eps);
    for (int64_t j = 0; j < n; ++j) {
      double yv = decode16(xr[j], dtype) / rms * decode16(gamma[j], dtype);
      if (beta) yv += decode16(beta[j], dtype);
      /* no smoothScales: quantize y directly; else input = y * smoothScales */
      in[j] = smooth ? yv * decode16(smooth[j], dtype) : yv;
    }
    if (in_dbg) memcpy(in_dbg + r * n, in, sizeof(double) * (size_t)n);
    quantize_row(in, n, qdtype, y + r * code_bytes, scale + r, &hits);
  }
  free(in);
  if (clamp_hits) *clamp_hits = hits;
  return ORC_OK;
}

/* ---- element-level entry points, exported so the tests can pin them ------ */
double orc_decode16(uint16_t bits, int dtype) { return decode16(bits, dtype); }
uint16_t orc_encode16_rne(float f, int dtype) { return encode16(f, dtype); }
double orc_round_half_even(double v) { return round_half_even(v); }

/* x = x1 + x2 for one element: binary32 add, RNE to the 16-bit dtype. */
uint16_t orc_add_round(uint16_t a, uint16_t b, int dtype) {
  float fa = (float)decode16(a, dtype);
  float fb = (float)decode16(b, dtype);
  float s = fa + fb;
  return encode16(s, dtype);
}

/* Batch forms of the element entry points (same definitions, over arrays). */
void orc_decode16_array(const uint16_t *bits, int64_t count, int dtype, double *out) {
  for (int64_t i = 0; i < count; ++i) out[i] = decode16(bits[i], dtype);
}
void orc_encode16_array(const float *f, int64_t count, int dtype, uint16_t *out) {
  for (int64_t i = 0; i < count; ++i) out[i] = encode16(f[i], dtype);
}
void orc_add_round_array(const uint16_t *a, const uint16_t *b, int64_t count, int dtype,
                         uint16_t *out) {
  for (int64_t i = 0; i < count; ++i) out[i] = orc_add_round(a[i], b[i], dtype);
}
