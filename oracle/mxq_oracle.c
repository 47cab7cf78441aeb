/*
 * mxq_oracle.c - scalar CPU oracle for block-scaled microscaling quantization.
 *
 * TEST INFRASTRUCTURE ONLY.  The product library never includes, links or
 * calls this file.  Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg load it.  It shares no code, header, table or constant
 * with the CUDA kernels.
 *
 * Every quantity is computed in IEEE double.  Every bf16/f16/f32 input, every
 * power-of-two block scale and every scaled value is exact in double, so the
 * only roundings are the ones the method names: the element cast (E2M1 by
 * the midpoint rule, E4M3 to nearest-even) and the final rounding to the
 * output dtype (nearest-even, subnormals kept, overflow to infinity).  Those
 * roundings are written out below from the format definitions.
 *
 * Sources (page title, then section / item):
 *   [MX]  "nemo_automodel.components.quantization.mxfp4": module docstring
 *         (packed layout), quantize_mxfp4 (scale rule, K % 32), dequantize_mxfp4,
 *         MXFP4GroupedMM (forward / backward), MXFP4_BLOCK_SIZE,
 *         _FP4_E2M1_TABLE, _FP4_E2M1_MIDPOINTS, _FP4_BYTE_TABLE.
 *   [CQ]  "nemo_automodel.components.models.deepseek_v41.quantization":
 *         quantize_cache, _power_of_two_ceiling, _CacheQuantization.forward.
 *   [MO]  "NVIDIA Model Optimizer: from mtq.quantize to a 4.95-bit
 *         DeepSeek-R1", section "NVFP4 in the code: two scales and a nibble"
 *         (E2M1 max 6, E4M3 max 448, scale clamp [2^-9, 448], tie rule and
 *         nibble order of _cast_fp4) and the numerics YAML of "mtq.quantize
 *         is three moves" (block 16, e4m3 scale).
 *
 * Readings where the pages are silent (each is a named choice, listed with
 * its reason in the design notes):
 *   - sign of values whose magnitude rounds to code 0: the code carries the
 *     sign bit iff the value is < 0, so -0.0 gives nibble 0 and a tiny
 *     negative gives nibble 8; nibble 8 decodes to +0.0 (table index 8).
 *   - all-zero MX block: scale exponent -127 (byte 0x00), all codes 0.
 *   - E8M0 exponent clamped to [-127, 127]; byte 0xFF (NaN) is never produced
 *     by quantization and decodes to NaN.
 *   - quantize_cache scale: the least power of two s with s*qmax >= amax,
 *     decided exactly, clamped to [2^-126, 2^127] (fp8, mxfp4) or
 *     [2^-9, 2^8] (nvfp4); an all-zero block takes the lower clamp.
 *   - quantize_cache fp8 element: E4M3 (finite max 448), nearest-even,
 *     saturating, sign of zero kept.
 *   - a final partial channel group uses only its real channels (zero
 *     padding cannot raise a block maximum).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Row loops whose iterations touch disjoint outputs may run on all host
   cores when the file is built with OpenMP (the benchmark's all-core CPU
   baseline).  Each row is computed by exactly the same operations in the
   same order either way, so the results are identical; without OpenMP the
   marker expands to nothing. */
#ifdef _OPENMP
#define ORC_PARALLEL_ROWS _Pragma("omp parallel for schedule(static)")
/* for loops over a row list of which each pass uses only a few entries */
#define ORC_PARALLEL_SPARSE_ROWS _Pragma("omp parallel for schedule(dynamic, 1)")
#else
#define ORC_PARALLEL_ROWS
#define ORC_PARALLEL_SPARSE_ROWS
#endif

/* dtype codes of this oracle's interface */
enum { ORC_BF16 = 0, ORC_F16 = 1, ORC_F32 = 2 };
/* cache formats of this oracle's interface */
enum { ORC_FP8 = 0, ORC_MXFP4 = 1, ORC_NVFP4 = 2 };
/* error codes */
enum { ORC_OK = 0, ORC_EARG = -1, ORC_EOFFS = -6 };

/* ------------------------------------------------------------------------ */
/* E2M1: [MX] _FP4_E2M1_TABLE, _FP4_E2M1_MIDPOINTS; [MO] _cast_fp4.          */
/* ------------------------------------------------------------------------ */

/* Code c in 0..7 is the magnitude, code c+8 its negative.  Index 8 is the
   literal 0.0 of the table, i.e. +0.0. */
static const double E2M1_TABLE[16] = {
    0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
    0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0};

/* Decision points between neighbouring magnitudes. */
static const double E2M1_MIDPOINTS[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};

double orc_e2m1_value(int code) { return E2M1_TABLE[code & 15]; }

/* The magnitude code is the number of midpoints that |v| lies above
   (searchsorted).  On an exact tie the cast takes the neighbour with the
   even code: for the midpoints at odd positions (0.75, 1.75, 3.5) that is
   the upper neighbour, for the others the lower one.  Magnitudes >= 5
   therefore saturate to code 7 (value 6).  The sign bit is set iff v < 0. */
int orc_e2m1_code(double v) {
  double a = fabs(v);
  int mag = 0;
  for (int i = 0; i < 7; ++i) {
    int above = a > E2M1_MIDPOINTS[i];
    int tie_up = (a == E2M1_MIDPOINTS[i]) && (i % 2 == 1);
    if (above || tie_up) mag += 1;
  }
  return mag | (v < 0.0 ? 8 : 0);
}

/* ------------------------------------------------------------------------ */
/* Rounding to binary formats, written from the IEEE-754 definitions.        */
/* ------------------------------------------------------------------------ */

/* Round v to the nearest number with p significant bits whose binary
   exponent is at least emin (below 2^emin the spacing stays 2^(emin-p+1),
   i.e. gradual underflow), ties to the even significand.  No overflow
   handling: callers apply their format's largest finite value. */
static double round_to_precision(double v, int p, int emin) {
  if (v == 0.0 || !isfinite(v)) return v;
  double a = fabs(v);
  int e = ilogb(a); /* floor(log2 a), exact */
  if (e < emin) e = emin;
  double ulp = ldexp(1.0, e - p + 1);
  double n = a / ulp; /* exact: division by a power of two */
  double f = floor(n);
  double rem = n - f;
  if (rem > 0.5 || (rem == 0.5 && fmod(f, 2.0) != 0.0)) f += 1.0;
  double r = f * ulp;
  return v < 0.0 ? -r : r;
}

/* bfloat16: 8 significant bits, emin -126, largest finite (2-2^-7)*2^127. */
double orc_round_bf16(double v) {
  double r = round_to_precision(v, 8, -126);
  if (fabs(r) > ldexp(255.0, 120)) r = copysign(INFINITY, v);
  return r;
}
/* binary16: 11 significant bits, emin -14, largest finite 65504. */
double orc_round_f16(double v) {
  double r = round_to_precision(v, 11, -14);
  if (fabs(r) > 65504.0) r = copysign(INFINITY, v);
  return r;
}
/* binary32: 24 significant bits, emin -126, largest finite (2-2^-23)*2^127. */
double orc_round_f32(double v) {
  double r = round_to_precision(v, 24, -126);
  if (fabs(r) > ldexp(16777215.0, 104)) r = copysign(INFINITY, v);
  return r;
}
/* E4M3 ("fn" flavour, no infinities): 4 significant bits, emin -6, largest
   finite 448; results beyond 448 saturate to +-448 ([MO]: 448 is the E4M3
   maximum).  The sign of zero is kept. */
double orc_round_e4m3(double v) {
  double r = round_to_precision(v, 4, -6);
  if (fabs(r) > 448.0) r = copysign(448.0, v);
  return r;
}

/* ------------------------------------------------------------------------ */
/* Bit-level encode / decode of the element dtypes.                          */
/* ------------------------------------------------------------------------ */

static double decode_bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16; /* bf16 is the top half of a binary32 */
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}
static double decode_f32(uint32_t u) {
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}
static double decode_f16(uint16_t h) {
  int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24);
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + m), e - 25);
  return s ? -v : v;
}

/* Encoders take a value already exactly representable in the target
   format (or +-inf, or NaN). */
static uint16_t encode_bf16(double v) {
  if (isnan(v)) return 0x7FC0;
  float f = (float)v; /* exact: v is a bf16 value */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}
static uint32_t encode_f32(double v) {
  if (isnan(v)) return 0x7FC00000u;
  float f = (float)v; /* exact */
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}
static uint16_t encode_f16(double v) {
  if (isnan(v)) return 0x7E00;
  uint16_t s = signbit(v) ? 0x8000 : 0;
  double a = fabs(v);
  if (isinf(a)) return s | 0x7C00;
  if (a < ldexp(1.0, -14)) return s | (uint16_t)(a / ldexp(1.0, -24));
  int e = ilogb(a);
  uint16_t m = (uint16_t)(a / ldexp(1.0, e - 10) - 1024.0);
  return s | (uint16_t)((e + 15) << 10) | m;
}
/* E4M3 byte of an exactly representable value with |v| <= 448. */
uint8_t orc_encode_e4m3(double v) {
  uint8_t s = signbit(v) ? 0x80 : 0;
  double a = fabs(v);
  if (a < ldexp(1.0, -6)) return s | (uint8_t)(a / ldexp(1.0, -9));
  int e = ilogb(a);
  uint8_t m = (uint8_t)(a / ldexp(1.0, e - 3) - 8.0);
  return s | (uint8_t)((e + 7) << 3) | m;
}
double orc_decode_e4m3(uint8_t b) {
  int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp((double)(8 + m), e - 10);
  return s ? -v : v;
}

static double load_elem(const void* p, int dtype, int64_t i) {
  switch (dtype) {
    case ORC_BF16: return decode_bf16(((const uint16_t*)p)[i]);
    case ORC_F16: return decode_f16(((const uint16_t*)p)[i]);
    default: return decode_f32(((const uint32_t*)p)[i]);
  }
}
/* Round v (any double) to dtype and store its bit pattern. */
static void store_rounded(void* p, int dtype, int64_t i, double v) {
  switch (dtype) {
    case ORC_BF16: ((uint16_t*)p)[i] = encode_bf16(isnan(v) ? v : orc_round_bf16(v)); break;
    case ORC_F16: ((uint16_t*)p)[i] = encode_f16(isnan(v) ? v : orc_round_f16(v)); break;
    default: ((uint32_t*)p)[i] = encode_f32(isnan(v) ? v : orc_round_f32(v)); break;
  }
}

/* Vector helpers for the tests: decode and round whole arrays. */
void orc_decode_array(const void* p, int dtype, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = load_elem(p, dtype, i);
}
void orc_round_array(const double* v, int dtype, int64_t n, void* out) {
  for (int64_t i = 0; i < n; ++i) store_rounded(out, dtype, i, v[i]);
}

/* ------------------------------------------------------------------------ */
/* MXFP4 pack / unpack ([MX] quantize_mxfp4, dequantize_mxfp4).              */
/* ------------------------------------------------------------------------ */

/* Block scale exponent of quantize_mxfp4: floor(log2(amax)) - 2, held in an
   E8M0 byte (exponent + 127) and therefore clamped to [-127, 127]; an
   all-zero block takes -127. */
int orc_mx_scale_exp(double amax) {
  if (amax == 0.0) return -127;
  int e = ilogb(amax) - 2;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

/* x: [rows, K] elements of `dtype`; packed: [rows, K/2] bytes, the code of
   column 2j in the low nibble of byte j and column 2j+1 in the high nibble;
   scales: [rows, K/32] E8M0 bytes, one per 32 contiguous columns. */
int orc_mx_quantize(const void* x, int dtype, int64_t rows, int64_t K, uint8_t* packed,
                    uint8_t* scales) {
  if (K % 32 != 0 || rows < 0) return ORC_EARG;
  ORC_PARALLEL_ROWS
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < K / 32; ++b) {
      int64_t base = r * K + b * 32;
      double amax = 0.0;
      for (int i = 0; i < 32; ++i) {
        double a = fabs(load_elem(x, dtype, base + i));
        if (a > amax) amax = a;
      }
      int e = orc_mx_scale_exp(amax);
      scales[r * (K / 32) + b] = (uint8_t)(e + 127);
      for (int j = 0; j < 16; ++j) {
        int lo = orc_e2m1_code(ldexp(load_elem(x, dtype, base + 2 * j), -e));
        int hi = orc_e2m1_code(ldexp(load_elem(x, dtype, base + 2 * j + 1), -e));
        packed[r * (K / 2) + b * 16 + j] = (uint8_t)(lo | (hi << 4));
      }
    }
  }
  return ORC_OK;
}

/* Value of one packed element: table value times 2^(byte - 127); scale byte
   0xFF is the E8M0 NaN. */
static double mx_element(const uint8_t* packed, const uint8_t* scales, int64_t K, int64_t r,
                         int64_t k) {
  uint8_t byte = packed[r * (K / 2) + k / 2];
  int nib = (k % 2 == 0) ? (byte & 15) : (byte >> 4);
  uint8_t s = scales[r * (K / 32) + k / 32];
  if (s == 0xFF) return NAN;
  return E2M1_TABLE[nib] * ldexp(1.0, (int)s - 127);
}

int orc_mx_dequantize(const uint8_t* packed, const uint8_t* scales, int64_t rows, int64_t K,
                      void* out, int out_dtype) {
  if (K % 32 != 0 || rows < 0) return ORC_EARG;
  ORC_PARALLEL_ROWS
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k)
      store_rounded(out, out_dtype, r * K + k, mx_element(packed, scales, K, r, k));
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Fake quantization of cache values ([CQ] quantize_cache).                  */
/* ------------------------------------------------------------------------ */

/* Largest representable element magnitude of each cache format. */
static double fmt_qmax(int fmt) { return fmt == ORC_FP8 ? 448.0 : 6.0; }
static int fmt_lo(int fmt) { return fmt == ORC_NVFP4 ? -9 : -126; }
static int fmt_hi(int fmt) { return fmt == ORC_NVFP4 ? 8 : 127; }

/* Exponent k of the block scale 2^k: _power_of_two_ceiling of amax/qmax,
   taken exactly (the least k with 2^k * qmax >= amax, decided by exact
   comparisons rather than a rounded quotient), clamped to the format's
   scale range; an all-zero block takes the lower clamp. */
int orc_cache_scale_exp(double amax, int fmt) {
  double qmax = fmt_qmax(fmt);
  int lo = fmt_lo(fmt), hi = fmt_hi(fmt);
  if (amax == 0.0) return lo;
  int k = ilogb(amax) - ilogb(qmax) - 1; /* 2^k * qmax < amax here */
  while (ldexp(qmax, k) < amax) ++k;
  if (k < lo) k = lo;
  if (k > hi) k = hi;
  return k;
}

/* Fake-quantized value of one element x under scale 2^k. */
double orc_cache_element(double x, int k, int fmt) {
  double v = ldexp(x, -k); /* exact */
  if (fmt == ORC_FP8) return ldexp(orc_round_e4m3(v), k);
  return ldexp(E2M1_TABLE[orc_e2m1_code(v)], k);
}

/* in / out: [rows, C] elements of `dtype` (distinct storage).  Channels are
   split into groups of B; the last group of a row may be shorter. */
int orc_quantize_cache(const void* in, void* out, int dtype, int64_t rows, int64_t C, int fmt,
                       int B) {
  if (B < 1 || C < 0 || rows < 0 || fmt < 0 || fmt > 2) return ORC_EARG;
  ORC_PARALLEL_ROWS
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c0 = 0; c0 < C; c0 += B) {
      int64_t c1 = c0 + B < C ? c0 + B : C;
      double amax = 0.0;
      for (int64_t c = c0; c < c1; ++c) {
        double a = fabs(load_elem(in, dtype, r * C + c));
        if (a > amax) amax = a;
      }
      int k = orc_cache_scale_exp(amax, fmt);
      for (int64_t c = c0; c < c1; ++c)
        store_rounded(out, dtype, r * C + c,
                      orc_cache_element(load_elem(in, dtype, r * C + c), k, fmt));
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Grouped GEMM over packed expert weights ([MX] MXFP4GroupedMM).            */
/* ------------------------------------------------------------------------ */

/* offs[e] is the end (exclusive) of expert e's contiguous rows; expert e
   owns rows [offs[e-1], offs[e]) with offs[-1] = 0.  Valid iff
   non-decreasing, non-negative and offs[E-1] == T. */
int orc_check_offs(const int32_t* offs, int64_t E, int64_t T) {
  int64_t prev = 0;
  for (int64_t e = 0; e < E; ++e) {
    if (offs[e] < prev) return ORC_EOFFS;
    prev = offs[e];
  }
  return prev == T ? ORC_OK : ORC_EOFFS;
}

/* a: bf16 [T, Kin]; packed: [E, N, K/2]; scales: [E, N, K/32]; weights of
   expert e: W_e[n][k] = dequantized value (exact in double).
   transpose_w = 0 (forward):  Kin = K, out[i][n] = sum_k a[t][k] W_e[n][k]
   transpose_w = 1 (input gradient): Kin = N, out[i][k] = sum_n a[t][n] W_e[n][k]
   for t = rows[i].  Sums run in double in index order; out is double and is
   NOT rounded to bf16 (the caller compares before or after rounding). */
int orc_grouped_mm(const uint16_t* a, const uint8_t* packed, const uint8_t* scales,
                   const int32_t* offs, int64_t T, int64_t E, int64_t N, int64_t K,
                   int transpose_w, const int64_t* rows, int64_t nrows, double* out) {
  if (E < 1 || K % 32 != 0 || N < 1 || T < 0) return ORC_EARG;
  if (orc_check_offs(offs, E, T) != ORC_OK) return ORC_EOFFS;
  int64_t kin = transpose_w ? N : K, nout = transpose_w ? K : N;
  double* w = (double*)malloc((size_t)(N * K) * sizeof(double));
  if (!w) return ORC_EARG;
  for (int64_t e = 0; e < E; ++e) {
    int64_t lo = e == 0 ? 0 : offs[e - 1], hi = offs[e];
    int have = 0;
    for (int64_t i = 0; i < nrows && !have; ++i) have = rows[i] >= lo && rows[i] < hi;
    if (!have) continue;
    const uint8_t* pe = packed + e * N * (K / 2);
    const uint8_t* se = scales + e * N * (K / 32);
    ORC_PARALLEL_ROWS
    for (int64_t n = 0; n < N; ++n)
      for (int64_t k = 0; k < K; ++k) w[n * K + k] = mx_element(pe, se, K, n, k);
    ORC_PARALLEL_SPARSE_ROWS
    for (int64_t i = 0; i < nrows; ++i) {
      int64_t t = rows[i];
      if (t < lo || t >= hi) continue;
      const uint16_t* at = a + t * kin;
      double* o = out + i * nout;
      for (int64_t j = 0; j < nout; ++j) o[j] = 0.0;
      if (!transpose_w) {
        for (int64_t n = 0; n < N; ++n) {
          double acc = 0.0;
          for (int64_t k = 0; k < K; ++k) acc += decode_bf16(at[k]) * w[n * K + k];
          o[n] = acc;
        }
      } else {
        for (int64_t n = 0; n < N; ++n) {
          double g = decode_bf16(at[n]);
          for (int64_t k = 0; k < K; ++k) o[k] += g * w[n * K + k];
        }
      }
    }
  }
  free(w);
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 two-level quantization ([MO] "NVFP4 in the code: two scales and a  */
/* nibble"; block 16 and e4m3 scales from the numerics YAML of "mtq.quantize */
/* is three moves").                                                         */
/* ------------------------------------------------------------------------ */

/* binary32 arithmetic, emulated: the exact real result rounded once to
   binary32.  For inputs that are binary32 values, computing in double and
   rounding to binary32 gives exactly the correctly rounded binary32 result
   for + - * / (double rounding is innocuous when 53 >= 2*24 + 2; Figueroa,
   "When is double rounding innocuous?", SIGNUM 1995). */
static double f32_mul(double a, double b) { return orc_round_f32(a * b); }
static double f32_div(double a, double b) { return orc_round_f32(a / b); }

/* Per-tensor scale g = max|W| / (6 * 448) as a binary32 value. */
double orc_nvfp4_global_scale(double amax) { return f32_div(amax, 6.0 * 448.0); }

/* Block scale s_b = E4M3(amax_b / (6 g)) with a zero quotient replaced by
   1.0 and the quotient clamped to [2^-9, 448] before the cast. */
double orc_nvfp4_block_scale(double amax_b, double g) {
  double q = f32_div(amax_b, f32_mul(6.0, g));
  if (q == 0.0) q = 1.0;
  if (q < ldexp(1.0, -9)) q = ldexp(1.0, -9);
  if (q > 448.0) q = 448.0;
  return orc_round_e4m3(q);
}

/* x: [rows, K] (K % 16 == 0).  packed [rows, K/2] (E2M1 codes, low nibble =
   even column); block_scales [rows, K/16] (E4M3 bytes); *global_scale = g.
   The element cast is E2M1(W / (s_b g)) with s_b * g and the quotient in
   binary32.  An all-zero tensor gives g = 0, codes 0 and block scales 1.0. */
int orc_nvfp4_quantize(const void* x, int dtype, int64_t rows, int64_t K, uint8_t* packed,
                       uint8_t* block_scales, float* global_scale) {
  if (K % 16 != 0 || rows < 0) return ORC_EARG;
  double amax = 0.0;
  for (int64_t i = 0; i < rows * K; ++i) {
    double a = fabs(load_elem(x, dtype, i));
    if (a > amax) amax = a;
  }
  double g = amax == 0.0 ? 0.0 : orc_nvfp4_global_scale(amax);
  *global_scale = (float)g;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < K / 16; ++b) {
      int64_t base = r * K + b * 16;
      double amax_b = 0.0;
      for (int i = 0; i < 16; ++i) {
        double a = fabs(load_elem(x, dtype, base + i));
        if (a > amax_b) amax_b = a;
      }
      double s = amax == 0.0 ? 1.0 : orc_nvfp4_block_scale(amax_b, g);
      block_scales[r * (K / 16) + b] = orc_encode_e4m3(s);
      double d = f32_mul(s, g);
      for (int j = 0; j < 8; ++j) {
        int lo = 0, hi = 0;
        if (amax != 0.0) {
          /* the sign bit follows x itself: a binary32 quotient of a tiny
             negative value may underflow to -0.0 */
          double x0 = load_elem(x, dtype, base + 2 * j), x1 = load_elem(x, dtype, base + 2 * j + 1);
          lo = (orc_e2m1_code(fabs(f32_div(x0, d))) & 7) | (x0 < 0.0 ? 8 : 0);
          hi = (orc_e2m1_code(fabs(f32_div(x1, d))) & 7) | (x1 < 0.0 ? 8 : 0);
        }
        packed[r * (K / 2) + b * 8 + j] = (uint8_t)(lo | (hi << 4));
      }
    }
  }
  return ORC_OK;
}

/* out[r][k] = E2M1(nibble) * s_b * g, evaluated in binary32 (the product of
   the code and the E4M3 scale is exact there; times g rounds once), then
   rounded to out_dtype. */
int orc_nvfp4_dequantize(const uint8_t* packed, const uint8_t* block_scales, float global_scale,
                         int64_t rows, int64_t K, void* out, int out_dtype) {
  if (K % 16 != 0 || rows < 0) return ORC_EARG;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = packed[r * (K / 2) + k / 2];
      int nib = (k % 2 == 0) ? (byte & 15) : (byte >> 4);
      double s = orc_decode_e4m3(block_scales[r * (K / 16) + k / 16]);
      double v = f32_mul(E2M1_TABLE[nib] * s, (double)global_scale);
      store_rounded(out, out_dtype, r * K + k, v);
    }
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Packed cache storage: the stored form of quantize_cache ([CQ]).           */
/* ------------------------------------------------------------------------ */

/* Scale byte of a cache block with scale 2^k: E8M0 (k + 127) for fp8 and
   mxfp4, the E4M3 encoding of 2^k for nvfp4. */
uint8_t orc_cache_scale_byte(int k, int fmt) {
  if (fmt == ORC_NVFP4) return orc_encode_e4m3(ldexp(1.0, k));
  return (uint8_t)(k + 127);
}

/* in [rows, C] (C % B == 0; B even for the fp4 formats).  codes: fp8 -> [rows, C] E4M3 bytes of
   x / 2^k; mxfp4/nvfp4 -> [rows, C/2] E2M1 codes (low nibble = even column,
   sign bit iff x < 0).  scales: [rows, C/B] scale bytes. */
int orc_quantize_cache_packed(const void* in, int dtype, int64_t rows, int64_t C, int fmt, int B,
                              uint8_t* codes, uint8_t* scales) {
  if (B < 1 || C % B != 0 || rows < 0 || fmt < 0 || fmt > 2) return ORC_EARG;
  if (fmt != ORC_FP8 && B % 2 != 0) return ORC_EARG; /* nibble pairs stay in a group */
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c0 = 0; c0 < C; c0 += B) {
      double amax = 0.0;
      for (int64_t c = c0; c < c0 + B; ++c) {
        double a = fabs(load_elem(in, dtype, r * C + c));
        if (a > amax) amax = a;
      }
      int k = orc_cache_scale_exp(amax, fmt);
      scales[r * (C / B) + c0 / B] = orc_cache_scale_byte(k, fmt);
      for (int64_t c = c0; c < c0 + B; ++c) {
        double x = load_elem(in, dtype, r * C + c);
        double v = ldexp(x, -k);
        if (fmt == ORC_FP8) {
          codes[r * C + c] = orc_encode_e4m3(orc_round_e4m3(v));
        } else {
          int code = orc_e2m1_code(v);
          uint8_t* byte = &codes[r * (C / 2) + c / 2];
          if (c % 2 == 0) *byte = (uint8_t)code;
          else *byte = (uint8_t)(*byte | (code << 4));
        }
      }
    }
  }
  return ORC_OK;
}

/* out[r][c] = round_dtype(decode(code) * scale); fp4 zeros are +0 (as in
   the fake quantization), fp8 keeps the sign of zero. */
int orc_dequantize_cache_packed(const uint8_t* codes, const uint8_t* scales, int64_t rows,
                                int64_t C, int fmt, int B, void* out, int out_dtype) {
  if (B < 1 || C % B != 0 || rows < 0 || fmt < 0 || fmt > 2) return ORC_EARG;
  if (fmt != ORC_FP8 && B % 2 != 0) return ORC_EARG; /* nibble pairs stay in a group */
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < C; ++c) {
      uint8_t sb = scales[r * (C / B) + c / B];
      double s = fmt == ORC_NVFP4 ? orc_decode_e4m3(sb)
                 : sb == 0xFF       ? NAN /* the E8M0 NaN */
                                    : ldexp(1.0, (int)sb - 127);
      double v;
      if (fmt == ORC_FP8) {
        v = orc_decode_e4m3(codes[r * C + c]) * s;
      } else {
        uint8_t byte = codes[r * (C / 2) + c / 2];
        v = E2M1_TABLE[(c % 2 == 0) ? (byte & 15) : (byte >> 4)] * s;
        if (v == 0.0) v = 0.0; /* a zero fp4 element is +0 whatever the signs */
      }
      store_rounded(out, out_dtype, r * C + c, v);
    }
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 block scale chosen by least squared weight error ([MO] "NVFP4's    */
/* own rules": mse).                                                         */
/* ------------------------------------------------------------------------ */

/* Squared weight error of one 16-block under block-scale code c (an E4M3
   byte, 1..126):  d = s_c * g in binary32; each weight is cast to E2M1 as
   the max rule casts it (binary32 quotient w / d, nearest-even, saturating);
   the error of weight i is e_i = q_i * d - w_i, which double arithmetic
   holds exactly; the sum of e_i^2 is accumulated over i = 0..15 in order,
   one fused multiply-add in double per term.  A code whose d underflows to
   zero can represent nothing and gets +infinity. */
double orc_nvfp4_block_sq_error(const double* w, double g, int code) {
  double d = f32_mul(orc_decode_e4m3((uint8_t)code), g);
  if (d == 0.0) return INFINITY;
  double err = 0.0;
  for (int i = 0; i < 16; ++i) {
    double q = orc_e2m1_value(orc_e2m1_code(fabs(f32_div(w[i], d)))) * (w[i] < 0.0 ? -1.0 : 1.0);
    double e = fma(q, d, -w[i]);
    err = fma(e, e, err);
  }
  return err;
}

/* The code with the least error over the 126 positive finite E4M3 codes,
   the smallest code among equal least errors. */
int orc_nvfp4_mse_code(const double* w, double g) {
  int best = 1;
  double best_err = INFINITY;
  for (int c = 1; c <= 126; ++c) {
    double err = orc_nvfp4_block_sq_error(w, g, c);
    if (err < best_err) {
      best_err = err;
      best = c;
    }
  }
  return best;
}

/* NVFP4 quantize with mse block scales, given the per-tensor scale g (the
   max rule's amax / 2688).  g == 0 (an all-zero tensor) gives the max
   rule's output: scale code 1.0 (0x38) and zero codes everywhere. */
int orc_nvfp4_quantize_mse_rows(const void* x, int dtype, int64_t rows, int64_t K, double g,
                                uint8_t* packed, uint8_t* block_scales) {
  if (K % 16 != 0 || rows < 0) return ORC_EARG;
  ORC_PARALLEL_ROWS
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < K / 16; ++b) {
      int64_t base = r * K + b * 16;
      double w[16];
      for (int i = 0; i < 16; ++i) w[i] = load_elem(x, dtype, base + i);
      int code = g == 0.0 ? 0x38 : orc_nvfp4_mse_code(w, g);
      block_scales[r * (K / 16) + b] = (uint8_t)code;
      double d = f32_mul(orc_decode_e4m3((uint8_t)code), g);
      for (int j = 0; j < 8; ++j) {
        int nib[2] = {0, 0};
        for (int h = 0; h < 2 && g != 0.0; ++h) {
          double xi = w[2 * j + h];
          if (xi == 0.0) continue; /* code 0, also where d underflowed to 0 */
          nib[h] = (orc_e2m1_code(fabs(f32_div(xi, d))) & 7) | (xi < 0.0 ? 8 : 0);
        }
        packed[r * (K / 2) + b * 8 + j] = (uint8_t)(nib[0] | (nib[1] << 4));
      }
    }
  }
  return ORC_OK;
}

int orc_nvfp4_quantize_mse(const void* x, int dtype, int64_t rows, int64_t K, uint8_t* packed,
                           uint8_t* block_scales, float* global_scale) {
  if (K % 16 != 0 || rows < 0) return ORC_EARG;
  double amax = 0.0;
  for (int64_t i = 0; i < rows * K; ++i) {
    double a = fabs(load_elem(x, dtype, i));
    if (a > amax) amax = a;
  }
  double g = amax == 0.0 ? 0.0 : orc_nvfp4_global_scale(amax);
  *global_scale = (float)g;
  return orc_nvfp4_quantize_mse_rows(x, dtype, rows, K, g, packed, block_scales);
}

/* ------------------------------------------------------------------------ */
/* W4A4 grouped GEMM: both operands MXFP4 ([MO] "W4A4 NVFP4 on FP4 tensor   */
/* cores", here with the MX format of [MX]).                                 */
/* ------------------------------------------------------------------------ */

/* x: bf16 [T, K] activations, quantized row by row with orc_mx_quantize
   (one E8M0 scale per 32 columns) and dequantized exactly; weights as in
   orc_grouped_mm.  out[i][n] = sum_k deq(q(x))[t][k] W_e[n][k] for t =
   rows[i], summed in double in index order (not rounded). */
int orc_w4a4_grouped_mm(const uint16_t* x, const uint8_t* packed, const uint8_t* scales,
                        const int32_t* offs, int64_t T, int64_t E, int64_t N, int64_t K,
                        const int64_t* rows, int64_t nrows, double* out) {
  if (E < 1 || K % 32 != 0 || N < 1 || T < 0) return ORC_EARG;
  if (orc_check_offs(offs, E, T) != ORC_OK) return ORC_EOFFS;
  uint8_t* qp = (uint8_t*)malloc((size_t)(K / 2));
  uint8_t* qs = (uint8_t*)malloc((size_t)(K / 32));
  double* xa = (double*)malloc((size_t)K * sizeof(double));
  double* w = (double*)malloc((size_t)(N * K) * sizeof(double));
  int rc = ORC_OK;
  if (!qp || !qs || !xa || !w) {
    rc = ORC_EARG;
    goto done;
  }
  for (int64_t e = 0; e < E; ++e) {
    int64_t lo = e == 0 ? 0 : offs[e - 1], hi = offs[e];
    int have = 0;
    for (int64_t i = 0; i < nrows && !have; ++i) have = rows[i] >= lo && rows[i] < hi;
    if (!have) continue;
    const uint8_t* pe = packed + e * N * (K / 2);
    const uint8_t* se = scales + e * N * (K / 32);
    for (int64_t n = 0; n < N; ++n)
      for (int64_t k = 0; k < K; ++k) w[n * K + k] = mx_element(pe, se, K, n, k);
    for (int64_t i = 0; i < nrows; ++i) {
      int64_t t = rows[i];
      if (t < lo || t >= hi) continue;
      orc_mx_quantize(x + t * K, ORC_BF16, 1, K, qp, qs);
      for (int64_t k = 0; k < K; ++k) xa[k] = mx_element(qp, qs, K, 0, k);
      for (int64_t n = 0; n < N; ++n) {
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) acc += xa[k] * w[n * K + k];
        out[i * N + n] = acc;
      }
    }
  }
done:
  free(qp);
  free(qs);
  free(xa);
  free(w);
  return rc;
}

/* ------------------------------------------------------------------------ */
/* W4A4 NVFP4 grouped GEMM ([MO] "W4A4 NVFP4 on FP4 tensor cores").          */
/* ------------------------------------------------------------------------ */

/* NVFP4 quantize of rows with a given per-tensor scale g (that of the
   whole tensor the rows belong to): the per-block steps of
   orc_nvfp4_quantize.  g == 0 (an all-zero tensor) gives codes 0 and block
   scales 1.0. */
int orc_nvfp4_quantize_rows(const void* x, int dtype, int64_t rows, int64_t K, double g,
                            uint8_t* packed, uint8_t* block_scales) {
  if (K % 16 != 0 || rows < 0) return ORC_EARG;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < K / 16; ++b) {
      int64_t base = r * K + b * 16;
      double amax_b = 0.0;
      for (int i = 0; i < 16; ++i) {
        double a = fabs(load_elem(x, dtype, base + i));
        if (a > amax_b) amax_b = a;
      }
      double s = g == 0.0 ? 1.0 : orc_nvfp4_block_scale(amax_b, g);
      block_scales[r * (K / 16) + b] = orc_encode_e4m3(s);
      double d = f32_mul(s, g);
      for (int j = 0; j < 8; ++j) {
        int nib[2] = {0, 0};
        for (int h = 0; h < 2 && g != 0.0; ++h) {
          double xi = load_elem(x, dtype, base + 2 * j + h);
          nib[h] = (orc_e2m1_code(fabs(f32_div(xi, d))) & 7) | (xi < 0.0 ? 8 : 0);
        }
        packed[r * (K / 2) + b * 8 + j] = (uint8_t)(nib[0] | (nib[1] << 4));
      }
    }
  }
  return ORC_OK;
}

/* Value of NVFP4 element k of a row: E2M1 code * E4M3 block scale * g,
   exact in double. */
static double nv_element(const uint8_t* packed_row, const uint8_t* scales_row, int64_t k,
                         double g) {
  uint8_t byte = packed_row[k / 2];
  int nib = (k % 2 == 0) ? (byte & 15) : (byte >> 4);
  return E2M1_TABLE[nib] * orc_decode_e4m3(scales_row[k / 16]) * g;
}

/* x: bf16 [T, K] activations, NVFP4-quantized as one tensor (its global
   scale from max |x| over all of x), then dequantized exactly; weights:
   packed [E, N, K/2], E4M3 block scales [E, N, K/16] and one global scale
   per expert.  out[i][n] = sum_k deq(q(x))[t][k] * deq(W_e)[n][k] for t =
   rows[i], summed in double in index order (not rounded). */
int orc_nvfp4_w4a4_grouped_mm(const uint16_t* x, const uint8_t* packed, const uint8_t* bscales,
                              const float* w_global, const int32_t* offs, int64_t T, int64_t E,
                              int64_t N, int64_t K, const int64_t* rows, int64_t nrows,
                              double* out) {
  if (E < 1 || K % 16 != 0 || N < 1 || T < 0) return ORC_EARG;
  if (orc_check_offs(offs, E, T) != ORC_OK) return ORC_EOFFS;
  double amax = 0.0;
  for (int64_t i = 0; i < T * K; ++i) {
    double a = fabs(decode_bf16(x[i]));
    if (a > amax) amax = a;
  }
  double gx = amax == 0.0 ? 0.0 : orc_nvfp4_global_scale(amax);
  uint8_t* qp = (uint8_t*)malloc((size_t)(K / 2));
  uint8_t* qs = (uint8_t*)malloc((size_t)(K / 16));
  double* xa = (double*)malloc((size_t)K * sizeof(double));
  double* w = (double*)malloc((size_t)(N * K) * sizeof(double));
  int rc = ORC_OK;
  if (!qp || !qs || !xa || !w) {
    rc = ORC_EARG;
    goto done;
  }
  for (int64_t e = 0; e < E; ++e) {
    int64_t lo = e == 0 ? 0 : offs[e - 1], hi = offs[e];
    int have = 0;
    for (int64_t i = 0; i < nrows && !have; ++i) have = rows[i] >= lo && rows[i] < hi;
    if (!have) continue;
    for (int64_t n = 0; n < N; ++n)
      for (int64_t k = 0; k < K; ++k)
        w[n * K + k] = nv_element(packed + (e * N + n) * (K / 2), bscales + (e * N + n) * (K / 16),
                                  k, (double)w_global[e]);
    for (int64_t i = 0; i < nrows; ++i) {
      int64_t t = rows[i];
      if (t < lo || t >= hi) continue;
      orc_nvfp4_quantize_rows(x + t * K, ORC_BF16, 1, K, gx, qp, qs);
      for (int64_t k = 0; k < K; ++k) xa[k] = nv_element(qp, qs, k, gx);
      for (int64_t n = 0; n < N; ++n) {
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) acc += xa[k] * w[n * K + k];
        out[i * N + n] = acc;
      }
    }
  }
done:
  free(qp);
  free(qs);
  free(xa);
  free(w);
  return rc;
}
