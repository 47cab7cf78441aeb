// Device-side building blocks shared by the mxq kernels (sm_100a only).
//
// Number formats: bf16 / f16 / f32 elements; E2M1 (4-bit: sign, 2 exponent
// bits, 1 mantissa bit, values {0,0.5,1,1.5,2,3,4,6}); E4M3 (8-bit "fn"
// flavour, finite max 448); E8M0 scale bytes (2^(byte-127)).
//
// Conversions to E2M1 / E4M3 use the sm_100a cvt instructions, which round
// to nearest-even and (with .satfinite) clamp to the largest finite value:
// the E2M1 grid rule of "NVIDIA Model Optimizer: from mtq.quantize to a
// 4.95-bit DeepSeek-R1" (section "NVFP4 in the code: two scales and a
// nibble": ties at 0.75, 1.75, 3.5 go up, i.e. half-to-even on the grid).
// Scale arithmetic is done on exponent fields, so no division, log or exp
// is ever evaluated.  Nothing here flushes subnormals: the library is built
// without fast-math and every float multiply used is exact.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "mxq.h"

namespace mxq {

constexpr int kBF16 = MXQ_BF16;
constexpr int kF16 = MXQ_F16;
constexpr int kF32 = MXQ_F32;

// ---------------------------------------------------- debug index checks
//
// The library's debug variant is built with -DMXQ_DEBUG_CHECKS.  There every
// checked global-memory access first tests its element index against the
// extent the kernel was launched for; a failed test records (check id,
// index, extent) in this translation unit's record (the first failure
// wins; a host reader per unit returns and clears it) and the access is
// skipped, so nothing traps and no out-of-range address is touched.  In the
// normal build a check is the constant true and compiles away.
enum MxqCheckId {
  kChkMxQuantIn = 1, kChkMxQuantOut, kChkMxQuantScale,
  kChkMxDeqIn, kChkMxDeqScale, kChkMxDeqOut,
  kChkCacheIn, kChkCacheOut, kChkCacheGenIn, kChkCacheGenOut,
  kChkNvAmaxIn, kChkNvQuantIn, kChkNvQuantOut, kChkNvQuantScale,
  kChkNvDeqIn, kChkNvDeqScale, kChkNvDeqOut,
  kChkMseIn, kChkMseOut, kChkMseScale,
  kChkPackIn, kChkPackOut, kChkPackScale, kChkUnpackIn, kChkUnpackScale, kChkUnpackOut,
  kChkGemmGenIn, kChkGemmGenW, kChkGemmGenOut,
  kChkGemmTcOut, kChkGemmTcScale, kChkGemmTcSmem, kChkGemmTcTmem,
  kChkW4Out, kChkW4Scale, kChkW4Smem, kChkGemmTcW,
  kChkSelfTest = 99
};

#ifdef MXQ_DEBUG_CHECKS
static __device__ unsigned long long g_mxq_check_record[3];
__device__ __forceinline__ bool mxq_in_range(int id, int64_t i, int64_t n) {
  if (i >= 0 && i < n) return true;
  if (atomicCAS(&g_mxq_check_record[0], 0ull, (unsigned long long)id) == 0ull) {
    g_mxq_check_record[1] = (unsigned long long)i;
    g_mxq_check_record[2] = (unsigned long long)n;
  }
  return false;
}
#define MXQ_IN_RANGE(id, i, n) ::mxq::mxq_in_range((id), (int64_t)(i), (int64_t)(n))
// Host reader of this unit's record: copies it to out[3], then clears it.
#define MXQ_DEFINE_CHECK_READER(fn)                                                    \
  int fn(unsigned long long* out) {                                                    \
    if (cudaMemcpyFromSymbol(out, g_mxq_check_record, 3 * sizeof(unsigned long long)) != \
        cudaSuccess)                                                                   \
      return MXQ_ERR_CUDA;                                                             \
    const unsigned long long zero[3] = {0ull, 0ull, 0ull};                             \
    return cudaMemcpyToSymbol(g_mxq_check_record, zero, sizeof(zero)) == cudaSuccess   \
               ? MXQ_OK                                                                \
               : MXQ_ERR_CUDA;                                                         \
  }
#else
#define MXQ_IN_RANGE(id, i, n) true
#define MXQ_DEFINE_CHECK_READER(fn) \
  int fn(unsigned long long* out) { \
    out[0] = out[1] = out[2] = 0ull; \
    return MXQ_ERR_UNSUPPORTED;      \
  }
#endif

// ---------------------------------------------------------------- memory

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ld_stream_u8(const void* p) {
  uint16_t r;
  asm volatile("ld.global.nc.u8 %0, [%1];" : "=h"(r) : "l"(p));
  return r;
}
__device__ __forceinline__ void st_v4(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// ------------------------------------------------------ element <-> f32

// Magnitude bits of an element widened to the f32 bit pattern of |x|
// (exact: bf16 is the top half of f32, f16 values are all f32 values).
template <int DT>
__device__ __forceinline__ uint32_t mag_as_f32_bits(uint32_t bits) {
  if constexpr (DT == kBF16) {
    return (bits & 0x7FFFu) << 16;
  } else if constexpr (DT == kF16) {
    float f = __half2float(__ushort_as_half((unsigned short)(bits & 0x7FFFu)));
    return __float_as_uint(f);
  } else {
    return bits & 0x7FFFFFFFu;
  }
}

template <int DT>
__device__ __forceinline__ float elem_to_f32(uint32_t bits) {
  if constexpr (DT == kBF16) {
    return __uint_as_float(bits << 16);
  } else if constexpr (DT == kF16) {
    return __half2float(__ushort_as_half((unsigned short)bits));
  } else {
    return __uint_as_float(bits);
  }
}

// Two f32 -> two elements of DT packed in a u32 (lo = a), nearest-even.
template <int DT>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  uint32_t r;
  if constexpr (DT == kBF16) {
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  } else {
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  }
  return r;
}

// Two binary32 products, or two fmas with a +0 addend, in one instruction
// (sm_100 mul / fma .rn.f32x2): each lane is rounded exactly as the scalar
// operation (mul.rn / fma.rn) rounds it, subnormals kept.
__device__ __forceinline__ void mul2_rn(float& y0, float& y1, float a0, float a1, float b0,
                                        float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\t"
      "mov.b64 a, {%2, %3};\n\t"
      "mov.b64 b, {%4, %5};\n\t"
      "mul.rn.f32x2 d, a, b;\n\t"
      "mov.b64 {%0, %1}, d;\n\t}"
      : "=f"(y0), "=f"(y1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
// y = a * b + 0 per lane: a zero product becomes +0, as fmaf(a, b, 0.0f).
__device__ __forceinline__ void fma2_rn_zero(float& y0, float& y1, float a0, float a1, float b0,
                                             float b1) {
  asm("{\n\t.reg .b64 a, b, c, d;\n\t"
      "mov.b64 a, {%2, %3};\n\t"
      "mov.b64 b, {%4, %5};\n\t"
      "mov.b64 c, 0;\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\t"
      "mov.b64 {%0, %1}, d;\n\t}"
      : "=f"(y0), "=f"(y1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// ---------------------------------------------------------- exponents

// floor(log2 v) of a positive finite f32 given by its bit pattern
// (subnormals included).
__device__ __forceinline__ int floor_log2_f32bits(uint32_t u) {
  int ef = (int)(u >> 23);
  if (ef > 0) return ef - 127;
  return (31 - __clz((int)u)) - 149;
}

// 23-bit fraction of the normalised significand of a positive f32.
__device__ __forceinline__ uint32_t frac23_f32bits(uint32_t u) {
  if ((u >> 23) > 0) return u & 0x7FFFFFu;
  int p = 31 - __clz((int)u);
  return (u << (23 - p)) & 0x7FFFFFu;
}

// 2^e as f32 for e in [-149, 127].
__device__ __forceinline__ float exp2i(int e) {
  if (e >= -126) return __uint_as_float((uint32_t)(e + 127) << 23);
  return __uint_as_float(1u << (e + 149));
}

// ---------------------------------------------------- E2M1 / E4M3 casts

// Two f32 -> one byte of E2M1 codes (a in the low nibble), nearest-even,
// saturating at +-6; the sign nibble bit follows the sign bit of the input.
__device__ __forceinline__ uint32_t e2m1x2(float a, float b) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(a), "f"(b));
  return r;
}

// E2M1 codes of the eight binary32 quotients w_j / d by IEEE division
// (element 2j in the low nibble of byte j): the rare path of e2m1x8_quot,
// inlined (as a call it cost the mse sweep 4 %).
static __device__ __forceinline__ uint32_t e2m1x8_div(float w0, float w1, float w2, float w3,
                                                   float w4, float w5, float w6, float w7,
                                                   float d) {
  return e2m1x2(__fdiv_rn(w0, d), __fdiv_rn(w1, d)) |
         (e2m1x2(__fdiv_rn(w2, d), __fdiv_rn(w3, d)) << 8) |
         (e2m1x2(__fdiv_rn(w4, d), __fdiv_rn(w5, d)) << 16) |
         (e2m1x2(__fdiv_rn(w6, d), __fdiv_rn(w7, d)) << 24);
}

// Bracket factors of a divisor d in [2^-126, 2^126) (quot_fast_ok):
// r = fl(1 / d), r_lo = fl(r (1 - 2^-19)), r_hi = fl(r (1 + 2^-19)).
__device__ __forceinline__ void bracket_factors(float d, float& r_lo, float& r_hi) {
  const float r = __frcp_rn(d);
  r_lo = r * (1.0f - 0x1p-19f);
  r_hi = r * (1.0f + 0x1p-19f);
}

// The codes of e2m1x8_div, with the divisions only where they can matter.
// For the rounded quotient v = fl(w / d), the products w * r_lo and
// w * r_hi (binary32) each lie within 5 * 2^-24 (relative) of
// v (1 -+ 2^-19), so they bracket v from below and above in magnitude, with
// its sign.  The cast to E2M1 is monotone, so where it gives the same codes
// at both ends of the brackets it gives them for v too; otherwise some
// quotient lies within ~2^-19 of an E2M1 decision point and the IEEE
// divisions decide.  Quotients near the binary32 underflow threshold are far
// below the first decision point (0.25): every end then casts to a zero
// magnitude with the sign of w, as v does.
__device__ __forceinline__ uint32_t e2m1x8_quot(const float* w, float d, float r_lo, float r_hi) {
  uint32_t a = 0, b = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float l0, l1, h0, h1;
    mul2_rn(l0, l1, w[2 * j], w[2 * j + 1], r_lo, r_lo);
    mul2_rn(h0, h1, w[2 * j], w[2 * j + 1], r_hi, r_hi);
    a |= e2m1x2(l0, l1) << (8 * j);
    b |= e2m1x2(h0, h1) << (8 * j);
  }
  return a == b ? a : e2m1x8_div(w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7], d);
}

__device__ __forceinline__ uint32_t e2m1x8_quot(const float* w, float d) {
  float r_lo, r_hi;
  bracket_factors(d, r_lo, r_hi);
  return e2m1x8_quot(w, d, r_lo, r_hi);
}

// Whether the bracket (e2m1x8_quot) may be used with divisor d: then r is
// a normal number.
__device__ __forceinline__ bool quot_fast_ok(float d) {
  return d >= 0x1p-126f && d < 0x1p126f;
}

// Eight f32 -> four bytes of E2M1 codes, element 2j in the low nibble of
// byte j.
__device__ __forceinline__ uint32_t e2m1x8(const float* v) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
        "f"(v[7]));
  return r;
}

// One byte of two E2M1 codes -> two exact f16 values (low nibble -> low half).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.u8.u32 t, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(r)
      : "r"(byte));
  return r;
}

// Two f32 -> two E4M3 bytes in a u16 (a in the low byte), nearest-even,
// saturating at +-448, sign of zero kept.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(r) : "f"(a), "f"(b));
  return r;
}

// Two E4M3 bytes (low byte first) -> two exact f16 values.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"((uint16_t)two));
  return r;
}

__device__ __forceinline__ float f16lo(uint32_t h2) {
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}
__device__ __forceinline__ float f16hi(uint32_t h2) {
  return __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
}

// ------------------------------------------------------------- helpers

template <int DT>
struct ElemTraits;
template <>
struct ElemTraits<kBF16> {
  static constexpr int kBytes = 2;
  static constexpr uint32_t kNaN = 0x7FC0u;
};
template <>
struct ElemTraits<kF16> {
  static constexpr int kBytes = 2;
  static constexpr uint32_t kNaN = 0x7E00u;
};
template <>
struct ElemTraits<kF32> {
  static constexpr int kBytes = 4;
  static constexpr uint32_t kNaN = 0x7FC00000u;
};

// Load 8 consecutive elements of DT as 8 raw bit patterns.
template <int DT>
__device__ __forceinline__ void load8(const void* base, int64_t item, uint32_t* bits) {
  if constexpr (ElemTraits<DT>::kBytes == 2) {
    uint4 v = ld_stream_v4((const char*)base + item * 16);
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      bits[2 * j] = w[j] & 0xFFFFu;
      bits[2 * j + 1] = w[j] >> 16;
    }
  } else {
    uint4 v0 = ld_stream_v4((const char*)base + item * 32);
    uint4 v1 = ld_stream_v4((const char*)base + item * 32 + 16);
    bits[0] = v0.x; bits[1] = v0.y; bits[2] = v0.z; bits[3] = v0.w;
    bits[4] = v1.x; bits[5] = v1.y; bits[6] = v1.z; bits[7] = v1.w;
  }
}

// Store 8 f32 values (already exact or to be rounded) as DT.
template <int DT>
__device__ __forceinline__ void store8(void* base, int64_t item, const float* v) {
  if constexpr (ElemTraits<DT>::kBytes == 2) {
    uint4 o;
    o.x = pack2<DT>(v[0], v[1]);
    o.y = pack2<DT>(v[2], v[3]);
    o.z = pack2<DT>(v[4], v[5]);
    o.w = pack2<DT>(v[6], v[7]);
    st_v4((char*)base + item * 16, o);
  } else {
    st_v4((char*)base + item * 32,
          make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                     __float_as_uint(v[3])));
    st_v4((char*)base + item * 32 + 16,
          make_uint4(__float_as_uint(v[4]), __float_as_uint(v[5]), __float_as_uint(v[6]),
                     __float_as_uint(v[7])));
  }
}

template <int DT>
__device__ __forceinline__ void store8_bits(void* base, int64_t item, uint32_t bits) {
  if constexpr (ElemTraits<DT>::kBytes == 2) {
    uint32_t w = bits | (bits << 16);
    st_v4((char*)base + item * 16, make_uint4(w, w, w, w));
  } else {
    st_v4((char*)base + item * 32, make_uint4(bits, bits, bits, bits));
    st_v4((char*)base + item * 32 + 16, make_uint4(bits, bits, bits, bits));
  }
}

}  // namespace mxq
