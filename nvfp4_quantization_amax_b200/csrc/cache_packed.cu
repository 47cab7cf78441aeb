// Packed (stored) form of the cache quantization, and its unpack, for
// sm_100a.
//
// quantize_cache rounds each group of B channels to fp8 or fp4 codes times a
// power-of-two scale 2^k and immediately multiplies back.  These kernels
// keep what that rounding produced instead: the element codes (one E4M3
// byte per element for fp8; two E2M1 nibbles per byte for mxfp4/nvfp4, the
// even channel in the low nibble) and one scale byte per group (E8M0, value
// 2^(byte-127), for fp8 and mxfp4; the E4M3 encoding of 2^k for nvfp4).
// Unpacking multiplies code by scale in f32 and rounds once to the output
// dtype, which is the arithmetic of the fake quantization, so
// unpack(pack(x)) equals quantize_cache(x) bit for bit.
//
// Layout of the fast kernels as in the fake-quantization kernel: an item is
// 8 consecutive channels (one 16-byte bf16/f16 load), B/8 lanes of a warp
// share one group and combine its maximum with xor-shuffles.
//
// Page references (title, then section):
//  "nemo_automodel.components.models.deepseek_v41.quantization":
//   _CacheQuantization.forward (fp8; mxfp4 with E8M0 scale; nvfp4 with E4M3
//   scale), quantize_cache, _power_of_two_ceiling.
//  "nemo_automodel.components.quantization.mxfp4": module docstring (low
//   nibble = even column).
#include "mxq.h"
#include "mxq_device.cuh"
#include "mxq_launch.h"

namespace mxq {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

template <int FMT>
struct PackedFormat;
template <>
struct PackedFormat<MXQ_FMT_FP8> {
  static constexpr int kLo = -126, kHi = 127, kQExp = 8;
  static constexpr uint32_t kQFrac = 0x600000u;  // 448 = 1.75 * 2^8
};
template <>
struct PackedFormat<MXQ_FMT_MXFP4> {
  static constexpr int kLo = -126, kHi = 127, kQExp = 2;
  static constexpr uint32_t kQFrac = 0x400000u;  // 6 = 1.5 * 2^2
};
template <>
struct PackedFormat<MXQ_FMT_NVFP4> {
  static constexpr int kLo = -9, kHi = 8, kQExp = 2;
  static constexpr uint32_t kQFrac = 0x400000u;
};

// Least k with 2^k * qmax >= amax, clamped to the format's range.
template <int FMT>
__device__ __forceinline__ int group_scale_exp(uint32_t amax_f32bits) {
  using F = PackedFormat<FMT>;
  if (amax_f32bits == 0) return F::kLo;
  int k = floor_log2_f32bits(amax_f32bits) - F::kQExp +
          (frac23_f32bits(amax_f32bits) > F::kQFrac ? 1 : 0);
  return k < F::kLo ? F::kLo : (k > F::kHi ? F::kHi : k);
}

// Scale byte of 2^k.  E4M3 of 2^k, k in [-9, 8]: subnormal 2^(k+9) / 2^-9
// steps below 2^-6, biased exponent (k + 7) above.
template <int FMT>
__device__ __forceinline__ uint32_t scale_byte(int k) {
  if constexpr (FMT == MXQ_FMT_NVFP4) {
    return k >= -6 ? (uint32_t)(k + 7) << 3 : 1u << (k + 9);
  } else {
    return (uint32_t)(k + 127);
  }
}

template <int FMT>
__device__ __forceinline__ float scale_value(uint32_t byte) {
  if constexpr (FMT == MXQ_FMT_NVFP4) {
    return f16lo(e4m3x2_to_f16x2(byte));
  } else {
    return byte == 0xFFu ? __uint_as_float(0x7FC00000u) : exp2i((int)byte - 127);
  }
}

// Element codes of eight values x * 2^-k.  fp8: E4M3 (sign of zero kept);
// fp4: E2M1 with the sign bit iff x < 0 (fmaf(x, inv, +0) turns -0 into +0
// and keeps the sign of a negative product that underflows).
template <int FMT>
__device__ __forceinline__ uint2 encode8(const float* x, float inv) {
  if constexpr (FMT == MXQ_FMT_FP8) {
    uint32_t b[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) b[j] = e4m3x2(x[2 * j] * inv, x[2 * j + 1] * inv);
    return make_uint2(b[0] | (b[1] << 16), b[2] | (b[3] << 16));
  } else {
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = fmaf(x[j], inv, 0.0f);
    return make_uint2(e2m1x8(v), 0u);
  }
}

// Eight decoded values (code times scale, exact in f32).
template <int FMT>
__device__ __forceinline__ void decode8(uint2 c, float s, float* v) {
  if constexpr (FMT == MXQ_FMT_FP8) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t w = j < 2 ? c.x : c.y;
      const uint32_t h2 = e4m3x2_to_f16x2((w >> (16 * (j & 1))) & 0xFFFFu);
      v[2 * j] = f16lo(h2) * s;
      v[2 * j + 1] = f16hi(h2) * s;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t h2 = e2m1x2_to_f16x2((c.x >> (8 * j)) & 0xFFu);
      v[2 * j] = fmaf(f16lo(h2), s, 0.0f);  // zero magnitudes give +0
      v[2 * j + 1] = fmaf(f16hi(h2), s, 0.0f);
    }
  }
}

template <int FMT>
__device__ __forceinline__ void store_codes(void* codes, int64_t item, uint2 c) {
  if constexpr (FMT == MXQ_FMT_FP8) {
    *(uint2*)((char*)codes + item * 8) = c;
  } else {
    *(uint32_t*)((char*)codes + item * 4) = c.x;
  }
}

template <int FMT>
__device__ __forceinline__ uint2 load_codes(const void* codes, int64_t item) {
  if constexpr (FMT == MXQ_FMT_FP8) {
    return __ldg((const uint2*)((const char*)codes + item * 8));
  } else {
    return make_uint2(__ldg((const uint32_t*)((const char*)codes + item * 4)), 0u);
  }
}

template <int DT, int FMT, int LPB>
__global__ void __launch_bounds__(kThreads)
pack_cache_kernel(const void* __restrict__ in, void* __restrict__ codes,
                  uint8_t* __restrict__ scales, int64_t n_items) {
  const int lane = threadIdx.x & 31;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t base = (int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31); base < n_items;
       base += stride * kUnroll) {
    uint32_t bits[kUnroll][8];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t item = base + u * stride + lane;
      if (item < n_items && MXQ_IN_RANGE(kChkPackIn, item, n_items)) load8<DT>(in, item, bits[u]);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t item = base + u * stride + lane;
      const bool valid = item < n_items;
      uint32_t m = 0;
      if (valid) {
#pragma unroll
        for (int j = 0; j < 8; ++j) m = max(m, mag_as_f32_bits<DT>(bits[u][j]));
      }
#pragma unroll
      for (int o = 1; o < LPB; o <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (!valid) continue;
      const int k = group_scale_exp<FMT>(m);
      float x[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) x[j] = elem_to_f32<DT>(bits[u][j]);
      if (MXQ_IN_RANGE(kChkPackOut, item, n_items))
        store_codes<FMT>(codes, item, encode8<FMT>(x, exp2i(-k)));
      if ((lane & (LPB - 1)) == 0 && MXQ_IN_RANGE(kChkPackScale, item / LPB, n_items / LPB))
        scales[item / LPB] = (uint8_t)scale_byte<FMT>(k);
    }
  }
}

template <int DT, int FMT, int LPB>
__global__ void __launch_bounds__(kThreads)
unpack_cache_kernel(const void* __restrict__ codes, const uint8_t* __restrict__ scales,
                    void* __restrict__ out, int64_t n_items) {
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t base = (int64_t)blockIdx.x * kThreads + threadIdx.x; base < n_items;
       base += stride * kUnroll) {
    uint2 c[kUnroll];
    uint32_t sb[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t item = base + u * stride;
      if (item < n_items) {
        c[u] = MXQ_IN_RANGE(kChkUnpackIn, item, n_items) ? load_codes<FMT>(codes, item)
                                                         : make_uint2(0u, 0u);
        sb[u] = MXQ_IN_RANGE(kChkUnpackScale, item / LPB, n_items / LPB)
                    ? (uint32_t)__ldg(scales + item / LPB)
                    : 0u;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t item = base + u * stride;
      if (item >= n_items) continue;
      float v[8];
      decode8<FMT>(c[u], scale_value<FMT>(sb[u]), v);
      if (MXQ_IN_RANGE(kChkUnpackOut, item, n_items)) store8<DT>(out, item, v);
    }
  }
}

// General kernels: any block size the format allows (even for fp4), any
// alignment; channels % B == 0.  One thread per (row, group).
template <int DT>
__device__ __forceinline__ uint32_t elem_bits_at(const void* p, int64_t i) {
  if constexpr (ElemTraits<DT>::kBytes == 2) return ((const uint16_t*)p)[i];
  else return ((const uint32_t*)p)[i];
}

template <int DT>
__device__ __forceinline__ void store_one(void* p, int64_t i, float v) {
  if constexpr (ElemTraits<DT>::kBytes == 2) ((uint16_t*)p)[i] = pack2<DT>(v, 0.0f) & 0xFFFFu;
  else ((float*)p)[i] = v;
}

template <int DT, int FMT>
__global__ void __launch_bounds__(kThreads)
pack_cache_general_kernel(const void* __restrict__ in, uint8_t* __restrict__ codes,
                          uint8_t* __restrict__ scales, int64_t n_groups, int B) {
  for (int64_t g = (int64_t)blockIdx.x * kThreads + threadIdx.x; g < n_groups;
       g += (int64_t)gridDim.x * kThreads) {
    const int64_t c0 = g * B;  // groups never straddle rows (channels % B == 0)
    [[maybe_unused]] const int64_t n_el = n_groups * B;
    auto elem = [&](int64_t i) {
      return MXQ_IN_RANGE(kChkPackIn, i, n_el) ? elem_bits_at<DT>(in, i) : 0u;
    };
    uint32_t m = 0;
    for (int c = 0; c < B; ++c) m = max(m, mag_as_f32_bits<DT>(elem(c0 + c)));
    const int k = group_scale_exp<FMT>(m);
    const float inv = exp2i(-k);
    if (MXQ_IN_RANGE(kChkPackScale, g, n_groups)) scales[g] = (uint8_t)scale_byte<FMT>(k);
    for (int c = 0; c < B; c += 2) {
      const float a = elem_to_f32<DT>(elem(c0 + c));
      const float b = c + 1 < B ? elem_to_f32<DT>(elem(c0 + c + 1)) : 0.0f;
      if constexpr (FMT == MXQ_FMT_FP8) {
        const uint32_t two = e4m3x2(a * inv, b * inv);
        if (MXQ_IN_RANGE(kChkPackOut, c0 + c, n_el)) codes[c0 + c] = (uint8_t)two;
        if (c + 1 < B && MXQ_IN_RANGE(kChkPackOut, c0 + c + 1, n_el))
          codes[c0 + c + 1] = (uint8_t)(two >> 8);
      } else {
        if (MXQ_IN_RANGE(kChkPackOut, (c0 + c) / 2, n_el / 2))
          codes[(c0 + c) / 2] = (uint8_t)e2m1x2(fmaf(a, inv, 0.0f), fmaf(b, inv, 0.0f));
      }
    }
  }
}

template <int DT, int FMT>
__global__ void __launch_bounds__(kThreads)
unpack_cache_general_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                            void* __restrict__ out, int64_t n_groups, int B) {
  for (int64_t g = (int64_t)blockIdx.x * kThreads + threadIdx.x; g < n_groups;
       g += (int64_t)gridDim.x * kThreads) {
    const int64_t c0 = g * B;
    [[maybe_unused]] const int64_t n_el = n_groups * B;
    const float s = scale_value<FMT>(MXQ_IN_RANGE(kChkUnpackScale, g, n_groups) ? scales[g] : 0u);
    for (int c = 0; c < B; ++c) {
      float v;
      if constexpr (FMT == MXQ_FMT_FP8) {
        v = f16lo(e4m3x2_to_f16x2(MXQ_IN_RANGE(kChkUnpackIn, c0 + c, n_el) ? codes[c0 + c] : 0u)) *
            s;
      } else {
        const uint32_t byte =
            MXQ_IN_RANGE(kChkUnpackIn, (c0 + c) / 2, n_el / 2) ? codes[(c0 + c) / 2] : 0u;
        const uint32_t h2 = e2m1x2_to_f16x2(((c0 + c) & 1) ? (byte >> 4) : (byte & 15u));
        v = fmaf(f16lo(h2), s, 0.0f);
      }
      if (MXQ_IN_RANGE(kChkUnpackOut, c0 + c, n_el)) store_one<DT>(out, c0 + c, v);
    }
  }
}

template <class Kernel>
int grid_over(Kernel kernel, int64_t n_units, int per_block) {
  return wave_grid((const void*)kernel, kThreads, n_units, per_block);
}

template <int DT, int FMT, int LPB>
void launch_fast(const void* in, void* codes, uint8_t* scales, void* out, bool pack,
                 int64_t n_items, cudaStream_t st) {
  const int per = kThreads * kUnroll;
  if (pack)
    pack_cache_kernel<DT, FMT, LPB><<<grid_over(pack_cache_kernel<DT, FMT, LPB>, n_items, per),
                                      kThreads, 0, st>>>(in, codes, scales, n_items);
  else
    unpack_cache_kernel<DT, FMT, LPB><<<grid_over(unpack_cache_kernel<DT, FMT, LPB>, n_items, per),
                                        kThreads, 0, st>>>(codes, scales, out, n_items);
}

template <int DT, int FMT>
void launch_fmt(const void* in, void* codes, uint8_t* scales, void* out, bool pack, int64_t rows,
                int64_t C, int B, bool fast, cudaStream_t st) {
  if (fast) {
    const int64_t n = rows * (C / 8);
    switch (B / 8) {
      case 1: launch_fast<DT, FMT, 1>(in, codes, scales, out, pack, n, st); break;
      case 2: launch_fast<DT, FMT, 2>(in, codes, scales, out, pack, n, st); break;
      case 4: launch_fast<DT, FMT, 4>(in, codes, scales, out, pack, n, st); break;
      case 8: launch_fast<DT, FMT, 8>(in, codes, scales, out, pack, n, st); break;
      case 16: launch_fast<DT, FMT, 16>(in, codes, scales, out, pack, n, st); break;
      default: launch_fast<DT, FMT, 32>(in, codes, scales, out, pack, n, st); break;
    }
    return;
  }
  const int64_t n_groups = rows * (C / B);
  if (pack)
    pack_cache_general_kernel<DT, FMT>
        <<<grid_over(pack_cache_general_kernel<DT, FMT>, n_groups, kThreads), kThreads, 0, st>>>(
            in, (uint8_t*)codes, scales, n_groups, B);
  else
    unpack_cache_general_kernel<DT, FMT>
        <<<grid_over(unpack_cache_general_kernel<DT, FMT>, n_groups, kThreads), kThreads, 0, st>>>(
            (const uint8_t*)codes, scales, out, n_groups, B);
}

template <int DT>
void launch_dt(const void* in, void* codes, uint8_t* scales, void* out, bool pack, int64_t rows,
               int64_t C, int fmt, int B, bool fast, cudaStream_t st) {
  switch (fmt) {
    case MXQ_FMT_FP8:
      launch_fmt<DT, MXQ_FMT_FP8>(in, codes, scales, out, pack, rows, C, B, fast, st);
      break;
    case MXQ_FMT_MXFP4:
      launch_fmt<DT, MXQ_FMT_MXFP4>(in, codes, scales, out, pack, rows, C, B, fast, st);
      break;
    default:
      launch_fmt<DT, MXQ_FMT_NVFP4>(in, codes, scales, out, pack, rows, C, B, fast, st);
      break;
  }
}

int launch_packed(const void* in, void* codes, uint8_t* scales, void* out, bool pack, int dt,
                  int64_t rows, int64_t C, int fmt, int B, bool fast, cudaStream_t st) {
  switch (dt) {
    case kBF16: launch_dt<kBF16>(in, codes, scales, out, pack, rows, C, fmt, B, fast, st); break;
    case kF16: launch_dt<kF16>(in, codes, scales, out, pack, rows, C, fmt, B, fast, st); break;
    default: launch_dt<kF32>(in, codes, scales, out, pack, rows, C, fmt, B, fast, st); break;
  }
  return cudaGetLastError() == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

}  // namespace

int launch_quantize_cache_packed(const void* in, int dt, int64_t rows, int64_t C, int fmt, int B,
                                 void* codes, void* scales, bool fast, cudaStream_t st) {
  return launch_packed(in, codes, (uint8_t*)scales, nullptr, true, dt, rows, C, fmt, B, fast, st);
}

int launch_dequantize_cache_packed(const void* codes, const void* scales, int64_t rows, int64_t C,
                                   int fmt, int B, void* out, int dt, bool fast, cudaStream_t st) {
  return launch_packed(nullptr, const_cast<void*>(codes), (uint8_t*)const_cast<void*>(scales),
                       out, false, dt, rows, C, fmt, B, fast, st);
}

MXQ_DEFINE_CHECK_READER(check_record_cache_packed)

}  // namespace mxq
