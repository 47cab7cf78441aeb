// HBM-bound kernels: MXFP4 pack (mx_quantize), MXFP4 unpack (mx_dequantize)
// and cache fake quantization (quantize_cache) for sm_100a.
//
// All three are streaming passes.  The work unit ("item") is 8 consecutive
// elements of one row: one 16-byte load of bf16/f16 input.  The pack gives
// each lane one whole 32-element block (four items, loads kept in L1), so a
// block's maximum, scale, code bytes and scale byte need no exchange between
// lanes.  In the unpack and the cache fake quantization a block of B
// channels is B/8 consecutive items, handled by B/8 consecutive lanes of one
// warp, which combine their block maximum with xor-shuffles; each thread
// keeps kUnroll independent items in flight (coalesced 16-byte loads with
// L1 no-allocate).  The grid is a whole number of waves over the SMs.
//
// Page references (title, then section):
//  "nemo_automodel.components.quantization.mxfp4": quantize_mxfp4 (scale
//   2^(floor(log2 amax) - 2), K % 32), dequantize_mxfp4, module docstring
//   (low nibble = even column, one E8M0 scale per 32 columns).
//  "nemo_automodel.components.models.deepseek_v41.quantization":
//   quantize_cache (formats, block sizes, zero-padded tail group),
//   _power_of_two_ceiling.
#include "mxq_device.cuh"
#include "mxq_launch.h"

namespace mxq {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

// Eight consecutive elements as raw bits: one 16-byte vector for bf16/f16,
// two for f32.
template <int DT>
struct Raw8 {
  uint4 a, b;
};

template <int DT>
__device__ __forceinline__ Raw8<DT> load_raw8(const void* base, int64_t item) {
  Raw8<DT> r;
  if constexpr (ElemTraits<DT>::kBytes == 2) {
    r.a = ld_stream_v4((const char*)base + item * 16);
  } else {
    r.a = ld_stream_v4((const char*)base + item * 32);
    r.b = ld_stream_v4((const char*)base + item * 32 + 16);
  }
  return r;
}

// Bits of element j (0..7).
template <int DT>
__device__ __forceinline__ uint32_t raw_elem(const Raw8<DT>& r, int j) {
  if constexpr (ElemTraits<DT>::kBytes == 2) {
    const uint32_t w = j < 2 ? r.a.x : j < 4 ? r.a.y : j < 6 ? r.a.z : r.a.w;
    return (j & 1) ? (w >> 16) : (w & 0xFFFFu);
  } else {
    const uint4& q = j < 4 ? r.a : r.b;
    const int k = j & 3;
    return k == 0 ? q.x : k == 1 ? q.y : k == 2 ? q.z : q.w;
  }
}

// f32 bit pattern of max |x| over the eight elements.  For 16-bit formats
// the magnitudes are compared pairwise as unsigned halves (monotone in |x|
// for finite values).
template <int DT>
__device__ __forceinline__ uint32_t raw_amax(const Raw8<DT>& r) {
  if constexpr (ElemTraits<DT>::kBytes == 2) {
    const uint32_t M = 0x7FFF7FFFu;
    const uint32_t m2 = __vmaxu2(__vmaxu2(r.a.x & M, r.a.y & M), __vmaxu2(r.a.z & M, r.a.w & M));
    return mag_as_f32_bits<DT>(max(m2 & 0xFFFFu, m2 >> 16));
  } else {
    const uint32_t M = 0x7FFFFFFFu;
    const uint32_t m = max(max(max(r.a.x & M, r.a.y & M), max(r.a.z & M, r.a.w & M)),
                           max(max(r.b.x & M, r.b.y & M), max(r.b.z & M, r.b.w & M)));
    return m;
  }
}

// ---------------------------------------------------------- mx_quantize

// Scale exponent of quantize_mxfp4 from the f32 bit pattern of a block's
// amax: floor(log2 amax) - 2 clamped to [-127, 127]; zero -> -127.
__device__ __forceinline__ int mx_scale_exp(uint32_t amax_f32bits) {
  if (amax_f32bits == 0) return -127;
  int e = floor_log2_f32bits(amax_f32bits) - 2;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// A 32-element block of the pack's input: its four items, read with 16-byte
// loads kept in L1 (a lane's loads read the halves of the same sectors).
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
template <int DT>
__device__ __forceinline__ Raw8<DT> load_raw8_l1(const void* base, int64_t item) {
  Raw8<DT> r;
  if constexpr (ElemTraits<DT>::kBytes == 2) {
    r.a = ld_nc_v4((const char*)base + item * 16);
  } else {
    r.a = ld_nc_v4((const char*)base + item * 32);
    r.b = ld_nc_v4((const char*)base + item * 32 + 16);
  }
  return r;
}

// One iteration of the pack: each lane one 32-element block (four items) at
// base + lane, with its maximum, scale, 16 code bytes and scale byte.
template <int DT, bool kFull>
__device__ __forceinline__ void mx_quantize_block(const void* __restrict__ x,
                                                  uint4* __restrict__ packed,
                                                  uint8_t* __restrict__ scales, int64_t n_blocks,
                                                  int64_t blk) {
  if (!kFull && blk >= n_blocks) return;
  if (!MXQ_IN_RANGE(kChkMxQuantIn, 4 * blk + 3, 4 * n_blocks)) return;
  Raw8<DT> raw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) raw[i] = load_raw8_l1<DT>(x, 4 * blk + i);
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) m = max(m, raw_amax<DT>(raw[i]));
  const int e = mx_scale_exp(m);
  const float inv = exp2i(-e);  // exact power of two
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float v[8];
    // x * 2^-e is exact; adding +0 in the same rounding turns -0.0 into
    // +0.0 (no sign bit for it) while a negative value that underflows
    // keeps its sign, so the code's sign bit is set iff x < 0.
#pragma unroll
    for (int j = 0; j < 8; j += 2)
      fma2_rn_zero(v[j], v[j + 1], elem_to_f32<DT>(raw_elem<DT>(raw[i], j)),
                   elem_to_f32<DT>(raw_elem<DT>(raw[i], j + 1)), inv, inv);
    c[i] = e2m1x8(v);
  }
  if (MXQ_IN_RANGE(kChkMxQuantOut, 4 * blk + 3, 4 * n_blocks))
    packed[blk] = make_uint4(c[0], c[1], c[2], c[3]);
  if (MXQ_IN_RANGE(kChkMxQuantScale, blk, n_blocks)) scales[blk] = (uint8_t)(e + 127);
}

template <int DT>
__global__ void __launch_bounds__(kThreads)
mx_quantize_kernel(const void* __restrict__ x, uint32_t* __restrict__ packed,
                   uint8_t* __restrict__ scales, int64_t n_items) {
  const int64_t n_blocks = n_items / 4;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t blk = (int64_t)blockIdx.x * kThreads + threadIdx.x; blk < n_blocks; blk += stride)
    mx_quantize_block<DT, true>(x, (uint4*)packed, scales, n_blocks, blk);
}

// -------------------------------------------------------- mx_dequantize

// One iteration of the unpack over the warp's kUnroll items.  kFull: all
// of them exist (no bounds tests).
template <int DT, bool kFull>
__device__ __forceinline__ void mx_dequantize_items(const uint32_t* __restrict__ packed,
                                                    const uint8_t* __restrict__ scales,
                                                    void* __restrict__ out, int64_t n_items,
                                                    int64_t base, int64_t stride, int lane) {
  auto in_range = [&](int64_t item) { return kFull || item < n_items; };
  uint32_t p[kUnroll], s[kUnroll];
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    int64_t item = base + u * stride + lane;
    if (in_range(item)) {
      p[u] = MXQ_IN_RANGE(kChkMxDeqIn, item, n_items) ? ld_stream_u32(packed + item) : 0u;
      s[u] = MXQ_IN_RANGE(kChkMxDeqScale, item >> 2, n_items / 4)
                 ? ld_stream_u8(scales + (item >> 2))
                 : 0u;
    }
  }
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    int64_t item = base + u * stride + lane;
    if (!in_range(item) || !MXQ_IN_RANGE(kChkMxDeqOut, item, n_items)) continue;
    if (s[u] == 0xFFu) {  // E8M0 NaN
      store8_bits<DT>(out, item, ElemTraits<DT>::kNaN);
      continue;
    }
    float scale = exp2i((int)s[u] - 127);  // 2^-127 .. 2^127, exact
    float v[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t h2 = e2m1x2_to_f16x2((p[u] >> (8 * j)) & 0xFFu);
      // value * scale is exact; adding +0 turns the -0 of nibble 8 into +0
      fma2_rn_zero(v[2 * j], v[2 * j + 1], f16lo(h2), f16hi(h2), scale, scale);
    }
    store8<DT>(out, item, v);
  }
}

template <int DT>
__global__ void __launch_bounds__(kThreads)
mx_dequantize_kernel(const uint32_t* __restrict__ packed, const uint8_t* __restrict__ scales,
                     void* __restrict__ out, int64_t n_items) {
  const int lane = threadIdx.x & 31;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t base = (int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31); base < n_items;
       base += stride * kUnroll) {
    if (base + (kUnroll - 1) * stride + 32 <= n_items)
      mx_dequantize_items<DT, true>(packed, scales, out, n_items, base, stride, lane);
    else
      mx_dequantize_items<DT, false>(packed, scales, out, n_items, base, stride, lane);
  }
}

// ------------------------------------------------------- quantize_cache

template <int FMT>
struct CacheFormat;
template <>
struct CacheFormat<MXQ_FMT_FP8> {
  static constexpr int kLo = -126, kHi = 127;
  // qmax = 448 = 1.75 * 2^8
  static constexpr int kQExp = 8;
  static constexpr uint32_t kQFrac = 0x600000u;
};
template <>
struct CacheFormat<MXQ_FMT_MXFP4> {
  static constexpr int kLo = -126, kHi = 127;
  // qmax = 6 = 1.5 * 2^2
  static constexpr int kQExp = 2;
  static constexpr uint32_t kQFrac = 0x400000u;
};
template <>
struct CacheFormat<MXQ_FMT_NVFP4> {
  static constexpr int kLo = -9, kHi = 8;
  static constexpr int kQExp = 2;
  static constexpr uint32_t kQFrac = 0x400000u;
};

// Exponent k of the least power of two with 2^k * qmax >= amax, clamped:
// with amax = 2^E * (1 + f) and qmax = 2^Q * (1 + g), k = E - Q when
// f <= g and E - Q + 1 otherwise.
template <int FMT>
__device__ __forceinline__ int cache_scale_exp(uint32_t amax_f32bits) {
  using F = CacheFormat<FMT>;
  if (amax_f32bits == 0) return F::kLo;
  int k = floor_log2_f32bits(amax_f32bits) - F::kQExp +
          (frac23_f32bits(amax_f32bits) > F::kQFrac ? 1 : 0);
  return k < F::kLo ? F::kLo : (k > F::kHi ? F::kHi : k);
}

// Fake-quantize 8 values already divided by the scale; multiply back by s.
template <int FMT>
__device__ __forceinline__ void fake_quant8(float* v, float s) {
  if constexpr (FMT == MXQ_FMT_FP8) {
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      uint32_t h2 = e4m3x2_to_f16x2(e4m3x2(v[j], v[j + 1]));
      mul2_rn(v[j], v[j + 1], f16lo(h2), f16hi(h2), s, s);  // exact; the sign of zero is kept
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      uint32_t h2 = e2m1x2_to_f16x2(e2m1x2(v[j], v[j + 1]));
      // exact; zero magnitudes become +0
      fma2_rn_zero(v[j], v[j + 1], f16lo(h2), f16hi(h2), s, s);
    }
  }
}

template <int DT, int FMT, int LPB>
__global__ void __launch_bounds__(kThreads)
quantize_cache_kernel(const void* __restrict__ in, void* __restrict__ out, int64_t n_items) {
  const int lane = threadIdx.x & 31;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t base = (int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31); base < n_items;
       base += stride * kUnroll) {
    Raw8<DT> raw[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t item = base + u * stride + lane;
      if (item < n_items && MXQ_IN_RANGE(kChkCacheIn, item, n_items))
        raw[u] = load_raw8<DT>(in, item);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t item = base + u * stride + lane;
      const bool valid = item < n_items;
      uint32_t m = valid ? raw_amax<DT>(raw[u]) : 0u;
#pragma unroll
      for (int o = 1; o < LPB; o <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (!valid) continue;
      const int k = cache_scale_exp<FMT>(m);
      const float inv = exp2i(-k), s = exp2i(k);
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; j += 2)  // exact
        mul2_rn(v[j], v[j + 1], elem_to_f32<DT>(raw_elem<DT>(raw[u], j)),
                elem_to_f32<DT>(raw_elem<DT>(raw[u], j + 1)), inv, inv);
      fake_quant8<FMT>(v, s);
      if (MXQ_IN_RANGE(kChkCacheOut, item, n_items)) store8<DT>(out, item, v);
    }
  }
}

// General kernel: any block size, any channel count, any alignment.  One
// thread per (row, group); the last group of a row may be partial.
template <int DT>
__device__ __forceinline__ uint32_t load_elem_bits(const void* p, int64_t i) {
  if constexpr (ElemTraits<DT>::kBytes == 2) return ((const uint16_t*)p)[i];
  else return ((const uint32_t*)p)[i];
}
template <int DT>
__device__ __forceinline__ void store_elem(void* p, int64_t i, float v) {
  if constexpr (DT == kBF16) {
    ((uint16_t*)p)[i] = pack2<DT>(v, 0.0f) & 0xFFFFu;
  } else if constexpr (DT == kF16) {
    ((uint16_t*)p)[i] = pack2<DT>(v, 0.0f) & 0xFFFFu;
  } else {
    ((float*)p)[i] = v;
  }
}

template <int DT, int FMT>
__global__ void __launch_bounds__(kThreads)
quantize_cache_general_kernel(const void* __restrict__ in, void* __restrict__ out, int64_t rows,
                              int64_t C, int B) {
  const int64_t groups_per_row = (C + B - 1) / B;
  const int64_t n_groups = rows * groups_per_row;
  for (int64_t g = (int64_t)blockIdx.x * kThreads + threadIdx.x; g < n_groups;
       g += (int64_t)gridDim.x * kThreads) {
    int64_t r = g / groups_per_row;
    int64_t c0 = (g % groups_per_row) * B;
    int64_t c1 = c0 + B < C ? c0 + B : C;
    uint32_t m = 0;
    for (int64_t c = c0; c < c1; ++c)
      if (MXQ_IN_RANGE(kChkCacheGenIn, r * C + c, rows * C))
        m = max(m, mag_as_f32_bits<DT>(load_elem_bits<DT>(in, r * C + c)));
    int k = cache_scale_exp<FMT>(m);
    float inv = exp2i(-k), s = exp2i(k);
    for (int64_t c = c0; c < c1; c += 8) {
      float v[8];
      int n = (int)(c1 - c < 8 ? c1 - c : 8);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        v[j] = j < n && MXQ_IN_RANGE(kChkCacheGenIn, r * C + c + j, rows * C)
                   ? elem_to_f32<DT>(load_elem_bits<DT>(in, r * C + c + j)) * inv
                   : 0.0f;
      fake_quant8<FMT>(v, s);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < n && MXQ_IN_RANGE(kChkCacheGenOut, r * C + c + j, rows * C))
          store_elem<DT>(out, r * C + c + j, v[j]);
    }
  }
}

// ------------------------------------------------------------ launchers

template <class Kernel>
static int grid_for(Kernel kernel, int64_t n_units, int per_block) {
  return wave_grid((const void*)kernel, kThreads, n_units, per_block);
}

int launch_mx_quantize(const void* x, int dt, int64_t rows, int64_t K, void* packed, void* scales,
                       cudaStream_t st) {
  const int64_t n_items = rows * (K / 8);
  const int per = kThreads * 4;  // items: one 32-block per thread and iteration
  auto* p = (uint32_t*)packed;
  auto* s = (uint8_t*)scales;
  switch (dt) {
    case kBF16:
      mx_quantize_kernel<kBF16><<<grid_for(mx_quantize_kernel<kBF16>, n_items, per), kThreads, 0,
                                  st>>>(x, p, s, n_items);
      break;
    case kF16:
      mx_quantize_kernel<kF16><<<grid_for(mx_quantize_kernel<kF16>, n_items, per), kThreads, 0,
                                 st>>>(x, p, s, n_items);
      break;
    default:
      mx_quantize_kernel<kF32><<<grid_for(mx_quantize_kernel<kF32>, n_items, per), kThreads, 0,
                                 st>>>(x, p, s, n_items);
      break;
  }
  return cudaGetLastError() == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

int launch_mx_dequantize(const void* packed, const void* scales, int64_t rows, int64_t K, void* out,
                         int dt, cudaStream_t st) {
  const int64_t n_items = rows * (K / 8);
  const int per = kThreads * kUnroll;
  auto* p = (const uint32_t*)packed;
  auto* s = (const uint8_t*)scales;
  switch (dt) {
    case kBF16:
      mx_dequantize_kernel<kBF16><<<grid_for(mx_dequantize_kernel<kBF16>, n_items, per), kThreads,
                                    0, st>>>(p, s, out, n_items);
      break;
    case kF16:
      mx_dequantize_kernel<kF16><<<grid_for(mx_dequantize_kernel<kF16>, n_items, per), kThreads,
                                   0, st>>>(p, s, out, n_items);
      break;
    default:
      mx_dequantize_kernel<kF32><<<grid_for(mx_dequantize_kernel<kF32>, n_items, per), kThreads,
                                   0, st>>>(p, s, out, n_items);
      break;
  }
  return cudaGetLastError() == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

template <int DT, int FMT, int LPB>
static void launch_cache_lpb(const void* in, void* out, int64_t n_items, cudaStream_t st) {
  const int grid = grid_for(quantize_cache_kernel<DT, FMT, LPB>, n_items, kThreads * kUnroll);
  quantize_cache_kernel<DT, FMT, LPB><<<grid, kThreads, 0, st>>>(in, out, n_items);
}

template <int DT, int FMT>
static void launch_cache_fast(const void* in, void* out, int64_t n_items, int lpb, cudaStream_t st) {
  switch (lpb) {
    case 1: launch_cache_lpb<DT, FMT, 1>(in, out, n_items, st); break;
    case 2: launch_cache_lpb<DT, FMT, 2>(in, out, n_items, st); break;
    case 4: launch_cache_lpb<DT, FMT, 4>(in, out, n_items, st); break;
    case 8: launch_cache_lpb<DT, FMT, 8>(in, out, n_items, st); break;
    case 16: launch_cache_lpb<DT, FMT, 16>(in, out, n_items, st); break;
    default: launch_cache_lpb<DT, FMT, 32>(in, out, n_items, st); break;
  }
}

template <int DT, int FMT>
static void launch_cache(const void* in, void* out, int64_t rows, int64_t C, int B, bool fast,
                         cudaStream_t st) {
  if (fast) {
    launch_cache_fast<DT, FMT>(in, out, rows * (C / 8), B / 8, st);
  } else {
    int64_t n_groups = rows * ((C + B - 1) / B);
    const int grid = grid_for(quantize_cache_general_kernel<DT, FMT>, n_groups, kThreads);
    quantize_cache_general_kernel<DT, FMT><<<grid, kThreads, 0, st>>>(in, out, rows, C, B);
  }
}

template <int DT>
static void launch_cache_dt(const void* in, void* out, int64_t rows, int64_t C, int fmt, int B,
                            bool fast, cudaStream_t st) {
  switch (fmt) {
    case MXQ_FMT_FP8: launch_cache<DT, MXQ_FMT_FP8>(in, out, rows, C, B, fast, st); break;
    case MXQ_FMT_MXFP4: launch_cache<DT, MXQ_FMT_MXFP4>(in, out, rows, C, B, fast, st); break;
    default: launch_cache<DT, MXQ_FMT_NVFP4>(in, out, rows, C, B, fast, st); break;
  }
}

int launch_quantize_cache(const void* in, void* out, int dt, int64_t rows, int64_t C, int fmt,
                          int B, bool fast, cudaStream_t st) {
  switch (dt) {
    case kBF16: launch_cache_dt<kBF16>(in, out, rows, C, fmt, B, fast, st); break;
    case kF16: launch_cache_dt<kF16>(in, out, rows, C, fmt, B, fast, st); break;
    default: launch_cache_dt<kF32>(in, out, rows, C, fmt, B, fast, st); break;
  }
  return cudaGetLastError() == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

MXQ_DEFINE_CHECK_READER(check_record_elementwise)

}  // namespace mxq
