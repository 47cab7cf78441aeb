// NVFP4 two-level quantization ("NVIDIA Model Optimizer: from mtq.quantize to
// a 4.95-bit DeepSeek-R1", section "NVFP4 in the code: two scales and a
// nibble"): a per-tensor binary32 scale g = max|W| / (6 * 448), one E4M3
// scale per 16 values s_b = E4M3(amax_b / (6 g)) (zero -> 1.0, clamped to
// [2^-9, 448]) and E2M1 codes of W / (s_b g), packed two per byte.
//
// Three launches on the caller's stream: clear the amax word of the
// workspace, a grid-wide amax (warp and CTA reductions, one atomicMax per
// CTA on the magnitude bits, which order like the values), then the
// streaming quantize pass (one 16-block per lane: its maximum, scale and
// codes need no exchange between lanes).  Every binary32 operation the recipe names
// (the divisions and products) is the IEEE-rounded one (div.rn / mul.rn), or
// gives provably the same E2M1 code (the guarded reciprocal quotient of
// e2m1x8_quot), so the codes match a plain float32 implementation bit for
// bit.
#include <mutex>

#include "mxq_device.cuh"
#include "mxq_launch.h"
#include "sm100_primitives.cuh"

namespace mxq {

namespace {

constexpr int kNvThreads = 256;
constexpr int kNvUnroll = 4;   // amax and unpack passes
// The quantize pass: one 16-block per lane and iteration (40 registers).
constexpr int kNvQUnroll = 1;

template <int DT>
__device__ __forceinline__ uint32_t elem_bits(const uint4& a, const uint4& b, int j) {
  if constexpr (ElemTraits<DT>::kBytes == 2) {
    const uint32_t w = j < 2 ? a.x : j < 4 ? a.y : j < 6 ? a.z : a.w;
    return (j & 1) ? (w >> 16) : (w & 0xFFFFu);
  } else {
    const uint4& q = j < 4 ? a : b;
    const int k = j & 3;
    return k == 0 ? q.x : k == 1 ? q.y : k == 2 ? q.z : q.w;
  }
}

// f32 bit pattern of max |x| over the eight elements.  For 16-bit formats
// the magnitudes are compared pairwise as unsigned halves (monotone in |x|
// for finite values).
template <int DT>
__device__ __forceinline__ uint32_t amax8(const uint4& a, const uint4& b) {
  if constexpr (ElemTraits<DT>::kBytes == 2) {
    const uint32_t M = 0x7FFF7FFFu;
    const uint32_t m2 = __vmaxu2(__vmaxu2(a.x & M, a.y & M), __vmaxu2(a.z & M, a.w & M));
    return mag_as_f32_bits<DT>(max(m2 & 0xFFFFu, m2 >> 16));
  } else {
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) m = max(m, mag_as_f32_bits<DT>(elem_bits<DT>(a, b, j)));
    return m;
  }
}

template <int DT>
__device__ __forceinline__ void load_vec8(const void* x, int64_t item, uint4& a, uint4& b) {
  if constexpr (ElemTraits<DT>::kBytes == 2) {
    a = ld_stream_v4((const char*)x + item * 16);
  } else {
    a = ld_stream_v4((const char*)x + item * 32);
    b = ld_stream_v4((const char*)x + item * 32 + 16);
  }
}

__global__ void clear_word_kernel(uint32_t* w) { *w = 0u; }

// The amax and quantize passes are launched with programmatic stream
// serialization: a pass's CTAs may be scheduled while the kernel before it
// finishes (each pass allows it for its successor at once), and wait for
// that kernel's results (sm100::griddep_wait) before touching what it wrote.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// max |x| over the tensor as binary32 bits, accumulated with atomicMax.
template <int DT>
__global__ void __launch_bounds__(kNvThreads)
nvfp4_amax_kernel(const void* __restrict__ x, int64_t n_items, uint32_t* __restrict__ amax_word) {
  griddep_launch_dependents();
  __shared__ uint32_t s_max[kNvThreads / 32];
  uint32_t m = 0;
  const int64_t stride = (int64_t)gridDim.x * kNvThreads;
  // kNvUnroll independent 16-byte loads in flight per thread
  for (int64_t base = (int64_t)blockIdx.x * kNvThreads + threadIdx.x; base < n_items;
       base += stride * kNvUnroll) {
    uint4 a[kNvUnroll], b[kNvUnroll];
#pragma unroll
    for (int u = 0; u < kNvUnroll; ++u)
      if (base + u * stride < n_items && MXQ_IN_RANGE(kChkNvAmaxIn, base + u * stride, n_items))
        load_vec8<DT>(x, base + u * stride, a[u], b[u]);
      else
        a[u] = b[u] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < kNvUnroll; ++u)
      if (base + u * stride < n_items) m = max(m, amax8<DT>(a[u], b[u]));
  }
  m = __reduce_max_sync(0xffffffffu, m);
  if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < kNvThreads / 32 ? s_max[threadIdx.x] : 0u;
    m = __reduce_max_sync(0xffffffffu, m);
    sm100::griddep_wait();  // the cleared word (x itself was complete before the clear)
    if (threadIdx.x == 0 && m != 0u) atomicMax(amax_word, m);
  }
}

// E2M1 codes of the eight binary32 quotients w_j / d, with -0.0 giving the
// code of +0.0 (no sign bit) and a nonzero weight whose quotient underflows
// keeping its sign.  r = fl32(1 / d) for d in the bracket's range, else 0:
// then the IEEE divisions decide.  Bracket (see e2m1x8_quot): the products
// are fma(w, r(1 -+ 2^-19), +0), which round exactly like w r(1 -+ 2^-19)
// except that a zero product is +0.
__device__ __forceinline__ uint32_t e2m1x8_quot_unsigned_zero(const float* w, float d, float r) {
  if (r != 0.0f) {
    const float r_lo = r * (1.0f - 0x1p-19f), r_hi = r * (1.0f + 0x1p-19f);
    float lo[8], hi[8];
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      fma2_rn_zero(lo[j], lo[j + 1], w[j], w[j + 1], r_lo, r_lo);
      fma2_rn_zero(hi[j], hi[j + 1], w[j], w[j + 1], r_hi, r_hi);
    }
    const uint32_t a = e2m1x8(lo);
    if (a == e2m1x8(hi)) return a;
  }
  return e2m1x8_div(w[0] + 0.0f, w[1] + 0.0f, w[2] + 0.0f, w[3] + 0.0f, w[4] + 0.0f, w[5] + 0.0f,
                    w[6] + 0.0f, w[7] + 0.0f, d);
}

// 16 elements of block blk as two items (16-byte loads kept in L1: the
// lane's second load reads the other half of the sectors its first one
// brought in).
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
template <int DT>
__device__ __forceinline__ void load_block16v(const void* x, int64_t blk, uint4& a0, uint4& b0,
                                              uint4& a1, uint4& b1) {
  if constexpr (ElemTraits<DT>::kBytes == 2) {
    a0 = ld_nc_v4((const char*)x + blk * 32);
    a1 = ld_nc_v4((const char*)x + blk * 32 + 16);
  } else {
    a0 = ld_nc_v4((const char*)x + blk * 64);
    b0 = ld_nc_v4((const char*)x + blk * 64 + 16);
    a1 = ld_nc_v4((const char*)x + blk * 64 + 32);
    b1 = ld_nc_v4((const char*)x + blk * 64 + 48);
  }
}

// One iteration of the quantize pass: each lane one 16-block (two items) of
// kNvQUnroll slots base + u stride + lane.  kFull: all of them exist.
template <int DT, bool kFull>
__device__ __forceinline__ void nvfp4_quantize_blocks(const void* __restrict__ x,
                                                      uint2* __restrict__ packed,
                                                      uint8_t* __restrict__ block_scales,
                                                      int64_t n_blocks, int64_t base,
                                                      int64_t stride, int lane, float t, bool zero,
                                                      const float* s_d, const float* s_r) {
  auto in_range = [&](int64_t blk) { return kFull || blk < n_blocks; };
  uint4 a0[kNvQUnroll], b0[kNvQUnroll], a1[kNvQUnroll], b1[kNvQUnroll];
#pragma unroll
  for (int u = 0; u < kNvQUnroll; ++u) {
    const int64_t blk = base + u * stride + lane;
    if (in_range(blk) && MXQ_IN_RANGE(kChkNvQuantIn, 2 * blk + 1, 2 * n_blocks))
      load_block16v<DT>(x, blk, a0[u], b0[u], a1[u], b1[u]);
  }
  if (zero) {
#pragma unroll
    for (int u = 0; u < kNvQUnroll; ++u) {
      const int64_t blk = base + u * stride + lane;
      if (!in_range(blk)) continue;
      if (MXQ_IN_RANGE(kChkNvQuantOut, 2 * blk + 1, 2 * n_blocks)) packed[blk] = make_uint2(0u, 0u);
      if (MXQ_IN_RANGE(kChkNvQuantScale, blk, n_blocks)) block_scales[blk] = 0x38u;  // E4M3 1.0
    }
    return;
  }
#pragma unroll
  for (int u = 0; u < kNvQUnroll; ++u) {
    const int64_t blk = base + u * stride + lane;
    if (!in_range(blk)) continue;
    const uint32_t m = max(amax8<DT>(a0[u], b0[u]), amax8<DT>(a1[u], b1[u]));
    float q = __fdiv_rn(__uint_as_float(m), t);
    if (q == 0.0f) q = 1.0f;
    q = fminf(fmaxf(q, 0.001953125f), 448.0f);  // [2^-9, 448]
    const uint32_t sc = e4m3x2(q, 0.0f) & 0xFFu;  // 0x01 .. 0x7E
    const float d = s_d[sc & 0x7Fu], r = s_r[sc & 0x7Fu];
    float w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = elem_to_f32<DT>(elem_bits<DT>(a0[u], b0[u], j));
    const uint32_t c0 = e2m1x8_quot_unsigned_zero(w, d, r);
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = elem_to_f32<DT>(elem_bits<DT>(a1[u], b1[u], j));
    const uint32_t c1 = e2m1x8_quot_unsigned_zero(w, d, r);
    if (MXQ_IN_RANGE(kChkNvQuantOut, 2 * blk + 1, 2 * n_blocks)) packed[blk] = make_uint2(c0, c1);
    if (MXQ_IN_RANGE(kChkNvQuantScale, blk, n_blocks)) block_scales[blk] = (uint8_t)sc;
  }
}

// At least four CTAs per SM for 16-bit inputs (at most 64 registers; the
// one-block-per-lane pass needs 40, and the occupancy query sizes the grid).
template <int DT>
__global__ void __launch_bounds__(kNvThreads, ElemTraits<DT>::kBytes == 2 ? 4 : 1)
nvfp4_quantize_kernel(const void* __restrict__ x, uint32_t* __restrict__ packed,
                      uint8_t* __restrict__ block_scales, float* __restrict__ global_scale,
                      const uint32_t* __restrict__ amax_word, int64_t n_items) {
  griddep_launch_dependents();
  sm100::griddep_wait();  // the amax pass has completed
  const float amax = __uint_as_float(*amax_word);
  const bool zero = amax == 0.0f;
  const float g = zero ? 0.0f : __fdiv_rn(amax, 2688.0f);  // 6 * 448
  const float t = __fmul_rn(6.0f, g);
  if (blockIdx.x == 0 && threadIdx.x == 0) *global_scale = g;
  // Per E4M3 scale code c: the divisor d = fl(s_c g) and, where the bracket
  // applies (quot_fast_ok), r = fl(1 / d), else 0.  Looked up per block.
  __shared__ float s_d[128], s_r[128];
  if (threadIdx.x < 128) {
    const float d = __fmul_rn(f16lo(e4m3x2_to_f16x2(threadIdx.x)), g);
    s_d[threadIdx.x] = d;
    s_r[threadIdx.x] = quot_fast_ok(d) ? __frcp_rn(d) : 0.0f;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t n_blocks = n_items / 2;
  const int64_t stride = (int64_t)gridDim.x * kNvThreads;
  for (int64_t base = (int64_t)blockIdx.x * kNvThreads + (threadIdx.x & ~31); base < n_blocks;
       base += stride * kNvQUnroll) {
    if (base + (kNvQUnroll - 1) * stride + 32 <= n_blocks)
      nvfp4_quantize_blocks<DT, true>(x, (uint2*)packed, block_scales, n_blocks, base, stride,
                                      lane, t, zero, s_d, s_r);
    else
      nvfp4_quantize_blocks<DT, false>(x, (uint2*)packed, block_scales, n_blocks, base, stride,
                                       lane, t, zero, s_d, s_r);
  }
}

template <int DT>
__global__ void __launch_bounds__(kNvThreads)
nvfp4_dequantize_kernel(const uint32_t* __restrict__ packed, const uint8_t* __restrict__ block_scales,
                        const float* __restrict__ global_scale, void* __restrict__ out,
                        int64_t n_items) {
  const float g = *global_scale;
  const int lane = threadIdx.x & 31;
  const int64_t stride = (int64_t)gridDim.x * kNvThreads;
  for (int64_t base = (int64_t)blockIdx.x * kNvThreads + (threadIdx.x & ~31); base < n_items;
       base += stride * kNvUnroll) {
    uint32_t p[kNvUnroll], sb[kNvUnroll];
#pragma unroll
    for (int u = 0; u < kNvUnroll; ++u) {
      const int64_t item = base + u * stride + lane;
      if (item < n_items) {
        p[u] = MXQ_IN_RANGE(kChkNvDeqIn, item, n_items) ? ld_stream_u32(packed + item) : 0u;
        sb[u] = MXQ_IN_RANGE(kChkNvDeqScale, item >> 1, n_items / 2)
                    ? ld_stream_u8(block_scales + (item >> 1))
                    : 0u;
      }
    }
#pragma unroll
    for (int u = 0; u < kNvUnroll; ++u) {
      const int64_t item = base + u * stride + lane;
      if (item >= n_items) continue;
      const float s = f16lo(e4m3x2_to_f16x2(sb[u]));
      float v[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t h2 = e2m1x2_to_f16x2((p[u] >> (8 * j)) & 0xFFu);
        // code * s_b is exact in binary32; times g rounds once; adding +0
        // in the same fma turns the -0 of nibble 8 into +0
        float c0, c1;
        mul2_rn(c0, c1, f16lo(h2), f16hi(h2), s, s);
        fma2_rn_zero(v[2 * j], v[2 * j + 1], c0, c1, g, g);
      }
      if (MXQ_IN_RANGE(kChkNvDeqOut, item, n_items)) store8<DT>(out, item, v);
    }
  }
}

template <class Kernel>
int grid_for(Kernel kernel, int64_t n_units, int per_block) {
  return wave_grid((const void*)kernel, kNvThreads, n_units, per_block);
}

// Launch with programmatic stream serialization (see griddep_launch_dependents).
template <class... Params, class... Args>
void launch_dependent(void (*kernel)(Params...), int grid, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kNvThreads, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int DT>
void run_amax(const void* x, int64_t n_items, uint32_t* amax_word, cudaStream_t st) {
  clear_word_kernel<<<1, 1, 0, st>>>(amax_word);
  if (n_items > 0) {
    const int grid = grid_for(nvfp4_amax_kernel<DT>, n_items, kNvThreads * kNvUnroll);
    launch_dependent(nvfp4_amax_kernel<DT>, grid, st, x, n_items, amax_word);
  }
}

template <int DT>
int run_quantize(const void* x, int64_t rows, int64_t K, void* packed, void* block_scales,
                 float* global_scale, uint32_t* amax_word, cudaStream_t st) {
  const int64_t n_items = rows * (K / 8);
  run_amax<DT>(x, n_items, amax_word, st);
  const int grid = grid_for(nvfp4_quantize_kernel<DT>, n_items / 2, kNvThreads * kNvQUnroll);
  launch_dependent(nvfp4_quantize_kernel<DT>, grid, st, x, (uint32_t*)packed,
                   (uint8_t*)block_scales, global_scale, (const uint32_t*)amax_word, n_items);
  return cudaGetLastError() == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

// Scratch of the allocation-free entry point: one copy per GPU that loads
// the library, alive until the process exits.  Host code must not pass the
// symbol itself to a kernel (on the host it names a stand-in, not device
// memory); it passes the address cudaGetSymbolAddress returns.
static __device__ __align__(256) uint32_t g_noalloc_scratch[MXQ_NOALLOC_SCRATCH_BYTES / 4];

}  // namespace

uint32_t* noalloc_scratch(size_t need_bytes, int* status) {
  if (need_bytes > sizeof(g_noalloc_scratch)) {
    *status = MXQ_ERR_UNSUPPORTED;
    return nullptr;
  }
  static std::mutex mu;
  static uint32_t* by_device[64] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *status = MXQ_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (by_device[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      *status = MXQ_ERR_CUDA;
      return nullptr;
    }
    by_device[dev] = (uint32_t*)p;
  }
  *status = MXQ_OK;
  return by_device[dev];
}

int launch_nvfp4_quantize(const void* x, int dt, int64_t rows, int64_t K, void* packed,
                          void* block_scales, float* global_scale, uint32_t* amax_word,
                          cudaStream_t st) {
  switch (dt) {
    case kBF16: return run_quantize<kBF16>(x, rows, K, packed, block_scales, global_scale, amax_word, st);
    case kF16: return run_quantize<kF16>(x, rows, K, packed, block_scales, global_scale, amax_word, st);
    default: return run_quantize<kF32>(x, rows, K, packed, block_scales, global_scale, amax_word, st);
  }
}

void launch_nvfp4_amax(const void* x, int dt, int64_t n_elems, uint32_t* amax_word,
                       cudaStream_t st) {
  switch (dt) {
    case kBF16: run_amax<kBF16>(x, n_elems / 8, amax_word, st); break;
    case kF16: run_amax<kF16>(x, n_elems / 8, amax_word, st); break;
    default: run_amax<kF32>(x, n_elems / 8, amax_word, st); break;
  }
}

int launch_nvfp4_dequantize(const void* packed, const void* block_scales, const float* global_scale,
                            int64_t rows, int64_t K, void* out, int dt, cudaStream_t st) {
  const int64_t n_items = rows * (K / 8);
  const int per = kNvThreads * kNvUnroll;
  auto* p = (const uint32_t*)packed;
  auto* s = (const uint8_t*)block_scales;
  switch (dt) {
    case kBF16:
      nvfp4_dequantize_kernel<kBF16><<<grid_for(nvfp4_dequantize_kernel<kBF16>, n_items, per),
                                       kNvThreads, 0, st>>>(p, s, global_scale, out, n_items);
      break;
    case kF16:
      nvfp4_dequantize_kernel<kF16><<<grid_for(nvfp4_dequantize_kernel<kF16>, n_items, per),
                                      kNvThreads, 0, st>>>(p, s, global_scale, out, n_items);
      break;
    default:
      nvfp4_dequantize_kernel<kF32><<<grid_for(nvfp4_dequantize_kernel<kF32>, n_items, per),
                                      kNvThreads, 0, st>>>(p, s, global_scale, out, n_items);
      break;
  }
  return cudaGetLastError() == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

MXQ_DEFINE_CHECK_READER(check_record_nvfp4)

}  // namespace mxq
