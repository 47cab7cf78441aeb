// NVFP4 with block scales chosen by least squared weight error ("NVIDIA
// Model Optimizer: from mtq.quantize to a 4.95-bit DeepSeek-R1", section
// "NVFP4's own rules", the mse rule): the per-tensor scale g is the max
// rule's (max |W| / 2688), and each 16-block tries all 126 positive finite
// E4M3 codes c as its scale, keeping the one whose reconstruction
// E2M1(w / d_c) * d_c, d_c = s_c * g, has the least sum of squared errors.
//
// Arithmetic, identical for every candidate and on every device: d_c is the
// binary32 product, the quotient w / d_c is the binary32 division (div.rn)
// and is cast to E2M1 as in the max rule; the error q * d_c - w is formed by
// one double fma, which is exact (q has 2 significant bits, d_c 24, and the
// two terms lie within 2^21 of each other), and the squares are summed over
// the block in element order by double fmas.  Among equal sums the smallest
// code wins.  A code whose d_c underflows to zero is skipped.  With g = 0
// (an all-zero tensor) the output is the max rule's: scale 1.0, zero codes.
//
// Work split: kLanes lanes share a block, each trying every kLanes-th code
// (only the codes that can win: see the pruning below), and combine (error,
// code) with shuffles; the lane of the first slot then writes the block's
// eight code bytes and its scale byte.  kLanes = 1: one thread searches a
// block's codes alone, from the top down, so its own best sum prunes every
// remaining code of the block, and no lane idles while another lane of its
// block is still searching (with 2 or 4 lanes per block the sweep took 13 %
// or 32 % longer on B200).
// This is ALU work (126 candidates x 16 divisions and fmas per block), so
// the grid is one thread per (block, lane slot) and the CTA scheduler
// balances the waves.
#include "mxq.h"
#include "mxq_device.cuh"
#include "mxq_launch.h"

namespace mxq {

namespace {

constexpr int kMseThreads = 256;
constexpr int kLanes = 1;  // lanes per 16-block

__device__ __forceinline__ double f16_to_f64(uint32_t h) {
  double r;
  asm("cvt.f64.f16 %0, %1;" : "=d"(r) : "h"((uint16_t)h));
  return r;
}

// 16 elements of a block as f32 (exact for every input dtype).
template <int DT>
__device__ __forceinline__ void load_block16(const void* x, int64_t blk, float* w) {
  uint32_t bits[16];
  load8<DT>(x, 2 * blk, bits);
  load8<DT>(x, 2 * blk + 1, bits + 8);
#pragma unroll
  for (int i = 0; i < 16; ++i) w[i] = elem_to_f32<DT>(bits[i]);
}

// Four CTAs per SM (64 registers, a few values spilled): the sweep is
// issue-bound with the blocks of a warp needing different numbers of codes,
// and the extra warps fill more issue slots.
template <int DT>
__global__ void __launch_bounds__(kMseThreads, 4)
nvfp4_mse_kernel(const void* __restrict__ x, uint2* __restrict__ packed,
                 uint8_t* __restrict__ block_scales, float* __restrict__ global_scale,
                 const uint32_t* __restrict__ amax_word, int64_t n_blocks) {
  __shared__ float s_d[128];  // d_c = s_c * g for every E4M3 code c < 128
  const float amax = __uint_as_float(*amax_word);
  const bool zero = amax == 0.0f;
  const float g = zero ? 0.0f : __fdiv_rn(amax, 2688.0f);  // 6 * 448
  if (blockIdx.x == 0 && threadIdx.x == 0) *global_scale = g;
  if (threadIdx.x < 128) {
    const float s = f16lo(e4m3x2_to_f16x2(threadIdx.x));
    s_d[threadIdx.x] = __fmul_rn(s, g);
  }
  __syncthreads();

  const int64_t t = (int64_t)blockIdx.x * kMseThreads + threadIdx.x;
  const int64_t blk = t / kLanes;
  const int slot = (int)(t % kLanes);
  // Lanes past the end take part in the shuffles with an empty search.
  const bool valid = blk < n_blocks;

  float w[16];
  if (valid && MXQ_IN_RANGE(kChkMseIn, blk, n_blocks)) load_block16<DT>(x, blk, w);
  else
    for (int i = 0; i < 16; ++i) w[i] = 0.0f;

  int best_c = 0x38;
  if (!zero) {
    double best = __longlong_as_double(0x7FF0000000000000LL);  // +inf
    best_c = 1;
    if (valid) {
      double wd[16];
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        wd[i] = (double)w[i];
        amax = fmaxf(amax, fabsf(w[i]));
      }
      // Codes are visited from the top down, and only where they can win:
      //  * from c_top = the smallest code whose quotient amax / d rounds to
      //    at most 0.25 (every weight's code is then 0, so every larger code
      //    reconstructs all zeros with exactly the same error and loses the
      //    tie to c_top); 126 if there is none;
      //  * down to the first code whose clipping error alone exceeds the
      //    best sum so far: with 6d < amax the largest weight is cut to 6d,
      //    so the sum is at least (amax - 6d)^2 (exact in double; the
      //    accumulated sum is within 2^-49 of the exact one), and it only
      //    grows as d shrinks.
      // Visiting in decreasing order with <= keeps the smallest code among
      // equal sums, as the full ascending sweep does.
      auto all_zero = [&](int c) {
        const float dc = s_d[c];
        return dc != 0.0f && __fdiv_rn(amax, dc) <= 0.25f;
      };
      int c_top = 126;
      if (all_zero(126)) {
        int lo = 1, hi = 126;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (all_zero(mid)) hi = mid;
          else lo = mid + 1;
        }
        c_top = lo;
      }
      const double amax_d = (double)amax;
      for (int c = c_top - slot; c >= 1; c -= kLanes) {
        const float d = s_d[c];
        if (d == 0.0f) break;  // d only shrinks further down
        const double dd = (double)d;
        const double t = amax_d - 6.0 * dd;
        if (t > 0.0 && t * t * (1.0 - 0x1p-40) > best) break;
        // the 16 E2M1 codes of fl32(w / d), eight per word
        uint32_t q[2];
        if (quot_fast_ok(d)) {
          float r_lo, r_hi;
          bracket_factors(d, r_lo, r_hi);
          q[0] = e2m1x8_quot(w, d, r_lo, r_hi);
          q[1] = e2m1x8_quot(w + 8, d, r_lo, r_hi);
        } else {
          q[0] = e2m1x8_div(w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7], d);
          q[1] = e2m1x8_div(w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15], d);
        }
        double err = 0.0;
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          const uint32_t h2 = e2m1x2_to_f16x2((q[i >> 3] >> (4 * (i & 7))) & 0xFFu);
          const double e0 = fma(f16_to_f64(h2 & 0xFFFFu), dd, -wd[i]);
          err = fma(e0, e0, err);
          const double e1 = fma(f16_to_f64(h2 >> 16), dd, -wd[i + 1]);
          err = fma(e1, e1, err);
        }
        if (err <= best) {  // descending: a tie goes to the smaller code
          best = err;
          best_c = c;
        }
      }
    }
    // (error, code) minimum over the kLanes slots; ties go to the smaller code
#pragma unroll
    for (int o = 1; o < kLanes; o <<= 1) {
      const double oe = __shfl_xor_sync(0xffffffffu, best, o);
      const int oc = __shfl_xor_sync(0xffffffffu, best_c, o);
      if (oe < best || (oe == best && oc < best_c)) {
        best = oe;
        best_c = oc;
      }
    }
  }
  if (!valid || slot != 0) return;

  uint2 codes = make_uint2(0u, 0u);
  if (!zero) {
    const float d = s_d[best_c];
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      // a zero weight (either sign) gives code 0, also when d underflowed;
      // a tiny negative weight keeps its sign bit
      v[i] = w[i] == 0.0f ? 0.0f : w[i];
    }
    if (quot_fast_ok(d)) {
      float r_lo, r_hi;
      bracket_factors(d, r_lo, r_hi);
      codes = make_uint2(e2m1x8_quot(v, d, r_lo, r_hi), e2m1x8_quot(v + 8, d, r_lo, r_hi));
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = v[i] == 0.0f ? 0.0f : __fdiv_rn(v[i], d);
      codes = make_uint2(e2m1x8(v), e2m1x8(v + 8));
    }
  }
  if (MXQ_IN_RANGE(kChkMseOut, blk, n_blocks)) packed[blk] = codes;
  if (MXQ_IN_RANGE(kChkMseScale, blk, n_blocks)) block_scales[blk] = (uint8_t)best_c;
}

int mse_grid(int64_t n_blocks) {
  const int64_t threads = n_blocks * kLanes;
  const int64_t g = (threads + kMseThreads - 1) / kMseThreads;
  return (int)(g < 1 ? 1 : g);
}

}  // namespace

int launch_nvfp4_quantize_mse(const void* x, int dt, int64_t rows, int64_t K, void* packed,
                              void* block_scales, float* global_scale, uint32_t* amax_word,
                              cudaStream_t st) {
  const int64_t n_blocks = rows * (K / 16);
  if (n_blocks > ((int64_t)INT32_MAX * kMseThreads) / kLanes) return MXQ_ERR_UNSUPPORTED;
  launch_nvfp4_amax(x, dt, rows * K, amax_word, st);
  const int grid = mse_grid(n_blocks);
  auto* p = (uint2*)packed;
  auto* s = (uint8_t*)block_scales;
  switch (dt) {
    case kBF16:
      nvfp4_mse_kernel<kBF16><<<grid, kMseThreads, 0, st>>>(x, p, s, global_scale, amax_word,
                                                            n_blocks);
      break;
    case kF16:
      nvfp4_mse_kernel<kF16><<<grid, kMseThreads, 0, st>>>(x, p, s, global_scale, amax_word,
                                                           n_blocks);
      break;
    default:
      nvfp4_mse_kernel<kF32><<<grid, kMseThreads, 0, st>>>(x, p, s, global_scale, amax_word,
                                                           n_blocks);
      break;
  }
  return cudaGetLastError() == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

MXQ_DEFINE_CHECK_READER(check_record_nvfp4_mse)

}  // namespace mxq
