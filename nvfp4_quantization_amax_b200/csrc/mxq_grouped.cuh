// Expert-partition helpers shared by the grouped GEMM kernels.
//
// offs[e] is the end (exclusive) of expert e's contiguous rows, so expert e
// owns rows [offs[e-1], offs[e]) with offs[-1] = 0 ("cumulative token
// counts", "nemo_automodel.components.quantization.mxfp4", MXFP4GroupedMM).
#pragma once

#include <cstdint>

#include "mxq_device.cuh"

namespace mxq {

// Weight decode of the tensor-core kernels: two E2M1 codes (one byte, low
// nibble first) -> two bf16 values times the block scale 2^(s-127): exact
// E2M1 -> f16 (cvt), exact f32 products, one rounding to bf16 that is exact
// whenever the weight is a bf16 value (every scale byte up to 252).
// 2^(s - 127) as f32: the exponent field s for s >= 1 (255 gives +inf, as
// exp2i(128) does), the subnormal 2^-127 for s = 0.
__device__ __forceinline__ float mx_block_scale(uint32_t s) {
  return __uint_as_float(max(s << 23, 0x00400000u));  // s <= 255: s << 23 >= 2^23 unless s = 0
}

__device__ __forceinline__ uint32_t mx_dequant_pair(uint32_t byte, float scale) {
  const uint32_t h2 = e2m1x2_to_f16x2(byte);
  float lo, hi;
  mul2_rn(lo, hi, f16lo(h2), f16hi(h2), scale, scale);
  return pack2<kBF16>(lo, hi);
}

// True iff offs is non-negative, non-decreasing and ends at T.  Called by
// every thread of a CTA (contains __syncthreads); block-uniform result.
__device__ __forceinline__ bool offs_valid(const int32_t* offs, int64_t E, int64_t T) {
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = (offs[E - 1] != T) ? 1 : 0;
  __syncthreads();
  for (int64_t e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t prev = e == 0 ? 0 : offs[e - 1];
    if (offs[e] < prev) s_bad = 1;
  }
  __syncthreads();
  return s_bad == 0;
}

// Maps a linear tile index to (expert, row tile, column tile).  Tiles are
// numbered expert by expert; inside an expert the column tile varies
// fastest, so consecutive tiles share the same rows of the activation.
// Sought indices must not decrease (each CTA walks its tiles in order).
struct TileWalker {
  const int32_t* offs;
  int64_t E;
  int64_t tile_rows;
  int64_t col_tiles;
  int64_t expert = 0;
  int64_t first_tile = 0;
  int64_t row0 = 0, row_end = 0, col_tile = 0;

  __device__ TileWalker(const int32_t* o, int64_t e, int64_t tr, int64_t ct)
      : offs(o), E(e), tile_rows(tr), col_tiles(ct) {}

  __device__ bool seek(int64_t tile) {
    while (expert < E) {
      int64_t lo = expert == 0 ? 0 : offs[expert - 1];
      int64_t hi = offs[expert];
      int64_t count = ((hi - lo + tile_rows - 1) / tile_rows) * col_tiles;
      if (tile < first_tile + count) {
        int64_t local = tile - first_tile;
        col_tile = local % col_tiles;
        row0 = lo + (local / col_tiles) * tile_rows;
        row_end = hi;
        return true;
      }
      first_tile += count;
      ++expert;
    }
    return false;
  }
};

}  // namespace mxq
