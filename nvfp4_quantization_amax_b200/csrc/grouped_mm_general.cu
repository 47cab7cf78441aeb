// General grouped GEMM over MXFP4-packed expert weights (any N, K, T, E,
// any alignment): CUDA-core FMA with smem tiling.  The tensor-core kernel
// (grouped_mm_tc.cu) takes the shapes it supports; this kernel covers the
// rest.  Semantics follow "nemo_automodel.components.quantization.mxfp4",
// MXFP4GroupedMM: forward y = x . W_e^T, backward grad_x = grad_out . W_e,
// with W_e dequantized on the fly (low nibble = even column, one E8M0 scale
// per 32 columns) and expert e owning rows [offs[e-1], offs[e]).
#include <cuda_bf16.h>

#include "mxq_device.cuh"
#include "mxq_grouped.cuh"
#include "mxq_launch.h"

namespace mxq {

namespace {

constexpr int kTM = 64, kTN = 64, kTK = 32, kGThreads = 256;

__constant__ float kE2M1Value[16] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f,
                                     0.0f, -0.5f, -1.0f, -1.5f, -2.0f, -3.0f, -4.0f, -6.0f};

__device__ __forceinline__ float weight_at(const uint8_t* packed, const uint8_t* scales,
                                           int64_t K, int64_t n, int64_t k, int64_t N) {
  if (!MXQ_IN_RANGE(kChkGemmGenW, n * K + k, N * K)) return 0.0f;
  uint32_t byte = packed[n * (K / 2) + k / 2];
  uint32_t nib = (k & 1) ? (byte >> 4) : (byte & 15u);
  uint32_t s = scales[n * (K / 32) + k / 32];
  if (s == 0xFFu) return __uint_as_float(0x7FC00000u);
  return kE2M1Value[nib] * exp2i((int)s - 127);
}

__global__ void __launch_bounds__(kGThreads)
grouped_mm_general_kernel(const __nv_bfloat16* __restrict__ a, const uint8_t* __restrict__ packed,
                          const uint8_t* __restrict__ scales, const int32_t* __restrict__ offs,
                          int64_t T, int64_t E, int64_t N, int64_t K, int transpose_w,
                          __nv_bfloat16* __restrict__ y, int32_t* dev_status) {
  __shared__ float As[kTK][kTM + 1];
  __shared__ float Ws[kTK][kTN + 1];
  if (!offs_valid(offs, E, T)) {
    if (blockIdx.x == 0 && threadIdx.x == 0 && dev_status) *dev_status = MXQ_ERR_BAD_OFFS;
    return;
  }
  const int64_t kin = transpose_w ? N : K;
  const int64_t nout = transpose_w ? K : N;
  const int64_t n_tiles_o = (nout + kTN - 1) / kTN;
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  TileWalker walk(offs, E, kTM, n_tiles_o);
  for (int64_t tile = blockIdx.x; walk.seek(tile); tile += gridDim.x) {
    const int64_t e = walk.expert, row0 = walk.row0, row_end = walk.row_end;
    const int64_t o0 = walk.col_tile * kTN;
    const uint8_t* pe = packed + e * N * (K / 2);
    const uint8_t* se = scales + e * N * (K / 32);
    float acc[4][4] = {};
    for (int64_t r0 = 0; r0 < kin; r0 += kTK) {
      for (int i = tid; i < kTM * kTK; i += kGThreads) {
        int t = i / kTK, kk = i % kTK;
        int64_t row = row0 + t, r = r0 + kk;
        As[kk][t] = (row < row_end && r < kin && MXQ_IN_RANGE(kChkGemmGenIn, row * kin + r, T * kin))
                        ? __bfloat162float(a[row * kin + r])
                        : 0.0f;
      }
      for (int i = tid; i < kTN * kTK; i += kGThreads) {
        int o = i / kTK, kk = i % kTK;
        int64_t oc = o0 + o, r = r0 + kk;
        float w = 0.0f;
        if (oc < nout && r < kin)
          w = transpose_w ? weight_at(pe, se, K, r, oc, N) : weight_at(pe, se, K, oc, r, N);
        Ws[kk][o] = w;
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < kTK; ++kk) {
        float av[4], wv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) wv[j] = Ws[kk][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], wv[j], acc[i][j]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int64_t row = row0 + ty * 4 + i;
      if (row >= row_end) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int64_t oc = o0 + tx * 4 + j;
        if (oc < nout && MXQ_IN_RANGE(kChkGemmGenOut, row * nout + oc, T * nout))
          y[row * nout + oc] = __float2bfloat16_rn(acc[i][j]);
      }
    }
  }
}

}  // namespace

int launch_grouped_mm_general(const void* a, const void* packed, const void* scales,
                              const int32_t* offs, int64_t T, int64_t E, int64_t N, int64_t K,
                              int transpose_w, void* y, int32_t* dev_status, cudaStream_t st) {
  int64_t nout = transpose_w ? K : N;
  // Upper bound on the tile count: every expert may add one ragged tile.
  int64_t tiles = ((T + kTM - 1) / kTM + E) * ((nout + kTN - 1) / kTN);
  int64_t grid = tiles < (int64_t)num_sms() * 4 ? tiles : (int64_t)num_sms() * 4;
  if (grid < 1) grid = 1;
  grouped_mm_general_kernel<<<(int)grid, kGThreads, 0, st>>>(
      (const __nv_bfloat16*)a, (const uint8_t*)packed, (const uint8_t*)scales, offs, T, E, N, K,
      transpose_w, (__nv_bfloat16*)y, dev_status);
  return cudaGetLastError() == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

MXQ_DEFINE_CHECK_READER(check_record_grouped_mm_general)

}  // namespace mxq
