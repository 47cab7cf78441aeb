// Tensor-core grouped GEMM over MXFP4-packed expert weights (sm_100a).
//
// Semantics ("nemo_automodel.components.quantization.mxfp4",
// MXFP4GroupedMM): expert e owns activation rows [offs[e-1], offs[e]);
//   forward  (transpose_w = 0): y[t, n] = sum_k x[t, k]  W_e[n, k]
//   backward (transpose_w = 1): y[t, k] = sum_n g[t, n]  W_e[n, k]
// with W_e[n, k] = E2M1(nibble) * 2^(scale - 127) decoded on the fly from
// the packed [E, N, K/2] bytes and [E, N, K/32] E8M0 scales.
//
// Mapping onto tcgen05 (one CTA per SM, persistent over tiles):
//   D[m, j] (f32, TMEM)  +=  A[m, r] (bf16, TMEM)  *  B[j, r] (bf16, smem)
// with m = an output feature (a weight row n in the forward, a column k in
// the backward; 128 per tile), j = a token of the expert (256 per tile) and
// r = the reduction index (64 per pipeline stage).
//   * B (activations) arrives by TMA, 128-byte swizzled, K-major.
//   * A (weights) never exists in bf16 outside the SM: dequantization warps
//     read the packed bytes from global memory, decode them exactly to bf16
//     in registers and write them straight into TMEM with tcgen05.st.  In
//     the backward the 8x8 blocks are transposed in registers with
//     movmatrix first, since TMEM lanes must be the output features k.
//   * One thread issues tcgen05.mma (M=128, N=256, K=16) and signals stage
//     release with tcgen05.commit.
//   * Four epilogue warps drain D (tcgen05.ld), round to bf16, stage the
//     tile in shared memory and store rows that belong to the expert.
// Every mbarrier wait is bounded: on a time-out the CTA stops all roles,
// drains what it issued, frees TMEM and reports MXQ_ERR_TIMEOUT.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "mxq.h"
#include "mxq_device.cuh"
#include "mxq_grouped.cuh"
#include "mxq_launch.h"
#include "sm100_primitives.cuh"

namespace mxq {

int launch_grouped_mm_general(const void* a, const void* packed, const void* scales,
                              const int32_t* offs, int64_t T, int64_t E, int64_t N, int64_t K,
                              int transpose_w, void* y, int32_t* dev_status, cudaStream_t st);

namespace {

using namespace sm100;

constexpr int kBM = 128;        // output features per tile (MMA M, TMEM lanes)
constexpr int kBN = 256;        // tokens per tile (MMA N)
constexpr int kBK = 64;         // reduction elements per stage (128 bytes of bf16)
constexpr int kStages = 4;
constexpr int kTmemCols = 512;
constexpr int kDCol = 0;        // accumulator: columns [0, 256)
constexpr int kACol = 256;      // A stages: 32 columns (64 bf16) each
constexpr int kEpiWarps = 4;    // warps 0..3
constexpr int kDqWarps = 8;     // warps 4..11
constexpr int kTmaWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kThreads = 14 * 32;
constexpr uint32_t kStageBytesB = kBN * kBK * 2;    // 32 KB
constexpr uint32_t kStagingBytes = kBN * kBM * 2;   // 64 KB
constexpr uint32_t kSmemBytes = 1024 + kStages * kStageBytesB + kStagingBytes + 256;
constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kBN);
constexpr uint64_t kDrainLimitNs = 1000000000ull;

struct Shared {
  uint64_t full_a[kStages];
  uint64_t full_b[kStages];
  uint64_t empty[kStages];
  uint64_t d_full, d_empty, drain;
  uint32_t tmem_base;
  int abort;
};

// Two E2M1 codes (one byte) -> two exact bf16 values times 2^(s-127).
__device__ __forceinline__ uint32_t dequant_pair(uint32_t byte, float scale) {
  uint32_t h2 = e2m1x2_to_f16x2(byte);
  return pack2<kBF16>(f16lo(h2) * scale, f16hi(h2) * scale);
}

__device__ __forceinline__ float e8m0_scale(uint32_t s) { return exp2i((int)s - 127); }

__device__ __forceinline__ uint4 ldg16(const uint8_t* p) {
  return *reinterpret_cast<const uint4*>(p);
}

// Named barrier 1 over the four epilogue warps (threads 0..127).
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Barrier 1 plus an OR over the epilogue warps: a uniform decision.
__device__ __forceinline__ bool epi_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

// Bounded wait whose outcome is the same on every lane of the warp (the
// tcgen05 ld/st that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit_ns) {
  bool ok = mbar_wait(bar, parity, abort, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

template <bool kDgrad>
__global__ void __launch_bounds__(kThreads, 1)
grouped_mm_tc_kernel(const __grid_constant__ CUtensorMap tmap_act, const uint8_t* __restrict__ packed,
                     const uint8_t* __restrict__ scales, const int32_t* __restrict__ offs, int64_t T,
                     int64_t E, int64_t N, int64_t K, __nv_bfloat16* __restrict__ y,
                     int32_t* dev_status, uint64_t wait_limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sB = smem;
  uint16_t* sY = (uint16_t*)(smem + kStages * kStageBytesB);
  Shared* sh = (Shared*)(smem + kStages * kStageBytesB + kStagingBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (!offs_valid(offs, E, T)) {
    if (blockIdx.x == 0 && threadIdx.x == 0 && dev_status) *dev_status = MXQ_ERR_BAD_OFFS;
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh->full_a[s], kDqWarps);
      mbar_init(&sh->full_b[s], 1);
      mbar_init(&sh->empty[s], 1);
    }
    mbar_init(&sh->d_full, 1);
    mbar_init(&sh->d_empty, kEpiWarps);
    mbar_init(&sh->drain, 1);
    sh->abort = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sh->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kTmaWarp && lane == 0) prefetch_tmap(&tmap_act);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = sh->tmem_base;
  volatile int* abort = &sh->abort;
  const int64_t kin = kDgrad ? N : K;
  const int64_t nout = kDgrad ? K : N;
  const int nk = (int)(kin / kBK);
  const int64_t col_tiles = nout / kBM;

  if (warp == kTmaWarp) {
    // ------------------------------------------------ TMA producer (B)
    if (lane == 0) {
      TileWalker walk(offs, E, kBN, col_tiles);
      uint32_t it = 0;
      for (int64_t tile = blockIdx.x; !*abort && walk.seek(tile); tile += gridDim.x) {
        for (int ks = 0; ks < nk; ++ks, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&sh->empty[s], ((it / kStages) & 1) ^ 1, abort, wait_limit_ns)) break;
          mbar_arrive_expect_tx(&sh->full_b[s], kStageBytesB);
          tma_load_2d(smem_addr(sB + s * kStageBytesB), &tmap_act, ks * kBK, (int32_t)walk.row0,
                      &sh->full_b[s]);
        }
      }
      // Loads still in flight land before the CTA may exit.
      int abort_local = 0;
      for (uint32_t j = it > kStages ? it - kStages : 0; j < it; ++j)
        mbar_wait(&sh->full_b[j % kStages], (j / kStages) & 1, &abort_local, kDrainLimitNs);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      TileWalker walk(offs, E, kBN, col_tiles);
      uint32_t it = 0, lt = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; ok && walk.seek(tile); tile += gridDim.x, ++lt) {
        if (!(ok = mbar_wait(&sh->d_empty, (lt & 1) ^ 1, abort, wait_limit_ns))) break;
        tc_fence_after();
        for (int ks = 0; ks < nk; ++ks, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!(ok = mbar_wait(&sh->full_a[s], ph, abort, wait_limit_ns))) break;
          if (!(ok = mbar_wait(&sh->full_b[s], ph, abort, wait_limit_ns))) break;
          tc_fence_after();
          const uint64_t bdesc = smem_desc_sw128(smem_addr(sB + s * kStageBytesB));
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_bf16_ts(tmem + kDCol, tmem + kACol + 32 * s + 8 * kk, bdesc + 2 * kk, kIdesc,
                        (ks | kk) != 0);
          mma_commit(&sh->empty[s]);
        }
        if (ok) mma_commit(&sh->d_full);
      }
      // Every MMA issued has completed before TMEM is released.
      mma_commit(&sh->drain);
      int abort_local = 0;
      mbar_wait(&sh->drain, 0, &abort_local, kDrainLimitNs);
    }
    __syncwarp();
  } else if (warp >= kEpiWarps) {
    // -------------------------------------------- dequantization (A)
    const int q = warp & 3;          // TMEM lane quarter
    const int h = (warp - kEpiWarps) >> 2;  // which half of the 64-wide stage
    TileWalker walk(offs, E, kBN, col_tiles);
    uint32_t it = 0;
    for (int64_t tile = blockIdx.x; !*abort && walk.seek(tile); tile += gridDim.x) {
      const int64_t e = walk.expert;
      const int64_t m0 = walk.col_tile * kBM;
      if constexpr (!kDgrad) {
        // Thread = weight row n; 32 consecutive k per stage half.
        const int64_t n = m0 + 32 * q + lane;
        const uint8_t* prow = packed + (e * N + n) * (K / 2) + 16 * h;
        const uint8_t* srow = scales + (e * N + n) * (K / 32) + h;
        uint4 pb[4];
        uint32_t sb[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (j < nk) {
            pb[j] = ldg16(prow + 32 * j);
            sb[j] = srow[2 * j];
          }
        bool ok = true;
        for (int ks0 = 0; ks0 < nk && ok; ks0 += 4) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int ks = ks0 + j;
            if (ks >= nk || !ok) break;
            const uint4 d = pb[j];
            const float sc = e8m0_scale(sb[j]);
            if (ks + 4 < nk) {
              pb[j] = ldg16(prow + 32 * (ks + 4));
              sb[j] = srow[2 * (ks + 4)];
            }
            uint32_t v[16];
            const uint32_t w[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = dequant_pair((w[i >> 2] >> (8 * (i & 3))) & 0xFFu, sc);
            const int s = it % kStages;
            if (!(ok = warp_wait(&sh->empty[s], ((it / kStages) & 1) ^ 1, abort, wait_limit_ns)))
              break;
            tc_fence_after();
            tmem_st_32x32b_x16(tmem + ((uint32_t)(32 * q) << 16) + kACol + 32 * s + 16 * h, v);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh->full_a[s]);
            ++it;
          }
        }
      } else {
        // Output features k = m0 + 32q + (0..31) are the TMEM lanes of this
        // warp; each stage half covers 32 reduction indices n.  Thread t
        // decodes byte (n0 + t/4, k/2 = kq/2 + 8r + 4b + t%4) for its four
        // rows n0 = base + 8j, then movmatrix transposes each 8x8 block.
        const int64_t kq = m0 + 32 * q;
        const int rsub = lane >> 2, csub = lane & 3;
        const uint8_t* pcol = packed + e * N * (K / 2) + kq / 2;
        const uint8_t* scol = scales + e * N * (K / 32) + kq / 32;
        uint4 pb[2][4];
        uint32_t sb[2][4];
        auto load = [&](int ks, uint4* P, uint32_t* S) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int64_t n = (int64_t)ks * kBK + 32 * h + 8 * j + rsub;
            P[j] = ldg16(pcol + n * (K / 2));
            S[j] = scol[n * (K / 32)];
          }
        };
        load(0, pb[0], sb[0]);
        if (nk > 1) load(1, pb[1], sb[1]);
        bool ok = true;
        for (int ks0 = 0; ks0 < nk && ok; ks0 += 2) {
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int ks = ks0 + u;
            if (ks >= nk || !ok) break;
            uint32_t v[2][8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float sc = e8m0_scale(sb[u][j]);
              const uint32_t w[4] = {pb[u][j].x, pb[u][j].y, pb[u][j].z, pb[u][j].w};
#pragma unroll
              for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                  const uint32_t byte = (w[2 * r + b] >> (8 * csub)) & 0xFFu;
                  v[r][2 * j + b] = movmatrix_trans(dequant_pair(byte, sc));
                }
            }
            if (ks + 2 < nk) load(ks + 2, pb[u], sb[u]);
            const int s = it % kStages;
            if (!(ok = warp_wait(&sh->empty[s], ((it / kStages) & 1) ^ 1, abort, wait_limit_ns)))
              break;
            tc_fence_after();
#pragma unroll
            for (int r = 0; r < 2; ++r)
              tmem_st_16x128b_x4(tmem + ((uint32_t)(32 * q + 16 * r) << 16) + kACol + 32 * s + 16 * h,
                                 v[r]);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh->full_a[s]);
            ++it;
          }
        }
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    TileWalker walk(offs, E, kBN, col_tiles);
    uint32_t lt = 0;
    for (int64_t tile = blockIdx.x; walk.seek(tile); tile += gridDim.x, ++lt) {
      // (also: the previous tile's staged rows have been stored)
      if (epi_any(*abort != 0)) break;
      const bool ok = mbar_wait(&sh->d_full, lt & 1, abort, wait_limit_ns);
      if (epi_any(!ok)) break;
      tc_fence_after();
      const int col = 32 * warp + lane;  // output feature within the tile
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * warp) << 16) + kDCol + 32 * c, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j)
          sY[(32 * c + j) * kBM + col] =
              __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j])));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->d_empty);
      epi_bar();  // the whole tile is staged
      const int64_t row0 = walk.row0;
      const int64_t rows = walk.row_end - row0 < kBN ? walk.row_end - row0 : kBN;
      const int64_t o0 = walk.col_tile * kBM;
      // two rows of 128 outputs (256 bytes each) per warp instruction
      for (int r = 2 * warp + (lane >> 4); r < rows; r += 2 * kEpiWarps) {
        const uint4 val = *reinterpret_cast<const uint4*>(sY + r * kBM + 8 * (lane & 15));
        *reinterpret_cast<uint4*>(y + (row0 + r) * nout + o0 + 8 * (lane & 15)) = val;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort && dev_status) atomicExch(dev_status, MXQ_ERR_TIMEOUT);
}

// ------------------------------------------------------------------ host

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  });
  return fn;
}

// Row-major bf16 [rows, cols] activations, boxes of 64 columns x 256 rows,
// 128-byte swizzle; rows past the end read as zero.
bool make_act_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {kBK, kBN};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

uint64_t g_wait_limit_ns = 2000000000ull;

template <bool kDgrad>
int launch_tc(const void* a, const void* packed, const void* scales, const int32_t* offs,
              int64_t T, int64_t E, int64_t N, int64_t K, void* y, int32_t* dev_status,
              cudaStream_t st) {
  const int64_t kin = kDgrad ? N : K, nout = kDgrad ? K : N;
  CUtensorMap map;
  if (!make_act_map(&map, a, T, kin)) return MXQ_ERR_CUDA;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(grouped_mm_tc_kernel<kDgrad>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  });
  if (attr_err != cudaSuccess) return MXQ_ERR_CUDA;
  int64_t tiles = ((T + kBN - 1) / kBN + E) * (nout / kBM);
  int64_t grid = tiles < num_sms() ? tiles : num_sms();
  grouped_mm_tc_kernel<kDgrad><<<(int)grid, kThreads, kSmemBytes, st>>>(
      map, (const uint8_t*)packed, (const uint8_t*)scales, offs, T, E, N, K, (__nv_bfloat16*)y,
      dev_status, g_wait_limit_ns);
  return cudaGetLastError() == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

}  // namespace

void set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns = ns; }

int launch_grouped_mm(const void* a, const void* packed, const void* scales, const int32_t* offs,
                      int64_t T, int64_t E, int64_t N, int64_t K, int transpose_w, void* y,
                      int32_t* dev_status, cudaStream_t st) {
  const int64_t kin = transpose_w ? N : K, nout = transpose_w ? K : N;
  const bool tc = kin % kBK == 0 && nout % kBM == 0 && ((uintptr_t)a & 15) == 0 &&
                  ((uintptr_t)y & 15) == 0 && T < (int64_t)1 << 31 && kin < (int64_t)1 << 31;
  if (tc) {
    return transpose_w ? launch_tc<true>(a, packed, scales, offs, T, E, N, K, y, dev_status, st)
                       : launch_tc<false>(a, packed, scales, offs, T, E, N, K, y, dev_status, st);
  }
  return launch_grouped_mm_general(a, packed, scales, offs, T, E, N, K, transpose_w, y,
                                   dev_status, st);
}

}  // namespace mxq
