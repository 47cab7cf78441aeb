// W4A4 grouped GEMMs on the block-scaled tensor cores (sm_100a): both the
// expert weights and the activations are 4-bit E2M1 codes (two per byte)
// with block scales, multiplied by tcgen05.mma with the scales applied
// inside the tensor core ("NVIDIA Model Optimizer: from mtq.quantize to a
// 4.95-bit DeepSeek-R1", section on W4A4 NVFP4 on FP4 tensor cores).  Two
// formats share the kernel:
//   MXFP4: one E8M0 scale per 32 K ("nemo_automodel.components.quantization.
//          mxfp4"), kind::mxf4, y = sum_k xq[t, k] W_e[n, k];
//   NVFP4: one UE4M3 scale per 16 K plus a per-tensor f32 scale for the
//          activations and one per expert weight ("NVFP4 in the code: two
//          scales and a nibble"), kind::mxf4nvf4, y = g_x g_w[e] sum_k ...
// The activations come quantized (mx_quantize / nvfp4_quantize), so every
// product of codes and block scales is exact and the tensor core only
// rounds the f32 accumulation; y is rounded once to bf16 (NVFP4: after the
// f32 product with g_x g_w[e]).
//
// Mapping (persistent, one CTA per SM, eight warps):
//   D[m, j] (f32, TMEM) += A[m, k] (weights, smem) * B[j, k] (tokens, smem)
// with m one of the CTA's 128 weight rows (TMEM lanes), j one of up to 256
// tokens of the expert and k the reduction index, 256 per pipeline stage
// (128 bytes of codes per row: one 128-byte-swizzled TMA row).
//   * warp 4 (one lane) TMA-loads both code tiles of a stage;
//   * warps 5 and 6 gather the stage's scale bytes (8 or 16 per row: 128
//     weight rows and 256 token rows, half of them each) from the row-major
//     [rows, K/32 or K/16] scale arrays and write them into the tensor
//     core's scale layout in shared memory: blocks of 128 rows x 4 scales,
//     row r at byte 16 (r % 32) + 4 (r / 32) + the scale's index.  Where the
//     rows allow it they load a row's scales of several stages at once (32
//     bytes: one L2 sector when the row is sector-aligned), since one
//     sector per row and stage is as many bytes into the SM as a quarter
//     of the stage's codes;
//   * warp 7 (one lane) copies those blocks into TMEM (tcgen05.cp, 32 lanes
//     x 128 bits, replicated to the four lane quarters) and issues four
//     K=64 MMAs per stage, each selecting its scales by block and byte id;
//   * warps 0-3 drain D, round to bf16, stage the tile in shared memory
//     (in passes of 64-128 tokens for NVFP4 and for the two-accumulator
//     tile, which leaves room for a third stage) and store the expert's
//     rows.
// The launch allows the CTAs to start while the previous kernel on the
// stream finishes (programmatic stream serialization): they set up their
// barriers and TMEM, then wait for that kernel's results before reading any
// input.  Every mbarrier wait is bounded: on a time-out the CTA stops all
// roles, drains what it issued, frees TMEM and reports MXQ_ERR_TIMEOUT.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "mxq.h"
#include "mxq_device.cuh"
#include "mxq_grouped.cuh"
#include "mxq_launch.h"
#include "sm100_primitives.cuh"
#include "tmap.h"

namespace mxq {

namespace {

using namespace sm100;

constexpr int kM = 128;                 // weight rows per MMA (TMEM lanes)
constexpr int kKB = 128;                // bytes of codes per row per stage (256 K)
constexpr int kMaxStages = 3;
constexpr uint32_t kSfBlock = 512;                // 128 rows x 4 scales
constexpr int kMaxSmemExperts = 256;
constexpr int kTmemCols = 512;

// The two block-scaled formats: MXFP4 (one E8M0 scale per 32 K; a stage's
// 8 scales per row fill 2 blocks, each MMA uses half a TMEM word) and NVFP4
// (one UE4M3 scale per 16 K; 16 scales per row, 4 blocks, each MMA uses a
// whole word), and two tile shapes: 128 weight rows x 256 tokens, or
// (kBig, when N is a multiple of 256) 256 weight rows x 224 tokens, two
// M=128 MMAs sharing each token tile (fewer operand bytes and scale copies
// per product; 224 is what TMEM holds beside the NVFP4 scale columns, and
// an expert of up to 1120 tokens takes five token tiles).
template <bool kNV, bool kBig>
struct W4Fmt {
  static constexpr int kScalesPerRow = kNV ? 16 : 8;       // per stage (256 K)
  static constexpr int kBlocks = kScalesPerRow / 4;         // per 128-row group
  static constexpr int kMG = kBig ? 2 : 1;                  // 128-row weight groups per tile
  static constexpr int kTileM = kM * kMG;                   // weight rows per tile
  static constexpr int kTileN = kBig ? 224 : 256;           // tokens per tile (MMA N)
  static constexpr uint32_t kABytes = kTileM * kKB;
  static constexpr uint32_t kBBytes = kTileN * kKB;
  static constexpr uint32_t kSfaBytes = kMG * kBlocks * kSfBlock;
  static constexpr uint32_t kSfbBytes = 2 * kBlocks * kSfBlock;  // two 128-row groups
  // TMEM: the kMG accumulators (kTileN columns each), then the A scales
  // (4 columns per block, group-major), then the B scales (8 per block).
  static constexpr int kSfaCol = kMG * kTileN;
  static constexpr int kSfbCol = kSfaCol + 4 * kMG * kBlocks;
  static constexpr int kStages = 3;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
  // Output tokens staged in shared memory at a time (bf16, 128 features
  // each): 128 x 256 tiles stage all 256 (MXFP4) or 128 (NVFP4, whose
  // stages carry twice the scale bytes) so that three stages fit; 256 x 224
  // tiles 96 (MXFP4) or 64 (NVFP4) of an accumulator's 224 per pass.
  static constexpr int kYRows = kBig ? (kNV ? 64 : 96) : (kNV ? 128 : 256);
  static constexpr uint32_t kStagingBytes = kYRows * kM * 2;
  static constexpr uint32_t kSmem =
      1024 + kStages * kStageBytes + kStagingBytes + 256 + 4 * kMaxSmemExperts;
  static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte alignment of swizzled tiles");
  static_assert(kSmem <= 232448, "shared memory per CTA");
  static_assert(kSfbCol + 8 * kBlocks <= kTmemCols, "TMEM columns");
};
constexpr int kEpiWarps = 4;
constexpr int kTmaWarp = 4;
constexpr int kSfWarp = 5;   // warps 5 and 6
constexpr int kSfWarps = 2;
constexpr int kMmaWarp = 7;
constexpr int kThreads = 8 * 32;
constexpr uint64_t kDrainLimitNs = 1000000000ull;


struct Shared {
  uint64_t full[kMaxStages];   // codes (TMA bytes) and scales (warp 5) of a stage are in smem
  uint64_t empty[kMaxStages];  // the stage's MMAs (and scale copies) completed
  uint64_t d_full, d_empty, drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ int64_t mma_n(int64_t rows) { return (rows + 15) & ~15; }

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

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

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit_ns) {
  const bool ok = mbar_wait(bar, parity, abort, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// Byte offset of (row r, scale s) inside a 128-row block of the tensor
// core's scale layout (s in 0..3).
__device__ __forceinline__ uint32_t sf_offset(int r) { return 16 * (r & 31) + 4 * ((r >> 5) & 3); }

// kWide: each scale load covers kG stages (32 bytes per row); otherwise one
// stage (8 or 16 bytes per row).  kBig: the 256 x 224 tile.
template <bool kNV, bool kWide, bool kBig>
__global__ void __launch_bounds__(kThreads, 1)
w4a4_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
               const uint8_t* __restrict__ x_scales, const uint8_t* __restrict__ w_scales,
               const float* __restrict__ x_global, const float* __restrict__ w_global,
               const int32_t* __restrict__ offs, int64_t T, int64_t E, int64_t N, int64_t K,
               __nv_bfloat16* __restrict__ y, int32_t* dev_status, uint64_t wait_limit_ns) {
  using F = W4Fmt<kNV, kBig>;
  constexpr int kStages = F::kStages;
  constexpr uint32_t kABytes = F::kABytes, kBBytes = F::kBBytes;
  constexpr int kTileN = F::kTileN, kMG = F::kMG;
  constexpr int kSfaCol = F::kSfaCol;
  constexpr uint32_t kStageBytes = F::kStageBytes;
  constexpr uint32_t kSfaBytes = F::kSfaBytes;
  constexpr int kSfbCol = F::kSfbCol;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint16_t* sY = (uint16_t*)(smem + kStages * kStageBytes);
  Shared* sh = (Shared*)((uint8_t*)sY + F::kStagingBytes);
  int32_t* s_offs = (int32_t*)((uint8_t*)sh + 256);
  auto sA = [&](int s) { return smem + s * kStageBytes; };
  auto sB = [&](int s) { return smem + s * kStageBytes + kABytes; };
  auto sSfa = [&](int s) { return smem + s * kStageBytes + kABytes + kBBytes; };
  auto sSfb = [&](int s) { return smem + s * kStageBytes + kABytes + kBBytes + kSfaBytes; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Set-up that reads nothing the previous kernel on the stream may still be
  // writing (the launch lets this CTA start while that kernel finishes).
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh->full[s], 1 + kSfWarps);  // TMA expect_tx arrive + scale warp arrives
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
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tmap(&tmap_x);
    prefetch_tmap(&tmap_w);
  }
  griddep_wait();  // the previous kernel's results (e.g. the activations) are complete
  if (!offs_valid(offs, E, T)) {  // (contains __syncthreads)
    if (blockIdx.x == 0 && threadIdx.x == 0 && dev_status) *dev_status = MXQ_ERR_BAD_OFFS;
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
      tc_fence_after();
      tmem_dealloc(sh->tmem_base, kTmemCols);
    }
    return;
  }
  const int32_t* t_offs = offs;
  if (E <= kMaxSmemExperts) {
    for (int64_t e = threadIdx.x; e < E; e += blockDim.x) s_offs[e] = offs[e];
    t_offs = s_offs;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = sh->tmem_base;
  volatile int* abort = &sh->abort;
  const int nk = (int)(K / 256);
  const int64_t col_tiles = N / F::kTileM;
  const int64_t srow = K / (kNV ? 16 : 32);  // scale bytes per row

  if (warp == kTmaWarp) {
    // --------------------------------------------------- TMA producer
    if (lane == 0) {
      TileWalker walk(t_offs, E, kTileN, col_tiles);
      uint32_t it = 0;
      for (int64_t tile = blockIdx.x; !*abort && walk.seek(tile); tile += gridDim.x) {
        const int32_t wy = (int32_t)(walk.expert * N + walk.col_tile * F::kTileM);
        const int32_t xy = (int32_t)walk.row0;
        bool ok = true;
        for (int ks = 0; ks < nk; ++ks, ++it) {
          const int s = it % kStages;
          if (!(ok = mbar_wait(&sh->empty[s], ((it / kStages) & 1) ^ 1, abort, wait_limit_ns)))
            break;
          mbar_arrive_expect_tx(&sh->full[s], kABytes + kBBytes);
          tma_load_2d(smem_addr(sA(s)), &tmap_w, ks * kKB, wy, &sh->full[s]);
          tma_load_2d(smem_addr(sB(s)), &tmap_x, ks * kKB, xy, &sh->full[s]);
        }
        if (!ok) break;
      }
      int abort_local = 0;
      for (uint32_t j = it > (uint32_t)kStages ? it - kStages : 0; j < it; ++j)
        mbar_wait(&sh->full[j % kStages], (j / kStages) & 1, &abort_local, kDrainLimitNs);
    }
    __syncwarp();
  } else if (warp >= kSfWarp && warp < kSfWarp + kSfWarps) {
    // ------------------------------------------- scale-factor producers
    // Stage ks needs scales kSPR ks .. kSPR ks + kSPR - 1 of every row:
    // weight rows n0 + m and token rows row0 + r (zero past the expert's
    // rows).  Scale warp u takes m = lane + 32 (kRowsW u + i) and
    // r = lane + 32 (kRowsX u + i).  Scales 0-3 go to block 0, 4-7 to
    // block 1, ... (of each 128-row group).  A load brings a row's scales of
    // kG consecutive stages (a group); the loads run one group ahead of the
    // stores (a cursor of its own walks the same (tile, group) sequence), so
    // their latency overlaps the tensor core's work.
    constexpr int kSPR = F::kScalesPerRow;
    constexpr int kG = kWide ? 32 / kSPR : 1;      // stages per load
    constexpr int kW = kG * kSPR / 4;              // 32-bit words per row and load
    constexpr int kRowsW = F::kTileM / (32 * kSfWarps);
    constexpr int kRowsX = (kTileN + 32 * kSfWarps - 1) / (32 * kSfWarps);  // rows past the tile read as 0
    const int u = warp - kSfWarp;
    using Buf = uint32_t[kRowsW + kRowsX][kW];
    TileWalker pwalk(t_offs, E, kTileN, col_tiles);
    int64_t ptile = blockIdx.x;
    bool phave = pwalk.seek(ptile);
    int pg = 0;  // group within the cursor's tile
    auto load_row = [&](uint32_t (&w)[kW], const uint8_t* p) {
      if constexpr (kW == 2) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
        w[0] = v.x; w[1] = v.y;
      } else {
#pragma unroll
        for (int h = 0; h < kW / 4; ++h) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(p) + h);
          w[4 * h] = v.x; w[4 * h + 1] = v.y; w[4 * h + 2] = v.z; w[4 * h + 3] = v.w;
        }
      }
    };
    auto issue = [&](Buf& buf) {
      if (!phave) return;
      const int64_t rows =
          pwalk.row_end - pwalk.row0 < kTileN ? pwalk.row_end - pwalk.row0 : kTileN;
      const int64_t wrow0 = pwalk.expert * N + pwalk.col_tile * F::kTileM;
      const int64_t col = (int64_t)4 * kW * pg;  // first scale byte of the group
#pragma unroll
      for (int i = 0; i < kRowsW; ++i) {
        const int64_t row = wrow0 + lane + 32 * (kRowsW * u + i);
        if (MXQ_IN_RANGE(kChkW4Scale, row * srow + col + 4 * kW - 1, E * N * srow))
          load_row(buf[i], w_scales + row * srow + col);
        else
#pragma unroll
          for (int k = 0; k < kW; ++k) buf[i][k] = 0u;
      }
#pragma unroll
      for (int i = 0; i < kRowsX; ++i) {
        const int r = lane + 32 * (kRowsX * u + i);
        const int64_t row = pwalk.row0 + r;
        if (r < rows && MXQ_IN_RANGE(kChkW4Scale, row * srow + col + 4 * kW - 1, T * srow))
          load_row(buf[kRowsW + i], x_scales + row * srow + col);
        else
#pragma unroll
          for (int k = 0; k < kW; ++k) buf[kRowsW + i][k] = 0u;
      }
      if (++pg * kG == nk) {
        pg = 0;
        ptile += gridDim.x;
        phave = pwalk.seek(ptile);
      }
    };
    // Stage q of the group in buf: word q kBlocks + b of a row (its scales
    // 4b..4b+3 of the stage) goes to block b; B blocks are ordered
    // (group 0, block b), (group 1, block b) for b = 0, 1, ...
    auto store = [&](int s, const Buf& buf, auto qc) {
      constexpr int q = decltype(qc)::value;
      uint8_t* fa = sSfa(s);
      uint8_t* fb = sSfb(s);
#pragma unroll
      for (int i = 0; i < kRowsW; ++i) {
        const int m = lane + 32 * (kRowsW * u + i);  // weight row of the tile
        const uint32_t o = sf_offset(m);
        const int g = m >> 7;  // 128-row group
#pragma unroll
        for (int b = 0; b < F::kBlocks; ++b)
          *reinterpret_cast<uint32_t*>(fa + (g * F::kBlocks + b) * kSfBlock + o) =
              buf[i][q * F::kBlocks + b];
      }
#pragma unroll
      for (int i = 0; i < kRowsX; ++i) {
        const int r = lane + 32 * (kRowsX * u + i);
        const uint32_t o = sf_offset(r);
        const int g = r >> 7;  // 128-row group
#pragma unroll
        for (int b = 0; b < F::kBlocks; ++b)
          *reinterpret_cast<uint32_t*>(fb + (2 * b + g) * kSfBlock + o) =
              buf[kRowsW + i][q * F::kBlocks + b];
      }
      fence_proxy_async_smem();  // visible to tcgen05.cp
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->full[s]);
    };
    // Stage q (runtime) of the group in buf, dispatched to a constant index.
    auto store_q = [&](int s, const Buf& buf, int q) {
      if constexpr (kG == 1) {
        store(s, buf, std::integral_constant<int, 0>{});
      } else if constexpr (kG == 2) {
        if (q == 0) store(s, buf, std::integral_constant<int, 0>{});
        else store(s, buf, std::integral_constant<int, 1>{});
      } else {
        static_assert(kG == 4, "stages per scale load");
        switch (q) {
          case 0: store(s, buf, std::integral_constant<int, 0>{}); break;
          case 1: store(s, buf, std::integral_constant<int, 1>{}); break;
          case 2: store(s, buf, std::integral_constant<int, 2>{}); break;
          default: store(s, buf, std::integral_constant<int, 3>{}); break;
        }
      }
    };
    Buf ba, bb;
    issue(ba);
    issue(bb);
    TileWalker walk(t_offs, E, kTileN, col_tiles);
    uint32_t it = 0, grp = 0;
    bool ok = true;
    for (int64_t tile = blockIdx.x; ok && walk.seek(tile); tile += gridDim.x) {
      for (int ks = 0; ks < nk && ok; ++ks, ++it) {
        const int s = it % kStages;
        if (!(ok = warp_wait(&sh->empty[s], ((it / kStages) & 1) ^ 1, abort, wait_limit_ns)))
          break;
        // group `grp` was loaded into buffer grp % 2; once its last stage
        // is stored, refill that buffer with group grp + 2
        const int q = ks % kG;
        const bool last = q == kG - 1;
        if ((grp & 1) == 0) {
          store_q(s, ba, q);
          if (last) issue(ba);
        } else {
          store_q(s, bb, q);
          if (last) issue(bb);
        }
        if (last) ++grp;
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      TileWalker walk(t_offs, E, kTileN, col_tiles);
      uint32_t it = 0, lt = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; ok && walk.seek(tile); tile += gridDim.x, ++lt) {
        if (!(ok = mbar_wait(&sh->d_empty, (lt & 1) ^ 1, abort, wait_limit_ns))) break;
        tc_fence_after();
        const int64_t rows =
            walk.row_end - walk.row0 < kTileN ? walk.row_end - walk.row0 : kTileN;
        const int n = (int)mma_n(rows);
        for (int ks = 0; ks < nk; ++ks, ++it) {
          const int s = it % kStages;
          if (!(ok = mbar_wait(&sh->full[s], (it / kStages) & 1, abort, wait_limit_ns))) break;
          tc_fence_after();
          // scales of the stage into TMEM (A: (group, block) group-major,
          // 4 columns each; B: (group, block) pairs (0,0) (1,0) (0,1) (1,1),
          // 8 columns per block index)
#pragma unroll
          for (int b = 0; b < kMG * F::kBlocks; ++b)
            tmem_cp_32x128b_warpx4(tmem + kSfaCol + 4 * b,
                                   smem_desc_noswz(smem_addr(sSfa(s) + b * kSfBlock), 128));
#pragma unroll
          for (int b = 0; b < 2 * F::kBlocks; ++b)
            tmem_cp_32x128b_warpx4(tmem + kSfbCol + 4 * b,
                                   smem_desc_noswz(smem_addr(sSfb(s) + b * kSfBlock), 128));
          const uint64_t adesc = smem_desc_sw128(smem_addr(sA(s)));
          const uint64_t bdesc = smem_desc_sw128(smem_addr(sB(s)));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // K=64 step kk: 32 bytes into the 128-byte swizzled rows.  MX:
            // its scales are 2kk, 2kk+1 (block kk/2, byte 2(kk%2)); NV: its
            // scales are 4kk..4kk+3 (block kk, the whole word)
            const uint32_t id = kNV ? 0u : 2u * (kk & 1);
            const uint32_t blk = kNV ? kk : kk >> 1;
            const uint32_t sfb = (tmem + kSfbCol + 8 * blk) | (id << 30);
            const uint32_t idesc = idesc_mxf4(kM, n, id, id, !kNV);
#pragma unroll
            for (int g = 0; g < kMG; ++g) {
              // weight group g: rows 128g .. +128 of the A tile, accumulator g
              const uint32_t sfa = (tmem + kSfaCol + 4 * (g * F::kBlocks + blk)) | (id << 30);
              const uint64_t ad = adesc + ((uint64_t)(g * kM * kKB) >> 4) + 2 * kk;
              const uint32_t d = tmem + (uint32_t)(g * kTileN);
              if constexpr (kNV)
                mma_nvf4_ss(d, ad, bdesc + 2 * kk, idesc, sfa, sfb, (ks | kk) != 0);
              else
                mma_mxf4_ss(d, ad, bdesc + 2 * kk, idesc, sfa, sfb, (ks | kk) != 0);
            }
          }
          mma_commit(&sh->empty[s]);
        }
        if (ok) mma_commit(&sh->d_full);
      }
      mma_commit(&sh->drain);
      int abort_local = 0;
      mbar_wait(&sh->drain, 0, &abort_local, kDrainLimitNs);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue
    TileWalker walk(t_offs, E, kTileN, col_tiles);
    uint32_t lt = 0;
    for (int64_t tile = blockIdx.x; walk.seek(tile); tile += gridDim.x, ++lt) {
      if (epi_any(*abort != 0)) break;
      const bool ok = mbar_wait(&sh->d_full, lt & 1, abort, wait_limit_ns);
      if (epi_any(!ok)) break;
      tc_fence_after();
      const int64_t row0 = walk.row0;
      const int64_t rows = walk.row_end - row0 < kTileN ? walk.row_end - row0 : kTileN;
      const int col = 32 * warp + lane;  // output feature within a weight group's 128
      // NV: the product of the two per-tensor scales, applied in f32
      const float gg = kNV ? __fmul_rn(x_global[0], w_global[walk.expert]) : 1.0f;
      constexpr int kYRows = F::kYRows;
      const int nc = (int)((rows + 31) / 32);  // 32-token chunks of D
      if (rows <= 0 && lane == 0) mbar_arrive(&sh->d_empty);
      // accumulator g (weight rows 128g .. of the tile), tokens p0 .. p0 +
      // kYRows - 1 per pass: staged, then stored
      bool first = true;
      for (int g = 0; g < kMG; ++g) {
        __nv_bfloat16* yt = y + row0 * N + walk.col_tile * F::kTileM + g * kM;
        for (int p0 = 0; p0 < rows; p0 += kYRows) {
          if (!first) epi_bar();  // the previous pass's rows are stored
          first = false;
          const int c_end = nc < (p0 + kYRows) / 32 ? nc : (p0 + kYRows) / 32;
#pragma unroll 1
          for (int c = p0 / 32; c < c_end; ++c) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * warp) << 16) + g * kTileN + 32 * c, v);
            tmem_wait_ld();
            if constexpr (kNV) {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * gg);
            }
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const uint32_t pr = pack2<kBF16>(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
              const int t = 32 * c + j - p0;  // token within the pass
              if (MXQ_IN_RANGE(kChkW4Smem, (t + 1) * kM + col, kYRows * kM)) {
                sY[t * kM + col] = (uint16_t)(pr & 0xFFFFu);
                sY[(t + 1) * kM + col] = (uint16_t)(pr >> 16);
              }
            }
          }
          if (g == kMG - 1 && p0 + kYRows >= rows) {  // every chunk of D is read
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh->d_empty);
          }
          epi_bar();  // the pass is staged
          const int r_end = rows < p0 + kYRows ? (int)rows : p0 + kYRows;
          for (int r = p0 + 2 * warp + (lane >> 4); r < r_end; r += 2 * kEpiWarps) {
            const uint4 val = *reinterpret_cast<const uint4*>(sY + (r - p0) * kM + 8 * (lane & 15));
            if (MXQ_IN_RANGE(kChkW4Out,
                             (row0 + r) * N + walk.col_tile * F::kTileM + g * kM + 8 * (lane & 15) + 7,
                             T * N))
              *reinterpret_cast<uint4*>(yt + (int64_t)r * N + 8 * (lane & 15)) = val;
          }
        }
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

template <bool kNV, bool kBig>
int launch_w4a4_shape(const void* xq, const void* xs, const float* xg, const void* packed,
                      const void* scales, const float* wg, const int32_t* offs, int64_t T,
                      int64_t E, int64_t N, int64_t K, void* y, int32_t* dev_status,
                      uint64_t wait_limit_ns, cudaStream_t st) {
  using F = W4Fmt<kNV, kBig>;
  CUtensorMap xmap, wmap;
  if (!make_tmap_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, T, K / 2, K / 2, kKB, F::kTileN,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, E * N, K / 2, K / 2, kKB,
                    F::kTileM, CU_TENSOR_MAP_SWIZZLE_128B))
    return MXQ_ERR_CUDA;
  // Scale loads of 32 bytes per row (several stages) when every row's
  // scales start on a 16-byte boundary and the stages split into whole
  // groups; 8 or 16 bytes per stage otherwise.
  const int64_t srow = K / (kNV ? 16 : 32);
  const int64_t group = kNV ? 2 : 4;
  const bool wide = srow % 16 == 0 && (K / 256) % group == 0;
  auto kernel = wide ? w4a4_tc_kernel<kNV, true, kBig> : w4a4_tc_kernel<kNV, false, kBig>;
  if (allow_dynamic_smem((const void*)kernel, (int)F::kSmem) != cudaSuccess) return MXQ_ERR_CUDA;
  const int64_t tiles = ((T + F::kTileN - 1) / F::kTileN + E) * (N / F::kTileM);
  const int64_t sms = num_sms();
  const int grid = (int)(tiles < sms ? tiles : sms);
  // Programmatic stream serialization: the CTAs may start their set-up while
  // the previous kernel on the stream (typically the activation quantizer)
  // finishes; they wait for its results before reading any input.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = F::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t err =
      cudaLaunchKernelEx(&cfg, kernel, xmap, wmap, (const uint8_t*)xs, (const uint8_t*)scales, xg,
                         wg, offs, T, E, N, K, (__nv_bfloat16*)y, dev_status, wait_limit_ns);
  return err == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

// The 256 x 224 tile where N allows it, the 128 x 256 one otherwise.
template <bool kNV>
int launch_w4a4(const void* xq, const void* xs, const float* xg, const void* packed,
                const void* scales, const float* wg, const int32_t* offs, int64_t T, int64_t E,
                int64_t N, int64_t K, void* y, int32_t* dev_status, uint64_t wait_limit_ns,
                cudaStream_t st) {
  if (N % 256 == 0)
    return launch_w4a4_shape<kNV, true>(xq, xs, xg, packed, scales, wg, offs, T, E, N, K, y,
                                        dev_status, wait_limit_ns, st);
  return launch_w4a4_shape<kNV, false>(xq, xs, xg, packed, scales, wg, offs, T, E, N, K, y,
                                       dev_status, wait_limit_ns, st);
}

}  // namespace

int launch_w4a4_grouped_mm(const void* xq, const void* xs, const void* packed, const void* scales,
                           const int32_t* offs, int64_t T, int64_t E, int64_t N, int64_t K,
                           void* y, int32_t* dev_status, uint64_t wait_limit_ns, cudaStream_t st) {
  return launch_w4a4<false>(xq, xs, nullptr, packed, scales, nullptr, offs, T, E, N, K, y,
                            dev_status, wait_limit_ns, st);
}

int launch_nvfp4_w4a4_grouped_mm(const void* xq, const void* xs, const float* xg,
                                 const void* packed, const void* scales, const float* wg,
                                 const int32_t* offs, int64_t T, int64_t E, int64_t N, int64_t K,
                                 void* y, int32_t* dev_status, uint64_t wait_limit_ns,
                                 cudaStream_t st) {
  return launch_w4a4<true>(xq, xs, xg, packed, scales, wg, offs, T, E, N, K, y, dev_status,
                           wait_limit_ns, st);
}

MXQ_DEFINE_CHECK_READER(check_record_w4a4)

}  // namespace mxq
