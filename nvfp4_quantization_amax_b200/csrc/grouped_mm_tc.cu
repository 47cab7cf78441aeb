// Tensor-core grouped GEMM over MXFP4-packed expert weights (sm_100a).
//
// Semantics ("nemo_automodel.components.quantization.mxfp4",
// MXFP4GroupedMM): expert e owns activation rows [offs[e-1], offs[e]);
//   forward  (transpose_w = 0): y[t, n] = sum_k x[t, k]  W_e[n, k]
//   backward (transpose_w = 1): y[t, k] = sum_n g[t, n]  W_e[n, k]
// with W_e[n, k] = E2M1(nibble) * 2^(scale - 127) decoded on the fly from
// the packed [E, N, K/2] bytes and [E, N, K/32] E8M0 scales.
//
// Mapping onto tcgen05 (persistent kernel, one CTA per SM):
//   D[m, j] (f32, TMEM)  +=  A[m, r] (bf16, TMEM)  *  B[j, r] (bf16, smem)
// with m an output feature (a weight row n in the forward, a column k in
// the backward), j a token of the expert and r the reduction index (64 per
// pipeline stage).  A tile is 128 output features per CTA by up to 256
// tokens; in the CTA-pair form two SMs of a cluster share one tile of 256
// output features (tcgen05.mma.cta_group::2), each holding its 128 features
// in TMEM and half of the tokens in shared memory, so each SM streams half
// as many activation bytes per MMA.
//   * B (activations) arrives by TMA, 128-byte swizzled, K-major.
//   * A (weights) never exists in bf16 outside the SM: dequantization warps
//     read the packed bytes from global memory, decode them exactly to bf16
//     in registers and write them straight into TMEM with tcgen05.st.  In
//     the backward the 8x8 blocks are transposed in registers with
//     movmatrix first, since TMEM lanes must be the output features k.
//   * One thread issues tcgen05.mma (K=16 steps; N = the tile's token count
//     rounded up, so ragged expert tails cost no idle columns) and releases
//     stages with tcgen05.commit.
//   * Four epilogue warps drain D (tcgen05.ld), round to bf16, stage the
//     tile in shared memory and store the rows that belong to the expert.
// Every mbarrier wait is bounded: on a time-out the CTA stops all roles,
// drains what it issued, frees TMEM and reports MXQ_ERR_TIMEOUT.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>

#include "mxq.h"
#include "mxq_device.cuh"
#include "mxq_grouped.cuh"
#include "mxq_launch.h"
#include "sm100_primitives.cuh"
#include "tmap.h"

namespace mxq {

int launch_grouped_mm_general(const void* a, const void* packed, const void* scales,
                              const int32_t* offs, int64_t T, int64_t E, int64_t N, int64_t K,
                              int transpose_w, void* y, int32_t* dev_status, cudaStream_t st);

namespace {

using namespace sm100;

constexpr int kBM = 128;        // output features per CTA (TMEM lanes)
constexpr int kBN = 256;        // tokens per tile (MMA N)
constexpr int kBox = 64;        // reduction elements per TMA box (128 bytes of bf16)
constexpr int kTmemCols = 512;
constexpr int kDCol = 0;        // accumulator: columns [0, 256)
constexpr int kACol = 256;      // A stages follow the accumulator
constexpr int kMaxStages = 4;
constexpr int kEpiWarps = 4;    // warps 0..3
constexpr int kDqWarps = 8;     // warps 4..11
constexpr int kTmaWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kThreads = 14 * 32;
constexpr uint32_t kStagingBytes = kBN * kBM * 2;   // 64 KB
constexpr int kMaxSmemExperts = 4096;               // offs cached in smem up to this E
constexpr int kMaxSmemExpertsW = 256;               // (when smem also holds weight slots)
constexpr int kWStages = 3;                         // packed-weight slots staged by TMA
constexpr uint64_t kDrainLimitNs = 1000000000ull;

template <bool kPair>
struct Geo {
  static constexpr int kCG = kPair ? 2 : 1;
  static constexpr int kTileM = kBM * kCG;            // output features per tile
  static constexpr int kRowsB = kBN / kCG;            // token rows per CTA per stage
  // Reduction depth of a stage: 128 in pairs (fewer, larger hand-offs
  // between the dequantization warps and the MMA), 64 alone.
  static constexpr int kBK = kPair ? 128 : 64;
  static constexpr int kBoxes = kBK / kBox;           // TMA boxes per stage
  static constexpr uint32_t kBoxBytes = kRowsB * kBox * 2;
  static constexpr uint32_t kStageBytes = kBoxes * kBoxBytes;
  static constexpr int kACols = kBK / 2;              // TMEM columns per A stage
  // One B stage per A stage; 4 x 32 KB of activations per CTA either way,
  // and 4 A stages of at most 64 columns beside the 256 accumulator columns.
  static constexpr int kStages = 4;
  static constexpr uint32_t kSmem =
      1024 + kStages * kStageBytes + kStagingBytes + 256 + 4 * kMaxSmemExperts;
  // With weight staging, the packed weight tile of a stage (64 bytes by
  // 128 rows: the input gradient's kBK rows n x 128 features k, or the
  // pair forward's 128 rows n x 128 k, 64-byte swizzled) and its scale
  // bytes (a 16-byte box per row) arrive by TMA into kWStages slots.
  static constexpr int kWRows = 128;
  static constexpr uint32_t kWBytes = kWRows * 64;
  static constexpr uint32_t kSBytes = kWRows * 16;
  static constexpr uint32_t kSmemW = 1024 + kStages * kStageBytes +
                                     kWStages * (kWBytes + kSBytes) + kStagingBytes + 256 +
                                     4 * kMaxSmemExpertsW;
  // Token count of a tile rounded to what the MMA accepts.
  __host__ __device__ static int64_t mma_n(int64_t rows) {
    return kPair ? (rows + 31) & ~31 : (rows + 15) & ~15;
  }
};

struct Shared {
  uint64_t full_a[kMaxStages];
  uint64_t full_b[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t wfull[kWStages];   // packed weights (+ scales) of a stage landed
  uint64_t wempty[kWStages];  // the dequantization warps are done with a slot
  uint64_t d_full, d_empty, drain;
  uint32_t tmem_base;
  uint32_t peer_issued;  // activation stages the odd CTA of a pair loaded (written into the even CTA)
  int abort;
};

__device__ __forceinline__ float scale_f32(uint32_t s) { return mx_block_scale(s); }
__device__ __forceinline__ uint32_t dequant_pair(uint32_t byte, float scale) {
  return mx_dequant_pair(byte, scale);
}

__device__ __forceinline__ uint4 ldg16(const uint8_t* p) {
  return *reinterpret_cast<const uint4*>(p);
}

// Input gradient: the feature held by TMEM lane L of a warp's 32.  Lane
// L = 8c + r carries row r of the transposed 8x8 block c, whose rows are
// the features k = 8(r >> 1) + 2c + (r & 1) (see the dequantization warps).
__device__ __forceinline__ int kperm(int L) {
  return ((L & 6) << 2) | ((L >> 3) << 1) | (L & 1);
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

// Bounded wait (the same form whether or not the peer CTA arrives too).
template <bool kPair>
__device__ __forceinline__ bool bwait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                      uint64_t limit_ns) {
  return mbar_wait(bar, parity, abort, limit_ns);
}

// Same outcome on every lane of the warp (the tcgen05 ld/st that follow
// are warp-collective).
template <bool kPair>
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit_ns) {
  const bool ok = bwait<kPair>(bar, parity, abort, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// Arrive on the even CTA's copy of a barrier (a local arrive when unpaired).
template <bool kPair>
__device__ __forceinline__ void arrive_leader(uint64_t* bar) {
  if constexpr (kPair) mbar_arrive_cluster(mapa_shared(smem_addr(bar), 0));
  else mbar_arrive(bar);
}

template <bool kDgrad, bool kPair>
__global__ void __launch_bounds__(kThreads, 1)
grouped_mm_tc_kernel(const __grid_constant__ CUtensorMap tmap_act,
                     const __grid_constant__ CUtensorMap tmap_w,
                     const __grid_constant__ CUtensorMap tmap_s, const uint8_t* __restrict__ packed,
                     const uint8_t* __restrict__ scales, const int32_t* __restrict__ offs, int64_t T,
                     int64_t E, int64_t N, int64_t K, __nv_bfloat16* __restrict__ y,
                     int32_t* dev_status, uint64_t wait_limit_ns, int scales_by_tma) {
  using G = Geo<kPair>;
  constexpr int S = G::kStages;
  // Weight staging by TMA: the input gradient always, the forward in pairs.
  constexpr bool kWTma = kDgrad || kPair;
  constexpr int kWS = kWTma ? kWStages : 0;
  constexpr int kWBoxRows = kDgrad ? G::kBK : kBM;  // rows of a weight / scale box
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sB = smem;
  uint8_t* sW = smem + S * G::kStageBytes;        // weight slots (kWTma only)
  uint8_t* sS = sW + kWS * G::kWBytes;
  uint16_t* sY = (uint16_t*)(sS + kWS * G::kSBytes);
  Shared* sh = (Shared*)((uint8_t*)sY + kStagingBytes);
  int32_t* s_offs = (int32_t*)((uint8_t*)sh + 256);
  constexpr int kOffsCache = kWTma ? kMaxSmemExpertsW : kMaxSmemExperts;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = kPair ? cluster_ctarank() : 0;  // 0 leads the pair
  const int64_t unit = kPair ? (int64_t)(blockIdx.x >> 1) : (int64_t)blockIdx.x;
  const int64_t units = kPair ? (int64_t)(gridDim.x >> 1) : (int64_t)gridDim.x;

  // Both CTAs of a pair read the same offs, so both leave here together.
  if (!offs_valid(offs, E, T)) {
    if (blockIdx.x == 0 && threadIdx.x == 0 && dev_status) *dev_status = MXQ_ERR_BAD_OFFS;
    return;
  }
  // Tile walks read the expert partition from shared memory when it fits.
  const int32_t* t_offs = offs;
  if (E <= kOffsCache) {
    for (int64_t e = threadIdx.x; e < E; e += blockDim.x) s_offs[e] = offs[e];
    t_offs = s_offs;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      // with weight staging each stage is decoded by the 4 warps of one
      // stage-parity group, otherwise by all 8 (two halves of the stage)
      mbar_init(&sh->full_a[s], (kWTma ? kDqWarps / 2 : kDqWarps) * G::kCG);
      mbar_init(&sh->full_b[s], 1);
      mbar_init(&sh->empty[s], 1);
    }
    for (int s = 0; s < kWS; ++s) {
      mbar_init(&sh->wfull[s], 1);
      mbar_init(&sh->wempty[s], kDqWarps / 2);
    }
    mbar_init(&sh->d_full, 1);
    mbar_init(&sh->d_empty, kEpiWarps * G::kCG);
    mbar_init(&sh->drain, 1);
    sh->peer_issued = 0;
    sh->abort = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_cg<G::kCG>(&sh->tmem_base, kTmemCols);
    tmem_relinquish_cg<G::kCG>();
  }
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tmap(&tmap_act);
    if constexpr (kWTma) {
      prefetch_tmap(&tmap_w);
      if (scales_by_tma) prefetch_tmap(&tmap_s);
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync();  // the peer's barriers exist before any remote arrive
  tc_fence_after();

  const uint32_t tmem = sh->tmem_base;
  volatile int* abort = &sh->abort;
  const int64_t kin = kDgrad ? N : K;
  const int64_t nout = kDgrad ? K : N;
  constexpr int kBK = G::kBK;
  const int nk = (int)(kin / kBK);
  const int64_t col_tiles = nout / G::kTileM;
  uint32_t b_issued = 0;  // activation stages this CTA loaded (TMA lane 0)

  if (warp == kTmaWarp) {
    // ------------------------------------------------ TMA producer (B)
    if (lane == 0) {
      TileWalker walk(t_offs, E, kBN, col_tiles);
      uint32_t it = 0;
      for (int64_t tile = unit; !*abort && walk.seek(tile); tile += units) {
        const int64_t rows = walk.row_end - walk.row0 < kBN ? walk.row_end - walk.row0 : kBN;
        // this CTA's share of the tile's tokens
        const int32_t yrow = (int32_t)(walk.row0 + rank * (G::mma_n(rows) / 2));
        for (int ks = 0; ks < nk; ++ks, ++it) {
          const int s = it % S;
          if (!bwait<kPair>(&sh->empty[s], ((it / S) & 1) ^ 1, abort, wait_limit_ns)) break;
          if constexpr (kPair) {
            if (rank == 0) mbar_arrive_expect_tx(&sh->full_b[s], 2 * G::kStageBytes);
            const uint32_t bar = mapa_shared(smem_addr(&sh->full_b[s]), 0);
#pragma unroll
            for (int b = 0; b < G::kBoxes; ++b)
              tma_load_2d_pair(smem_addr(sB + s * G::kStageBytes + b * G::kBoxBytes), &tmap_act,
                               ks * kBK + b * kBox, yrow, bar);
          } else {
            mbar_arrive_expect_tx(&sh->full_b[s], G::kStageBytes);
#pragma unroll
            for (int b = 0; b < G::kBoxes; ++b)
              tma_load_2d(smem_addr(sB + s * G::kStageBytes + b * G::kBoxBytes), &tmap_act,
                          ks * kBK + b * kBox, yrow, &sh->full_b[s]);
          }
        }
      }
      b_issued = it;
      // Loads still in flight land before the CTA may exit.  (In pairs both
      // CTAs' loads count on the even CTA's barriers: see the teardown.)
      if constexpr (!kPair) {
        int abort_local = 0;
        for (uint32_t j = it > (uint32_t)S ? it - S : 0; j < it; ++j)
          bwait<kPair>(&sh->full_b[j % S], (j / S) & 1, &abort_local, kDrainLimitNs);
      }
    }
    if constexpr (kWTma) {
      if (lane == 1) {
        // -------------------------------------------- weight producer
        // Input gradient, stage ks of a tile: packed rows n = ks*kBK ..
        // +kBK of expert e, bytes m0/2 .. +64 (this CTA's 128 features k).
        // Forward: rows n = m0 .. +128 (this CTA's features), bytes
        // ks*kBK/2 .. +64.  Scale bytes: the 16-byte box holding the 4 the
        // stage needs, on the same rows.
        const uint32_t tx = kWBoxRows * 64 + (scales_by_tma ? kWBoxRows * 16 : 0);
        TileWalker walk(t_offs, E, kBN, col_tiles);
        uint32_t wit = 0;
        for (int64_t tile = unit; !*abort && walk.seek(tile); tile += units) {
          const int64_t m0 = walk.col_tile * G::kTileM + rank * kBM;
          const int32_t wy = (int32_t)(walk.expert * N);
          bool ok = true;
          for (int ks = 0; ks < nk; ++ks, ++wit) {
            const int ws = wit % kWS;
            if (!(ok = bwait<kPair>(&sh->wempty[ws], ((wit / kWS) & 1) ^ 1, abort, wait_limit_ns)))
              break;
            int32_t wx, sx, y0;
            if constexpr (kDgrad) {
              wx = (int32_t)(m0 / 2);
              sx = (int32_t)((m0 / 32) & ~(int64_t)15);
              y0 = wy + ks * kBK;
            } else {
              wx = ks * (kBK / 2);
              sx = (ks * (kBK / 32)) & ~15;
              y0 = wy + (int32_t)m0;
            }
            mbar_arrive_expect_tx(&sh->wfull[ws], tx);
            tma_load_2d(smem_addr(sW + ws * G::kWBytes), &tmap_w, wx, y0, &sh->wfull[ws]);
            if (scales_by_tma)
              tma_load_2d(smem_addr(sS + ws * G::kSBytes), &tmap_s, sx, y0, &sh->wfull[ws]);
          }
          if (!ok) break;
        }
        int abort_local = 0;
        for (uint32_t j = wit > (uint32_t)kWS ? wit - kWS : 0; j < wit; ++j)
          bwait<kPair>(&sh->wfull[j % kWS], (j / kWS) & 1, &abort_local, kDrainLimitNs);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0 && rank == 0) {
      TileWalker walk(t_offs, E, kBN, col_tiles);
      uint32_t it = 0, lt = 0;
      bool ok = true;
      for (int64_t tile = unit; ok && walk.seek(tile); tile += units, ++lt) {
        if (!(ok = bwait<kPair>(&sh->d_empty, (lt & 1) ^ 1, abort, wait_limit_ns))) break;
        tc_fence_after();
        const int64_t rows = walk.row_end - walk.row0 < kBN ? walk.row_end - walk.row0 : kBN;
        const uint32_t idesc = idesc_bf16_f32(G::kTileM, (int)G::mma_n(rows));
        for (int ks = 0; ks < nk; ++ks, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!(ok = bwait<kPair>(&sh->full_a[s], ph, abort, wait_limit_ns))) break;
          if (!(ok = bwait<kPair>(&sh->full_b[s], ph, abort, wait_limit_ns))) break;
          tc_fence_after();
          const uint64_t bdesc = smem_desc_sw128(smem_addr(sB + s * G::kStageBytes));
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            // K16 step kk: box kk/4, 32-byte column offset kk%4 inside it
            const uint64_t bd = bdesc + (uint64_t)(((kk >> 2) * G::kBoxBytes) >> 4) + 2 * (kk & 3);
            const uint32_t a = tmem + kACol + G::kACols * s + 8 * kk;
            if constexpr (kPair)
              mma_bf16_ts_pair(tmem + kDCol, a, bd, idesc, (ks | kk) != 0);
            else
              mma_bf16_ts(tmem + kDCol, a, bd, idesc, (ks | kk) != 0);
          }
          if constexpr (kPair) mma_commit_pair(&sh->empty[s]);
          else mma_commit(&sh->empty[s]);
        }
        if (ok) {
          if constexpr (kPair) mma_commit_pair(&sh->d_full);
          else mma_commit(&sh->d_full);
        }
      }
      // Every MMA issued has completed before TMEM is released.
      if constexpr (kPair) mma_commit_pair(&sh->drain);
      else mma_commit(&sh->drain);
      int abort_local = 0;
      mbar_wait(&sh->drain, 0, &abort_local, kDrainLimitNs);
    } else if (kPair && lane == 0) {
      // the leader's last commit (multicast) also lands here before this
      // CTA may exit
      int abort_local = 0;
      mbar_wait(&sh->drain, 0, &abort_local, kDrainLimitNs);
    }
    __syncwarp();
  } else if (warp >= kEpiWarps) {
    // -------------------------------------------- dequantization (A)
    const int q = warp & 3;                  // TMEM lane quarter
    // which half of a stage (no weight staging), or which stage parity
    // (weight staging: warps h = 0 decode even stages, h = 1 odd ones)
    const int h = (warp - kEpiWarps) >> 2;
    uint32_t it_base = 0;  // stages of the tiles before this one
    TileWalker walk(t_offs, E, kBN, col_tiles);
    uint32_t it = 0;  // stage counter of the unstaged forward
    bool ok = true;
    for (int64_t tile = unit; ok && walk.seek(tile); tile += units) {
      const int64_t e = walk.expert;
      const int64_t m0 = walk.col_tile * G::kTileM + rank * kBM;  // this CTA's features
      if constexpr (!kDgrad && kWTma) {
        // Thread = weight row n = m0 + 32q + lane (slot row 32q + lane);
        // the warp decodes every other stage (parity h): k = ks*kBK ..
        // +128, the four 16-byte chunks of the 64-byte slot row (64-byte
        // swizzle) and scale bytes 4ks .. 4ks+3 of the row's 16-byte scale
        // box, in two halves of 64 k.  The other parity group's decode
        // overlaps this group's TMEM-store wait.
        static_assert(kBK == 128, "weight staging of the forward assumes 128-deep stages");
        const int row = 32 * q + lane;
        const int swz = (row >> 1) & 3;
        const uint8_t* srow = scales + (e * N + m0 + row) * (K / 32);
        for (int ks = h; ks < nk && ok; ks += 2) {
          const uint32_t wi = it_base + ks;  // stage index (weight slots and A slots)
          const int ws = wi % kWS;
          if (!(ok = warp_wait<kPair>(&sh->wfull[ws], (wi / kWS) & 1, abort, wait_limit_ns)))
            break;
          const uint8_t* wrow = sW + ws * G::kWBytes + row * 64;
          uint4 d[4];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            d[c] = *reinterpret_cast<const uint4*>(wrow + 16 * (c ^ swz));
          uint32_t sb4;
          if (scales_by_tma)
            sb4 = *reinterpret_cast<const uint32_t*>(sS + ws * G::kSBytes + row * 16 + ((4 * ks) & 15));
          else if (MXQ_IN_RANGE(kChkGemmTcScale, (e * N + m0 + row) * (K / 32) + 4 * ks + 3,
                                E * N * (K / 32)))
            sb4 = *reinterpret_cast<const uint32_t*>(srow + 4 * ks);
          else
            sb4 = 0u;
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh->wempty[ws]);
          const int s = wi % S;
          bool waited = false;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t v[32];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const uint4 dd = d[2 * hh + c];
              const uint32_t w[4] = {dd.x, dd.y, dd.z, dd.w};
              const uint32_t sbyte = (sb4 >> (8 * (2 * hh + c))) & 0xFFu;
              const float sc = scale_f32(sbyte);
#pragma unroll
              for (int i = 0; i < 16; ++i)
                v[16 * c + i] = dequant_pair((w[i >> 2] >> (8 * (i & 3))) & 0xFFu, sc);
            }
            if (!waited) {
              if (!(ok = warp_wait<kPair>(&sh->empty[s], ((wi / S) & 1) ^ 1, abort, wait_limit_ns)))
                break;
              tc_fence_after();
              waited = true;
            }
            const uint32_t col = kACol + G::kACols * s + 32 * hh;
#pragma unroll
            for (int c = 0; c < 2; ++c)
              tmem_st_32x32b_x16(tmem + ((uint32_t)(32 * q) << 16) + col + 16 * c, v + 16 * c);
          }
          if (!ok) break;
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) arrive_leader<kPair>(&sh->full_a[s]);
        }
        it_base += nk;
      } else if constexpr (!kDgrad) {
        // Thread = weight row n; kBK/2 consecutive k (kBK/4 bytes, one or
        // two 16-byte loads, one scale per 32 k) per stage half.
        constexpr int kV = kBK / 64;  // 16-byte loads per thread per stage
        const int64_t n = m0 + 32 * q + lane;
        const uint8_t* prow = packed + (e * N + n) * (K / 2) + (kBK / 4) * h;
        const uint8_t* srow = scales + (e * N + n) * (K / 32) + kV * h;
        uint4 pb[4][kV];
        uint32_t sb[4][kV];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (j < nk) {
#pragma unroll
            for (int c = 0; c < kV; ++c) {
              const bool in = MXQ_IN_RANGE(
                  kChkGemmTcW, (e * N + n) * (K / 2) + (kBK / 4) * h + (kBK / 2) * j + 16 * c + 15,
                  E * N * (K / 2));
              pb[j][c] = in ? ldg16(prow + (kBK / 2) * j + 16 * c) : make_uint4(0u, 0u, 0u, 0u);
              sb[j][c] = in ? srow[(kBK / 32) * j + c] : 0u;
            }
          }
        for (int ks0 = 0; ks0 < nk && ok; ks0 += 4) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int ks = ks0 + j;
            if (ks >= nk || !ok) break;
            uint4 d[kV];
            float sc[kV];
#pragma unroll
            for (int c = 0; c < kV; ++c) {
              d[c] = pb[j][c];
              sc[c] = scale_f32(sb[j][c]);
            }
            if (ks + 4 < nk) {
#pragma unroll
              for (int c = 0; c < kV; ++c) {
                pb[j][c] = ldg16(prow + (kBK / 2) * (ks + 4) + 16 * c);
                sb[j][c] = srow[(kBK / 32) * (ks + 4) + c];
              }
            }
            uint32_t v[16 * kV];
#pragma unroll
            for (int c = 0; c < kV; ++c) {
              const uint32_t w[4] = {d[c].x, d[c].y, d[c].z, d[c].w};
#pragma unroll
              for (int i = 0; i < 16; ++i)
                v[16 * c + i] = dequant_pair((w[i >> 2] >> (8 * (i & 3))) & 0xFFu, sc[c]);
            }
            const int s = it % S;
            if (!(ok = warp_wait<kPair>(&sh->empty[s], ((it / S) & 1) ^ 1, abort, wait_limit_ns)))
              break;
            tc_fence_after();
            const uint32_t col = kACol + G::kACols * s + 16 * kV * h;
#pragma unroll
            for (int c = 0; c < kV; ++c)
              tmem_st_32x32b_x16(tmem + ((uint32_t)(32 * q) << 16) + col + 16 * c, v + 16 * c);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_leader<kPair>(&sh->full_a[s]);
            ++it;
          }
        }
      } else {
        // The warp's 32 output features k = m0 + 32q + (0..31) are TMEM
        // lanes 32q..32q+31, in the order kperm() gives; the warp decodes
        // every other stage (parity h), all kBK reduction indices n of it,
        // in sub-steps of 32.  In a
        // sub-step thread t reads 4 contiguous bytes (word t%4 of the
        // warp's 16 bytes) of rows n = base + 8j + t/4, j = 0..3, from the
        // TMA-staged tile.  Byte c of the word (k = 8(t%4) + 2c, +1) goes
        // to 8x8 block c; movmatrix transposes each block so that a thread
        // holds bf16 pairs along n, and block c fills TMEM lanes 8c..8c+7.
        const int rsub = lane >> 2, csub = lane & 3;
        const uint8_t* scol = scales + e * N * (K / 32) + (m0 + 32 * q) / 32;
        const int soff = (int)((m0 / 32) & 15) + q;  // this warp's byte in a scale box row
        constexpr int kSubAll = kBK / 32;  // sub-steps of 32 rows n per stage
        for (int ks = h; ks < nk && ok; ks += 2) {
          const uint32_t wi = it_base + ks;
          const int ws = wi % kWS;
          if (!(ok = warp_wait<kPair>(&sh->wfull[ws], (wi / kWS) & 1, abort, wait_limit_ns)))
            break;
          // this thread's word of row rsub; rows 8j further on share its
          // 64-byte swizzle phase ((row >> 1) & 3 = (rsub >> 1) & 3)
          const uint8_t* wst = sW + ws * G::kWBytes + rsub * 64 + 16 * (q ^ ((rsub >> 1) & 3)) + 4 * csub;
          const uint8_t* sst = sS + ws * G::kSBytes + rsub * 16 + soff;
          uint32_t wd[kSubAll][4];
          float sc[kSubAll][4];
#pragma unroll
          for (int sub_i = 0; sub_i < kSubAll; ++sub_i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int row = 32 * sub_i + 8 * j + rsub;  // n within the stage
              wd[sub_i][j] = *reinterpret_cast<const uint32_t*>(wst + (32 * sub_i + 8 * j) * 64);
              [[maybe_unused]] const int64_t gi = e * N * (K / 32) + (m0 + 32 * q) / 32 +
                                 ((int64_t)ks * kBK + row) * (K / 32);
              const uint32_t sb =
                  scales_by_tma
                      ? (uint32_t)sst[(32 * sub_i + 8 * j) * 16]
                      : (MXQ_IN_RANGE(kChkGemmTcScale, gi, E * N * (K / 32))
                             ? (uint32_t)scol[((int64_t)ks * kBK + row) * (K / 32)]
                             : 0u);
              sc[sub_i][j] = scale_f32(sb);
            }
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh->wempty[ws]);
          const int s = wi % S;
#pragma unroll
          for (int sub_i = 0; sub_i < kSubAll; ++sub_i) {
            uint32_t v[2][8];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
              for (int c = 0; c < 4; ++c)
                v[c >> 1][2 * j + (c & 1)] =
                    movmatrix_trans(dequant_pair((wd[sub_i][j] >> (8 * c)) & 0xFFu, sc[sub_i][j]));
            if (sub_i == 0) {
              if (!(ok = warp_wait<kPair>(&sh->empty[s], ((wi / S) & 1) ^ 1, abort, wait_limit_ns)))
                break;
              tc_fence_after();
            }
            const uint32_t col = kACol + G::kACols * s + 16 * sub_i;
#pragma unroll
            for (int r = 0; r < 2; ++r)
              tmem_st_16x128b_x4(tmem + ((uint32_t)(32 * q + 16 * r) << 16) + col, v[r]);
          }
          if (!ok) break;
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) arrive_leader<kPair>(&sh->full_a[s]);
        }
        it_base += nk;
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    TileWalker walk(t_offs, E, kBN, col_tiles);
    uint32_t lt = 0;
    for (int64_t tile = unit; walk.seek(tile); tile += units, ++lt) {
      // (also orders the previous tile's staging reads before new writes)
      if (epi_any(*abort != 0)) break;
      const bool ok = bwait<kPair>(&sh->d_full, lt & 1, abort, wait_limit_ns);
      if (epi_any(!ok)) break;
      tc_fence_after();
      const int64_t row0 = walk.row0;
      const int64_t rows = walk.row_end - row0 < kBN ? walk.row_end - row0 : kBN;
      // output feature within this CTA's 128 (TMEM lane 32 warp + lane)
      const int col = 32 * warp + (kDgrad ? kperm(lane) : lane);
#pragma unroll 1
      for (int c = 0; c < (int)((rows + 31) / 32); ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * warp) << 16) + kDCol + 32 * c, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const uint32_t pr = pack2<kBF16>(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
          if (MXQ_IN_RANGE(kChkGemmTcSmem, (32 * c + j + 1) * kBM + col, kBN * kBM)) {
            sY[(32 * c + j) * kBM + col] = (uint16_t)(pr & 0xFFFFu);
            sY[(32 * c + j + 1) * kBM + col] = (uint16_t)(pr >> 16);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_leader<kPair>(&sh->d_empty);
      epi_bar();  // the whole tile is staged
      __nv_bfloat16* yt = y + row0 * nout + walk.col_tile * G::kTileM + rank * kBM;
      // two rows of 128 outputs (256 bytes each) per warp instruction
      for (int r = 2 * warp + (lane >> 4); r < rows; r += 2 * kEpiWarps) {
        const uint4 val = *reinterpret_cast<const uint4*>(sY + r * kBM + 8 * (lane & 15));
        const int64_t col0 = walk.col_tile * G::kTileM + rank * kBM + 8 * (lane & 15);
        if (MXQ_IN_RANGE(kChkGemmTcOut, (row0 + r) * nout + col0 + 7, T * nout))
          *reinterpret_cast<uint4*>(yt + (int64_t)r * nout + 8 * (lane & 15)) = val;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) {
    // After an abort the two CTAs may have loaded different numbers of
    // activation stages, and the odd CTA's loads count on the even CTA's
    // barriers.  The odd CTA reports its count; the even CTA settles the
    // stages only one of them loaded (completing the transaction bytes that
    // will never come, or expecting the ones that will) and waits, bounded,
    // until every load of either CTA has landed.  Without an abort both
    // counts are equal and every stage has long completed.
    if (rank == 1 && warp == kTmaWarp && lane == 0)
      st_shared_cluster_u32(mapa_shared(smem_addr(&sh->peer_issued), 0), b_issued);
    cluster_sync();
    if (rank == 0 && warp == kTmaWarp && lane == 0) {
      const uint32_t mine = b_issued, peer = sh->peer_issued;
      const uint32_t lo = mine < peer ? mine : peer, hi = mine < peer ? peer : mine;
      for (uint32_t j = lo; j < hi; ++j) {
        if (j < mine) mbar_complete_tx(&sh->full_b[j % S], G::kStageBytes);
        else mbar_arrive_expect_tx(&sh->full_b[j % S], G::kStageBytes);
      }
      int abort_local = 0;
      for (uint32_t j = hi > (uint32_t)S ? hi - S : 0; j < hi; ++j)
        mbar_wait(&sh->full_b[j % S], (j / S) & 1, &abort_local, kDrainLimitNs);
    }
    cluster_sync();  // no peer still uses this CTA's TMEM, barriers or shared memory
  }
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_cg<G::kCG>(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort && dev_status) atomicExch(dev_status, MXQ_ERR_TIMEOUT);
}

// ------------------------------------------------------------------ host

// Row-major bf16 [rows, cols] activations, boxes of 64 columns x box_rows
// rows, 128-byte swizzle; rows past the end read as zero.
bool make_act_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows) {
  return make_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rows, cols, cols * 2, kBox,
                      box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Packed weights viewed as bytes [rows, row_bytes]; boxes of box_cols bytes
// x box_rows rows, with the given swizzle.
bool make_byte_map(CUtensorMap* map, const void* base, int64_t rows, int64_t row_bytes,
                   int box_cols, int box_rows, CUtensorMapSwizzle swz) {
  return make_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, rows, row_bytes, row_bytes,
                      box_cols, box_rows, swz);
}

std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};

template <bool kDgrad, bool kPair>
int launch_tc(const void* a, const void* packed, const void* scales, const int32_t* offs,
              int64_t T, int64_t E, int64_t N, int64_t K, void* y, int32_t* dev_status,
              cudaStream_t st) {
  using G = Geo<kPair>;
  const int64_t kin = kDgrad ? N : K, nout = kDgrad ? K : N;
  constexpr bool kWTma = kDgrad || kPair;
  constexpr uint32_t kSmem = kWTma ? G::kSmemW : G::kSmem;
  constexpr int kWBoxRows = kDgrad ? G::kBK : kBM;
  CUtensorMap map, wmap = {}, smap = {};
  if (!make_act_map(&map, a, T, kin, G::kRowsB)) return MXQ_ERR_CUDA;
  // The input gradient and the pair forward stage W by TMA; the scales
  // too when their rows (K/32 bytes) are a whole number of 16-byte units.
  int scales_by_tma = 0;
  if constexpr (kWTma) {
    if (!make_byte_map(&wmap, packed, E * N, K / 2, 64, kWBoxRows, CU_TENSOR_MAP_SWIZZLE_64B))
      return MXQ_ERR_CUDA;
    if ((K / 32) % 16 == 0 && ((uintptr_t)scales & 15) == 0) {
      if (!make_byte_map(&smap, scales, E * N, K / 32, 16, kWBoxRows, CU_TENSOR_MAP_SWIZZLE_NONE))
        return MXQ_ERR_CUDA;
      scales_by_tma = 1;
    }
  }
  auto kernel = grouped_mm_tc_kernel<kDgrad, kPair>;
  if (allow_dynamic_smem((const void*)kernel, (int)kSmem) != cudaSuccess) return MXQ_ERR_CUDA;
  // Upper bound on the tile count: every expert may add one ragged tile.
  const int64_t tiles = ((T + kBN - 1) / kBN + E) * (nout / G::kTileM);
  const int64_t slots = num_sms() / G::kCG;
  const int64_t units = tiles < slots ? tiles : slots;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(units * G::kCG), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = G::kCG;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(&cfg, kernel, map, wmap, smap, (const uint8_t*)packed,
                                       (const uint8_t*)scales, offs, T, E, N, K,
                                       (__nv_bfloat16*)y, dev_status, g_wait_limit_ns.load(),
                                       scales_by_tma);
  return err == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

}  // namespace

uint64_t get_wait_limit_ns() { return g_wait_limit_ns.load(); }

uint64_t set_wait_limit_ns(uint64_t ns) {
  const uint64_t prev = g_wait_limit_ns;
  g_wait_limit_ns = ns;
  return prev;
}

int launch_grouped_mm(const void* a, const void* packed, const void* scales, const int32_t* offs,
                      int64_t T, int64_t E, int64_t N, int64_t K, int transpose_w, void* y,
                      int32_t* dev_status, cudaStream_t st) {
  const int64_t kin = transpose_w ? N : K, nout = transpose_w ? K : N;
  // Every tensor-core form reads the packed weights in 16-byte units (TMA
  // tiles, or 16-byte loads in the single-CTA forward) and addresses weight
  // rows with 32-bit TMA coordinates.
  const bool w_ok = ((uintptr_t)packed & 15) == 0 && E * N < (int64_t)1 << 31;
  const bool tc = kin % Geo<false>::kBK == 0 && nout % kBM == 0 && ((uintptr_t)a & 15) == 0 &&
                  ((uintptr_t)y & 15) == 0 && T < (int64_t)1 << 31 && kin < (int64_t)1 << 31 &&
                  w_ok;
  if (!tc)
    return launch_grouped_mm_general(a, packed, scales, offs, T, E, N, K, transpose_w, y,
                                     dev_status, st);
  const bool pair = nout % (2 * kBM) == 0 && kin % Geo<true>::kBK == 0 && num_sms() >= 2 && w_ok;
  if (transpose_w)
    return pair ? launch_tc<true, true>(a, packed, scales, offs, T, E, N, K, y, dev_status, st)
                : launch_tc<true, false>(a, packed, scales, offs, T, E, N, K, y, dev_status, st);
  return pair ? launch_tc<false, true>(a, packed, scales, offs, T, E, N, K, y, dev_status, st)
              : launch_tc<false, false>(a, packed, scales, offs, T, E, N, K, y, dev_status, st);
}

MXQ_DEFINE_CHECK_READER(check_record_grouped_mm_tc)

}  // namespace mxq
