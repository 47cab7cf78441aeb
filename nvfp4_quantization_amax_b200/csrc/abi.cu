// extern "C" entry points of libmxq.so: argument validation on the host,
// then a launch on the caller's stream.  Declarations and the contract of
// each call are in include/mxq.h.
#include <cuda_runtime.h>

#include <cstdint>
#include <initializer_list>
#include <map>
#include <mutex>
#include <tuple>

#include "mxq.h"
#include "mxq_device.cuh"
#include "mxq_launch.h"

namespace mxq {

// Debug variant: a checked store one element past the extent it was given
// (the caller's buffer holds two words, so even an unchecked store would
// stay inside it).  The check records (kChkSelfTest, 1, 1) and skips it.
__global__ void debug_selftest_kernel(int32_t* words) {
  if (MXQ_IN_RANGE(kChkSelfTest, 1, 1)) words[1] = 1;
}

MXQ_DEFINE_CHECK_READER(check_record_abi)

int num_sms() {
  static std::mutex mu;
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

int resident_ctas(const void* kernel, int threads, size_t smem) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, int, size_t>, int> cached;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  const auto key = std::make_tuple(kernel, dev, threads, smem);
  std::lock_guard<std::mutex> lock(mu);
  const auto it = cached.find(key);
  if (it != cached.end()) return it->second;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess ||
      n < 1) {
    (void)cudaGetLastError();  // not sticky; keep it out of the launch checks
    n = 1;
  }
  cached[key] = n;
  return n;
}

cudaError_t allow_dynamic_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, int>, cudaError_t> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  const auto key = std::make_tuple(kernel, dev, bytes);
  std::lock_guard<std::mutex> lock(mu);
  const auto it = done.find(key);
  if (it != done.end()) return it->second;
  const cudaError_t err =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err != cudaSuccess) (void)cudaGetLastError();  // reported by the return value
  done[key] = err;
  return err;
}

int wave_grid(const void* kernel, int threads, int64_t n_units, int64_t per_cta) {
  int64_t need = (n_units + per_cta - 1) / per_cta;
  const int64_t wave = (int64_t)num_sms() * resident_ctas(kernel, threads, 0);
  if (need > wave) need = wave;
  return (int)(need < 1 ? 1 : need);
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
// Elements must sit on their own size (2 or 4 bytes) for the general kernels.
static bool elem_aligned(const void* p, int d) {
  return ((uintptr_t)p & (uintptr_t)((d == MXQ_F32 ? 4 : 2) - 1)) == 0;
}
// An int32 word (offs, a status word) sits on a 4-byte boundary; null passes.
static bool word_aligned(const void* p) { return ((uintptr_t)p & 3u) == 0; }
static bool valid_dtype(int d) { return d == MXQ_BF16 || d == MXQ_F16 || d == MXQ_F32; }
static int elem_bytes(int d) { return d == MXQ_F32 ? 4 : 2; }

static bool overlap(const void* a, int64_t na, const void* b, int64_t nb) {
  auto x = (uintptr_t)a, y = (uintptr_t)b;
  return x < y + (uintptr_t)nb && y < x + (uintptr_t)na;
}

// A byte extent of a call's buffer: where it starts and how long it is.
struct Extent {
  const void* p;
  int64_t bytes;
};

// Whether every output extent is disjoint from every other extent (inputs
// may overlap one another).  Null or empty extents take no part.
static bool no_alias(std::initializer_list<Extent> outputs, std::initializer_list<Extent> inputs) {
  for (auto o = outputs.begin(); o != outputs.end(); ++o) {
    if (!o->p || o->bytes <= 0) continue;
    for (auto q = o + 1; q != outputs.end(); ++q)
      if (q->p && q->bytes > 0 && overlap(o->p, o->bytes, q->p, q->bytes)) return false;
    for (const Extent& i : inputs)
      if (i.p && i.bytes > 0 && overlap(o->p, o->bytes, i.p, i.bytes)) return false;
  }
  return true;
}

// rows x cols elements of up to 8 bytes have a byte extent below 2^62.
static bool fits(int64_t rows, int64_t cols) {
  return rows >= 0 && cols >= 0 && (cols == 0 || rows <= ((int64_t)1 << 59) / cols);
}

}  // namespace mxq

using namespace mxq;

extern "C" {

int mx_quantize(const void* x, int x_dtype, int64_t rows, int64_t K, void* packed, void* scales,
                void* stream) {
  if (!valid_dtype(x_dtype)) return MXQ_ERR_INVALID_ARG;
  if (rows < 0 || K < 0 || K % 32 != 0) return MXQ_ERR_SHAPE;
  if (rows == 0 || K == 0) return MXQ_OK;
  if (!x || !packed || !scales) return MXQ_ERR_INVALID_ARG;
  if (!fits(rows, K)) return MXQ_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(packed)) return MXQ_ERR_ALIGNMENT;
  if (!no_alias({{packed, rows * K / 2}, {scales, rows * K / 32}},
                {{x, rows * K * elem_bytes(x_dtype)}}))
    return MXQ_ERR_INVALID_ARG;
  return launch_mx_quantize(x, x_dtype, rows, K, packed, scales, (cudaStream_t)stream);
}

int mx_dequantize(const void* packed, const void* scales, int64_t rows, int64_t K, void* out,
                  int out_dtype, void* stream) {
  if (!valid_dtype(out_dtype)) return MXQ_ERR_INVALID_ARG;
  if (rows < 0 || K < 0 || K % 32 != 0) return MXQ_ERR_SHAPE;
  if (rows == 0 || K == 0) return MXQ_OK;
  if (!packed || !scales || !out) return MXQ_ERR_INVALID_ARG;
  if (!fits(rows, K)) return MXQ_ERR_SHAPE;
  if (!aligned16(packed) || !aligned16(out)) return MXQ_ERR_ALIGNMENT;
  if (!no_alias({{out, rows * K * elem_bytes(out_dtype)}},
                {{packed, rows * K / 2}, {scales, rows * K / 32}}))
    return MXQ_ERR_INVALID_ARG;
  return launch_mx_dequantize(packed, scales, rows, K, out, out_dtype, (cudaStream_t)stream);
}

int quantize_cache(const void* in, void* out, int dtype, int64_t rows, int64_t channels,
                   int format, int32_t block_size, void* stream) {
  if (!valid_dtype(dtype)) return MXQ_ERR_INVALID_ARG;
  if (format != MXQ_FMT_FP8 && format != MXQ_FMT_MXFP4 && format != MXQ_FMT_NVFP4)
    return MXQ_ERR_INVALID_ARG;
  if (rows < 0 || channels < 0 || block_size < 1) return MXQ_ERR_SHAPE;
  if (rows == 0 || channels == 0) return MXQ_OK;
  if (!in || !out) return MXQ_ERR_INVALID_ARG;
  if (!fits(rows, channels)) return MXQ_ERR_SHAPE;
  int64_t bytes = rows * channels * elem_bytes(dtype);
  if (overlap(in, bytes, out, bytes)) return MXQ_ERR_INVALID_ARG;
  if (!elem_aligned(in, dtype) || !elem_aligned(out, dtype)) return MXQ_ERR_ALIGNMENT;
  int B = block_size;
  bool pow2_b = B >= 8 && B <= 256 && (B & (B - 1)) == 0;
  bool fast = pow2_b && channels % B == 0 && aligned16(in) && aligned16(out);
  return launch_quantize_cache(in, out, dtype, rows, channels, format, B, fast,
                               (cudaStream_t)stream);
}

static int check_packed_cache(int dtype, int64_t rows, int64_t C, int format, int32_t B) {
  if (!valid_dtype(dtype)) return MXQ_ERR_INVALID_ARG;
  if (format != MXQ_FMT_FP8 && format != MXQ_FMT_MXFP4 && format != MXQ_FMT_NVFP4)
    return MXQ_ERR_INVALID_ARG;
  if (rows < 0 || C < 0 || B < 1 || C % B != 0) return MXQ_ERR_SHAPE;
  if (format != MXQ_FMT_FP8 && B % 2 != 0) return MXQ_ERR_SHAPE;
  return MXQ_OK;
}

static bool packed_fast(int32_t B, const void* elems, const void* codes) {
  return B >= 8 && B <= 256 && (B & (B - 1)) == 0 && aligned16(elems) && aligned16(codes);
}

int quantize_cache_packed(const void* in, int dtype, int64_t rows, int64_t channels, int format,
                          int32_t block_size, void* codes, void* scales, void* stream) {
  int rc = check_packed_cache(dtype, rows, channels, format, block_size);
  if (rc != MXQ_OK) return rc;
  if (rows == 0 || channels == 0) return MXQ_OK;
  if (!in || !codes || !scales) return MXQ_ERR_INVALID_ARG;
  if (!fits(rows, channels)) return MXQ_ERR_SHAPE;
  if (!elem_aligned(in, dtype)) return MXQ_ERR_ALIGNMENT;
  const int64_t code_bytes = format == MXQ_FMT_FP8 ? rows * channels : rows * channels / 2;
  if (!no_alias({{codes, code_bytes}, {scales, rows * (channels / block_size)}},
                {{in, rows * channels * elem_bytes(dtype)}}))
    return MXQ_ERR_INVALID_ARG;
  return launch_quantize_cache_packed(in, dtype, rows, channels, format, block_size, codes, scales,
                                      packed_fast(block_size, in, codes), (cudaStream_t)stream);
}

int dequantize_cache_packed(const void* codes, const void* scales, int64_t rows, int64_t channels,
                            int format, int32_t block_size, void* out, int out_dtype,
                            void* stream) {
  int rc = check_packed_cache(out_dtype, rows, channels, format, block_size);
  if (rc != MXQ_OK) return rc;
  if (rows == 0 || channels == 0) return MXQ_OK;
  if (!codes || !scales || !out) return MXQ_ERR_INVALID_ARG;
  if (!fits(rows, channels)) return MXQ_ERR_SHAPE;
  if (!elem_aligned(out, out_dtype)) return MXQ_ERR_ALIGNMENT;
  const int64_t code_bytes = format == MXQ_FMT_FP8 ? rows * channels : rows * channels / 2;
  if (!no_alias({{out, rows * channels * elem_bytes(out_dtype)}},
                {{codes, code_bytes}, {scales, rows * (channels / block_size)}}))
    return MXQ_ERR_INVALID_ARG;
  return launch_dequantize_cache_packed(codes, scales, rows, channels, format, block_size, out,
                                        out_dtype, packed_fast(block_size, out, codes),
                                        (cudaStream_t)stream);
}

int mxfp4_grouped_mm(const void* a, const void* packed, const void* scales, const int32_t* offs,
                     int64_t T, int64_t E, int64_t N, int64_t K, int transpose_w, void* y,
                     int32_t* dev_status, void* stream) {
  if (T < 0 || E < 1 || N < 1 || K < 32 || K % 32 != 0) return MXQ_ERR_SHAPE;
  if (transpose_w != 0 && transpose_w != 1) return MXQ_ERR_INVALID_ARG;
  if (!packed || !scales || !offs) return MXQ_ERR_INVALID_ARG;
  if (T == 0) return MXQ_OK;
  if (!a || !y) return MXQ_ERR_INVALID_ARG;
  if (!fits(T, N > K ? N : K) || !fits(E, N) || !fits(E * N, K)) return MXQ_ERR_SHAPE;
  if (E > 65536) return MXQ_ERR_UNSUPPORTED;
  // bf16 elements on their own size, int32 words on theirs: the general
  // kernel reads and writes them one element at a time.
  if (!elem_aligned(a, MXQ_BF16) || !elem_aligned(y, MXQ_BF16) || !word_aligned(offs) ||
      !word_aligned(dev_status))
    return MXQ_ERR_ALIGNMENT;
  {
    const int64_t kin = transpose_w ? N : K, nout = transpose_w ? K : N;
    if (!no_alias({{y, T * nout * 2}, {dev_status, 4}},
                  {{a, T * kin * 2}, {packed, E * N * K / 2}, {scales, E * N * K / 32},
                   {offs, E * 4}}))
      return MXQ_ERR_INVALID_ARG;
  }
  return launch_grouped_mm(a, packed, scales, offs, T, E, N, K, transpose_w, y, dev_status,
                           (cudaStream_t)stream);
}

int mxfp4_w4a4_grouped_mm(const void* x_packed, const void* x_scales, const void* packed,
                          const void* scales, const int32_t* offs, int64_t T, int64_t E, int64_t N,
                          int64_t K, void* y, int32_t* dev_status, void* stream) {
  if (T < 0 || E < 1 || N < 1 || K < 32 || K % 32 != 0) return MXQ_ERR_SHAPE;
  if (!packed || !scales || !offs) return MXQ_ERR_INVALID_ARG;
  if (T == 0) return MXQ_OK;
  if (!x_packed || !x_scales || !y) return MXQ_ERR_INVALID_ARG;
  if (!fits(T, N > K ? N : K) || !fits(E, N) || !fits(E * N, K)) return MXQ_ERR_SHAPE;
  if (K % 256 != 0 || N % 128 != 0 || T >= ((int64_t)1 << 31) || E * N >= ((int64_t)1 << 31))
    return MXQ_ERR_UNSUPPORTED;
  if (!aligned16(x_packed) || !aligned16(x_scales) || !aligned16(packed) || !aligned16(scales) ||
      !aligned16(y) || !word_aligned(offs) || !word_aligned(dev_status))
    return MXQ_ERR_ALIGNMENT;
  if (!no_alias({{y, T * N * 2}, {dev_status, 4}},
                {{x_packed, T * K / 2}, {x_scales, T * K / 32}, {packed, E * N * K / 2},
                 {scales, E * N * K / 32}, {offs, E * 4}}))
    return MXQ_ERR_INVALID_ARG;
  return launch_w4a4_grouped_mm(x_packed, x_scales, packed, scales, offs, T, E, N, K, y,
                                dev_status, get_wait_limit_ns(), (cudaStream_t)stream);
}

int nvfp4_w4a4_grouped_mm(const void* x_packed, const void* x_block_scales,
                          const float* x_global_scale, const void* packed,
                          const void* block_scales, const float* w_global_scales,
                          const int32_t* offs, int64_t T, int64_t E, int64_t N, int64_t K, void* y,
                          int32_t* dev_status, void* stream) {
  if (T < 0 || E < 1 || N < 1 || K < 16 || K % 16 != 0) return MXQ_ERR_SHAPE;
  if (!packed || !block_scales || !w_global_scales || !offs) return MXQ_ERR_INVALID_ARG;
  if (T == 0) return MXQ_OK;
  if (!x_packed || !x_block_scales || !x_global_scale || !y) return MXQ_ERR_INVALID_ARG;
  if (!fits(T, N > K ? N : K) || !fits(E, N) || !fits(E * N, K)) return MXQ_ERR_SHAPE;
  if (K % 256 != 0 || N % 128 != 0 || T >= ((int64_t)1 << 31) || E * N >= ((int64_t)1 << 31))
    return MXQ_ERR_UNSUPPORTED;
  if (!aligned16(x_packed) || !aligned16(x_block_scales) || !aligned16(packed) ||
      !aligned16(block_scales) || !aligned16(y) || !word_aligned(offs) ||
      !word_aligned(dev_status) || !word_aligned(x_global_scale) || !word_aligned(w_global_scales))
    return MXQ_ERR_ALIGNMENT;
  if (!no_alias({{y, T * N * 2}, {dev_status, 4}},
                {{x_packed, T * K / 2}, {x_block_scales, T * K / 16}, {x_global_scale, 4},
                 {packed, E * N * K / 2}, {block_scales, E * N * K / 16},
                 {w_global_scales, E * 4}, {offs, E * 4}}))
    return MXQ_ERR_INVALID_ARG;
  return launch_nvfp4_w4a4_grouped_mm(x_packed, x_block_scales, x_global_scale, packed,
                                      block_scales, w_global_scales, offs, T, E, N, K, y,
                                      dev_status, get_wait_limit_ns(), (cudaStream_t)stream);
}

int nvfp4_quantize(const void* x, int x_dtype, int64_t rows, int64_t K, void* packed,
                   void* block_scales, float* global_scale, void* workspace, void* stream) {
  if (!valid_dtype(x_dtype)) return MXQ_ERR_INVALID_ARG;
  if (rows < 0 || K < 0 || K % 16 != 0) return MXQ_ERR_SHAPE;
  if (!global_scale || !workspace) return MXQ_ERR_INVALID_ARG;
  if (rows > 0 && K > 0 && (!x || !packed || !block_scales)) return MXQ_ERR_INVALID_ARG;
  if (!fits(rows, K)) return MXQ_ERR_SHAPE;
  if (!aligned16(workspace) || !word_aligned(global_scale) ||
      (rows > 0 && K > 0 && (!aligned16(x) || !aligned16(packed))))
    return MXQ_ERR_ALIGNMENT;
  if (!no_alias({{packed, rows * K / 2}, {block_scales, rows * K / 16}, {global_scale, 4},
                 {workspace, MXQ_NVFP4_WORKSPACE_BYTES}},
                {{x, rows * K * elem_bytes(x_dtype)}}))
    return MXQ_ERR_INVALID_ARG;
  return launch_nvfp4_quantize(x, x_dtype, rows, K, packed, block_scales, global_scale,
                               (uint32_t*)workspace, (cudaStream_t)stream);
}

int nvfp4_quantize_mse(const void* x, int x_dtype, int64_t rows, int64_t K, void* packed,
                       void* block_scales, float* global_scale, void* workspace, void* stream) {
  if (!valid_dtype(x_dtype)) return MXQ_ERR_INVALID_ARG;
  if (rows < 0 || K < 0 || K % 16 != 0) return MXQ_ERR_SHAPE;
  if (!global_scale || !workspace) return MXQ_ERR_INVALID_ARG;
  if (rows > 0 && K > 0 && (!x || !packed || !block_scales)) return MXQ_ERR_INVALID_ARG;
  if (!fits(rows, K)) return MXQ_ERR_SHAPE;
  if (!aligned16(workspace) || !word_aligned(global_scale) ||
      (rows > 0 && K > 0 && (!aligned16(x) || !aligned16(packed))))
    return MXQ_ERR_ALIGNMENT;
  if (!no_alias({{packed, rows * K / 2}, {block_scales, rows * K / 16}, {global_scale, 4},
                 {workspace, MXQ_NVFP4_WORKSPACE_BYTES}},
                {{x, rows * K * elem_bytes(x_dtype)}}))
    return MXQ_ERR_INVALID_ARG;
  return launch_nvfp4_quantize_mse(x, x_dtype, rows, K, packed, block_scales, global_scale,
                                   (uint32_t*)workspace, (cudaStream_t)stream);
}

int nvfp4_quantize_noalloc(const void* x, int x_dtype, int64_t rows, int64_t K, void* packed,
                           void* block_scales, float* global_scale, void* stream) {
  if (!valid_dtype(x_dtype)) return MXQ_ERR_INVALID_ARG;
  if (rows < 0 || K < 0 || K % 16 != 0) return MXQ_ERR_SHAPE;
  if (!global_scale) return MXQ_ERR_INVALID_ARG;
  if (rows > 0 && K > 0 && (!x || !packed || !block_scales)) return MXQ_ERR_INVALID_ARG;
  if (!fits(rows, K)) return MXQ_ERR_SHAPE;
  if (!word_aligned(global_scale) || (rows > 0 && K > 0 && (!aligned16(x) || !aligned16(packed))))
    return MXQ_ERR_ALIGNMENT;
  if (!no_alias({{packed, rows * K / 2}, {block_scales, rows * K / 16}, {global_scale, 4}},
                {{x, rows * K * elem_bytes(x_dtype)}}))
    return MXQ_ERR_INVALID_ARG;
  int status = MXQ_OK;
  uint32_t* scratch = noalloc_scratch(MXQ_NVFP4_WORKSPACE_BYTES, &status);
  if (!scratch) return status;
  return launch_nvfp4_quantize(x, x_dtype, rows, K, packed, block_scales, global_scale, scratch,
                               (cudaStream_t)stream);
}

int nvfp4_dequantize(const void* packed, const void* block_scales, const float* global_scale,
                     int64_t rows, int64_t K, void* out, int out_dtype, void* stream) {
  if (!valid_dtype(out_dtype)) return MXQ_ERR_INVALID_ARG;
  if (rows < 0 || K < 0 || K % 16 != 0) return MXQ_ERR_SHAPE;
  if (rows == 0 || K == 0) return MXQ_OK;
  if (!packed || !block_scales || !global_scale || !out) return MXQ_ERR_INVALID_ARG;
  if (!fits(rows, K)) return MXQ_ERR_SHAPE;
  if (!aligned16(packed) || !aligned16(out) || !word_aligned(global_scale))
    return MXQ_ERR_ALIGNMENT;
  if (!no_alias({{out, rows * K * elem_bytes(out_dtype)}},
                {{packed, rows * K / 2}, {block_scales, rows * K / 16}, {global_scale, 4}}))
    return MXQ_ERR_INVALID_ARG;
  return launch_nvfp4_dequantize(packed, block_scales, global_scale, rows, K, out, out_dtype,
                                 (cudaStream_t)stream);
}

const char* mxq_status_string(int status) {
  switch (status) {
    case MXQ_OK: return "MXQ_OK";
    case MXQ_ERR_INVALID_ARG: return "MXQ_ERR_INVALID_ARG";
    case MXQ_ERR_SHAPE: return "MXQ_ERR_SHAPE";
    case MXQ_ERR_ALIGNMENT: return "MXQ_ERR_ALIGNMENT";
    case MXQ_ERR_UNSUPPORTED: return "MXQ_ERR_UNSUPPORTED";
    case MXQ_ERR_CUDA: return "MXQ_ERR_CUDA";
    case MXQ_ERR_BAD_OFFS: return "MXQ_ERR_BAD_OFFS";
    case MXQ_ERR_TIMEOUT: return "MXQ_ERR_TIMEOUT";
    default: return "MXQ_ERR_UNKNOWN";
  }
}

int mxq_debug_checks(int64_t* record) {
  if (!record) return MXQ_ERR_INVALID_ARG;
  record[0] = record[1] = record[2] = 0;
#ifdef MXQ_DEBUG_CHECKS
  using Reader = int (*)(unsigned long long*);
  const Reader readers[] = {check_record_abi,         check_record_elementwise,
                            check_record_cache_packed, check_record_nvfp4,
                            check_record_nvfp4_mse,    check_record_grouped_mm_general,
                            check_record_grouped_mm_tc, check_record_w4a4};
  int status = MXQ_OK;
  for (Reader rd : readers) {
    unsigned long long r[3];
    const int rc = rd(r);
    if (rc != MXQ_OK) status = rc;
    else if (r[0] != 0 && record[0] == 0)
      for (int i = 0; i < 3; ++i) record[i] = (int64_t)r[i];
  }
  return status;
#else
  return MXQ_ERR_UNSUPPORTED;
#endif
}

int mxq_debug_selftest(int32_t* dev_words, void* stream) {
  if (!dev_words) return MXQ_ERR_INVALID_ARG;
  if (((uintptr_t)dev_words & 3) != 0) return MXQ_ERR_ALIGNMENT;
#ifdef MXQ_DEBUG_CHECKS
  debug_selftest_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(dev_words);
  return cudaGetLastError() == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
#else
  (void)stream;
  return MXQ_ERR_UNSUPPORTED;
#endif
}

uint64_t mxq_set_wait_limit_ns(uint64_t ns) { return set_wait_limit_ns(ns); }

int mxq_version(void) { return 100; }

}  // extern "C"
