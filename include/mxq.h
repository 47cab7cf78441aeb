/*
 * mxq.h - C ABI of libmxq.so: block-scaled microscaling quantization on
 * NVIDIA B200 (sm_100a).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers named as device buffers are CUDA device pointers owned by the
 *    caller.  The library allocates nothing and keeps no pointer after a
 *    call returns.
 *  - Tensors are dense and row-major.  Leading dimensions are flattened into
 *    `rows` (rows = numel / last_dim).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Every call is asynchronous on that stream; the library never
 *    synchronizes.
 *  - Return value: MXQ_OK (0) or a negative mxq_status.  Argument errors are
 *    detected on the host before anything is launched and leave every output
 *    untouched.  MXQ_ERR_CUDA reports a failed launch (cudaGetLastError).
 *  - Outputs never alias: an output buffer that overlaps an input or another
 *    output of the same call (by the byte extents the sizes give) is
 *    MXQ_ERR_INVALID_ARG.  Sizes whose byte extents do not fit in 62 bits
 *    are MXQ_ERR_SHAPE.
 *  - Element dtypes are mxq_dtype values; floating-point results are rounded
 *    to nearest-even with subnormals kept and overflow to +-infinity.
 *  - Inputs are expected to be finite; NaN/Inf inputs give unspecified
 *    (but memory-safe) results.
 *
 * Sources.  The operations follow these pages (title, then section):
 *  [MX] "nemo_automodel.components.quantization.mxfp4": module docstring
 *       (packed layout), quantize_mxfp4, dequantize_mxfp4, MXFP4GroupedMM,
 *       _FP4_E2M1_TABLE, _FP4_E2M1_MIDPOINTS, MXFP4_BLOCK_SIZE.
 *  [CQ] "nemo_automodel.components.models.deepseek_v41.quantization":
 *       quantize_cache, _power_of_two_ceiling.
 *  [MO] "NVIDIA Model Optimizer: from mtq.quantize to a 4.95-bit
 *       DeepSeek-R1", section "NVFP4 in the code: two scales and a nibble"
 *       (E2M1 tie rule and nibble packing, E4M3 maximum 448).
 */
#ifndef MXQ_H
#define MXQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MXQ_OK = 0,
  MXQ_ERR_INVALID_ARG = -1, /* null pointer, bad enum, aliasing in/out    */
  MXQ_ERR_SHAPE = -2,       /* negative size, K % 32 != 0, ...            */
  MXQ_ERR_ALIGNMENT = -3,   /* a pointer the call needs aligned is not    */
  MXQ_ERR_UNSUPPORTED = -4, /* valid request this library does not handle */
  MXQ_ERR_CUDA = -5,        /* launch failed                              */
  MXQ_ERR_BAD_OFFS = -6,    /* device-side: offs not a valid partition    */
  MXQ_ERR_TIMEOUT = -7      /* device-side: a pipeline wait gave up       */
} mxq_status;

typedef enum { MXQ_BF16 = 0, MXQ_F16 = 1, MXQ_F32 = 2 } mxq_dtype;

typedef enum { MXQ_FMT_FP8 = 0, MXQ_FMT_MXFP4 = 1, MXQ_FMT_NVFP4 = 2 } mxq_format;

/* MXFP4 quantize + pack along the last dimension  ([MX] quantize_mxfp4).
 *
 *  x       device, [rows, K] elements of x_dtype (bf16, f16 or f32), 16-byte
 *          aligned.
 *  packed  device, [rows, K/2] bytes, 16-byte aligned (output).  Byte j of a
 *          row holds the E2M1 code of column 2j in its low nibble and of
 *          column 2j+1 in its high nibble ([MX] module docstring).
 *  scales  device, [rows, K/32] bytes (output): one E8M0 scale (float8_e8m0fnu
 *          bits, value 2^(byte-127)) per 32 contiguous columns.
 *
 *  Per 32-column block: amax = max |x|; scale exponent e = floor(log2(amax))
 *  - 2, clamped to [-127, 127] (an all-zero block takes -127, byte 0x00);
 *  code = E2M1 cast of x / 2^e: the nearest of {0,0.5,1,1.5,2,3,4,6}, ties
 *  to the even code (ties at 0.75, 1.75, 3.5 go up, [MO] _cast_fp4), values
 *  beyond 6 saturate to 6, sign bit set iff x < 0.
 *  Errors: K % 32 != 0 -> MXQ_ERR_SHAPE; null or misaligned x/packed ->
 *  MXQ_ERR_INVALID_ARG / MXQ_ERR_ALIGNMENT.  rows == 0 or K == 0: no-op. */
int mx_quantize(const void* x, int x_dtype, int64_t rows, int64_t K, void* packed,
                void* scales, void* stream);

/* MXFP4 unpack + scale ([MX] dequantize_mxfp4).
 *
 *  packed  device, [rows, K/2] bytes, 16-byte aligned (layout as above).
 *  scales  device, [rows, K/32] E8M0 bytes.
 *  out     device, [rows, K] elements of out_dtype, 16-byte aligned (output).
 *
 *  out[r][k] = E2M1_TABLE[nibble] * 2^(scale_byte - 127), rounded to
 *  out_dtype (exact in bf16/f32 except overflow; f16 overflows above 65504
 *  to +-inf).  Nibble 8 decodes to +0.0.  Scale byte 0xFF (E8M0 NaN) gives
 *  NaN (bf16 0x7FC0, f16 0x7E00, f32 0x7FC00000) for its 32 values.
 *  Errors as for mx_quantize. */
int mx_dequantize(const void* packed, const void* scales, int64_t rows, int64_t K, void* out,
                  int out_dtype, void* stream);

/* Fake quantization of cache values ([CQ] quantize_cache).
 *
 *  in, out  device, [rows, channels] elements of dtype; out must not overlap
 *           in (the result is independently stored).
 *  format   MXQ_FMT_FP8 (E4M3 elements), MXQ_FMT_MXFP4 (E2M1 elements,
 *           E8M0-range scales) or MXQ_FMT_NVFP4 (E2M1 elements, E4M3-range
 *           scales).
 *  block_size  channels per scale (>= 1).  A final partial group of a row
 *           uses its own channels only (the page's zero padding).
 *
 *  Per group: amax = max |x|; qmax = 448 (fp8) or 6 (fp4); scale s = the
 *  least power of two with s*qmax >= amax (_power_of_two_ceiling of
 *  amax/qmax, decided exactly), clamped to [2^-126, 2^127] (fp8, mxfp4) or
 *  [2^-9, 2^8] (nvfp4); an all-zero group takes the lower clamp.
 *  out = round_dtype(q(x/s) * s) with q the E4M3 cast (nearest-even,
 *  saturating at 448, sign of zero kept) or the E2M1 cast above (a zero
 *  magnitude gives +0.0).
 *  Fast path: block_size in {8,16,32,64,128,256}, channels % block_size == 0,
 *  16-byte aligned in/out.  Anything else runs a slower general kernel.
 *  Errors: block_size < 1 -> MXQ_ERR_SHAPE; bad format/dtype or overlapping
 *  in/out -> MXQ_ERR_INVALID_ARG; in/out not aligned to the element size ->
 *  MXQ_ERR_ALIGNMENT. */
int quantize_cache(const void* in, void* out, int dtype, int64_t rows, int64_t channels,
                   int format, int32_t block_size, void* stream);

/* Packed (stored) cache quantization ([CQ] _CacheQuantization.forward:
 * fp8; mxfp4 with an E8M0 scale; nvfp4 with an E4M3 scale).  Keeps the codes
 * and scales that quantize_cache rounds to instead of multiplying back.
 *
 *  in       device, [rows, channels] elements of dtype (bf16, f16 or f32).
 *  codes    device (output).  fp8: [rows, channels] E4M3 bytes (the cast of
 *           x / 2^k, sign of zero kept).  mxfp4, nvfp4: [rows, channels/2]
 *           bytes of two E2M1 codes, the even channel in the low nibble, sign
 *           bit iff x < 0 (as mx_quantize).
 *  scales   device, [rows, channels/block_size] bytes (output): the group's
 *           scale 2^k (k chosen exactly as in quantize_cache) as an E8M0 byte
 *           k + 127 for fp8 and mxfp4, as the E4M3 encoding of 2^k for nvfp4
 *           (k in [-9, 8] is always an E4M3 value).
 *  block_size  channels per scale; channels % block_size == 0 (no partial
 *           group is stored) and, for mxfp4/nvfp4, block_size even.
 *  dequantize_cache_packed(quantize_cache_packed(x)) equals
 *  quantize_cache(x) bit for bit.
 *  Fast path: block_size in {8,...,256} a power of two, 16-byte aligned in
 *  and codes; anything else valid runs a slower general kernel.
 *  Errors: bad dtype/format or null pointer -> MXQ_ERR_INVALID_ARG;
 *  block_size < 1, channels % block_size != 0 or an odd fp4 block_size ->
 *  MXQ_ERR_SHAPE; in not aligned to its element size -> MXQ_ERR_ALIGNMENT.
 *  rows == 0 or channels == 0: no-op. */
int quantize_cache_packed(const void* in, int dtype, int64_t rows, int64_t channels, int format,
                          int32_t block_size, void* codes, void* scales, void* stream);

/* Unpack the stored cache form: out = round_dtype(code value * scale), the
 * product taken in f32 (exact for every code and scale the packer writes).
 * fp4 zero codes (either sign) give +0.0; an E8M0 byte 0xFF gives NaN.
 * Arguments, layout and errors as quantize_cache_packed, with out
 * [rows, channels] of out_dtype. */
int dequantize_cache_packed(const void* codes, const void* scales, int64_t rows, int64_t channels,
                            int format, int32_t block_size, void* out, int out_dtype,
                            void* stream);

/* Grouped GEMM over MXFP4-packed expert weights, dequantized on the fly
 * ([MX] MXFP4GroupedMM forward and backward).
 *
 *  a        device, bf16 [T, Kin], rows grouped contiguously by expert,
 *           aligned to 2 bytes (16 for the tensor-core path, below).
 *  packed   device, [E, N, K/2] bytes; scales device, [E, N, K/32] E8M0
 *           bytes: W_e[n][k] = dequantized value, exactly representable in
 *           bf16 for scale bytes <= 252.
 *  offs     device, int32 [E], 4-byte aligned: inclusive prefix sums of the
 *           expert row counts; expert e owns rows [offs[e-1], offs[e]) with
 *           offs[-1] = 0.
 *  transpose_w = 0 (forward):        Kin = K, y bf16 [T, N], y = a . W_e^T
 *  transpose_w = 1 (input gradient): Kin = N, y bf16 [T, K], y = a . W_e
 *  Products accumulate in fp32; y is rounded to bf16 (nearest-even).
 *  dev_status  device int32 (nullable, 4-byte aligned).  If offs is not
 *           non-decreasing
 *           with offs[E-1] == T the kernel writes MXQ_ERR_BAD_OFFS there and
 *           leaves y unwritten; if a pipeline wait gives up it writes
 *           MXQ_ERR_TIMEOUT.  The kernel never writes MXQ_OK: clear the word
 *           before the call to read it afterwards.
 *  Errors (host): K % 32 != 0, E < 1, N < 1, T < 0 -> MXQ_ERR_SHAPE; null
 *  pointers -> MXQ_ERR_INVALID_ARG; a or y not on a 2-byte boundary, offs or
 *  dev_status not on a 4-byte boundary -> MXQ_ERR_ALIGNMENT.  The
 *  tensor-core path needs the output width (N, or K for the input gradient)
 *  a multiple of 128, the reduction width a multiple of 64, and a, y and
 *  packed 16-byte aligned; other valid calls run a slower general kernel
 *  with the same results up to the order of the fp32 accumulation. */
int mxfp4_grouped_mm(const void* a, const void* packed, const void* scales, const int32_t* offs,
                     int64_t T, int64_t E, int64_t N, int64_t K, int transpose_w, void* y,
                     int32_t* dev_status, void* stream);

/* W4A4 grouped GEMM: MXFP4 activations times MXFP4 expert weights on the
 * block-scaled tensor cores ([MO] "W4A4 NVFP4 on FP4 tensor cores", with
 * the MX format of [MX]).
 *
 *  x_packed, x_scales  device, the activations as mx_quantize writes them:
 *           [T, K/2] E2M1 bytes and [T, K/32] E8M0 bytes, rows grouped
 *           contiguously by expert.
 *  packed, scales, offs, dev_status  as mxfp4_grouped_mm (forward).
 *  y        device, bf16 [T, N]: y[t, n] = sum_k xq[t, k] W_e[n, k] with xq
 *           the dequantized activation; products are exact, the sum is
 *           accumulated in f32 by the tensor core and rounded once to bf16.
 *  Every pointer 16-byte aligned, except offs and dev_status (4 bytes).
 *  Errors: K % 32 != 0, E < 1, N < 1, T < 0 -> MXQ_ERR_SHAPE; null ->
 *  MXQ_ERR_INVALID_ARG; misaligned -> MXQ_ERR_ALIGNMENT; K % 256 != 0 or
 *  N % 128 != 0 (shapes this kernel does not tile) -> MXQ_ERR_UNSUPPORTED.
 *  T == 0: no-op. */
int mxfp4_w4a4_grouped_mm(const void* x_packed, const void* x_scales, const void* packed,
                          const void* scales, const int32_t* offs, int64_t T, int64_t E, int64_t N,
                          int64_t K, void* y, int32_t* dev_status, void* stream);

/* W4A4 grouped GEMM in NVFP4: activations and expert weights both NVFP4 on
 * the block-scaled tensor cores ([MO] "W4A4 NVFP4 on FP4 tensor cores";
 * two-level format of [MO] "NVFP4 in the code: two scales and a nibble").
 *
 *  x_packed, x_block_scales, x_global_scale  device, the activations as
 *           nvfp4_quantize writes them for the whole [T, K] tensor: [T, K/2]
 *           E2M1 bytes, [T, K/16] E4M3 bytes, one float g_x.
 *  packed, block_scales  device, [E, N, K/2] and [E, N, K/16] bytes: each
 *           expert's weight in NVFP4 (e.g. nvfp4_quantize of W_e).
 *  w_global_scales  device, float [E]: each expert's g.
 *  offs, dev_status, y  as mxfp4_w4a4_grouped_mm; the two global-scale
 *           pointers 4-byte aligned, every other pointer 16-byte aligned.
 *  y[t, n] = g_x g_w[e] sum_k (code * s_b)_x[t, k] (code * s_b)_w[n, k]: the
 *  tensor core multiplies codes and block scales exactly and accumulates in
 *  f32; the product of the two global scales multiplies the f32 sum, and y is
 *  rounded to bf16.
 *  Errors as mxfp4_w4a4_grouped_mm (K % 16 != 0 -> MXQ_ERR_SHAPE; K % 256 or
 *  N % 128 nonzero -> MXQ_ERR_UNSUPPORTED). */
int nvfp4_w4a4_grouped_mm(const void* x_packed, const void* x_block_scales,
                          const float* x_global_scale, const void* packed,
                          const void* block_scales, const float* w_global_scales,
                          const int32_t* offs, int64_t T, int64_t E, int64_t N, int64_t K, void* y,
                          int32_t* dev_status, void* stream);

/* Device workspace nvfp4_quantize needs (bytes, 16-byte aligned). */
#define MXQ_NVFP4_WORKSPACE_BYTES 16

/* NVFP4 two-level quantize + pack along the last dimension ([MO] "NVFP4 in
 * the code: two scales and a nibble"; block 16 with E4M3 scales from the
 * numerics YAML in "mtq.quantize is three moves").
 *
 *  x             device, [rows, K] elements of x_dtype, K % 16 == 0, 16-byte
 *                aligned.
 *  packed        device, [rows, K/2] bytes (output), 16-byte aligned: E2M1
 *                codes, low nibble = even column.
 *  block_scales  device, [rows, K/16] E4M3 bytes (output), one per 16 values.
 *  global_scale  device, one float (output), 4-byte aligned: g = max|x| /
 *                (6 * 448).
 *  workspace     device, MXQ_NVFP4_WORKSPACE_BYTES bytes of scratch, owned by
 *                the caller, clobbered; calls that overlap on the GPU must not
 *                share it.
 *
 *  In binary32 arithmetic: g = amax / 2688; per block s_b = E4M3(amax_b /
 *  (6 g)) after replacing a zero quotient by 1.0 and clamping to [2^-9, 448];
 *  code = E2M1(x / (s_b * g)) (nearest-even on the grid, saturating at 6,
 *  sign bit iff x < 0).  An all-zero tensor gives g = 0, codes 0 and block
 *  scales 1.0.  Precondition: max|x| is 0 or at least 2^-126.
 *  Errors: K % 16 != 0 -> MXQ_ERR_SHAPE; null -> MXQ_ERR_INVALID_ARG;
 *  misaligned x/packed/workspace/global_scale -> MXQ_ERR_ALIGNMENT. */
int nvfp4_quantize(const void* x, int x_dtype, int64_t rows, int64_t K, void* packed,
                   void* block_scales, float* global_scale, void* workspace, void* stream);

/* NVFP4 unpack: out[r][k] = round_dtype(fl32(E2M1(nibble) * s_b * g)) (the
 * binary32 product, rounded once more to out_dtype).  Nibble 8 gives +0.0.
 *  packed [rows, K/2] (16-byte aligned), block_scales [rows, K/16] E4M3,
 *  global_scale device float (4-byte aligned), out [rows, K] (16-byte
 *  aligned).  Errors as for nvfp4_quantize. */
int nvfp4_dequantize(const void* packed, const void* block_scales, const float* global_scale,
                     int64_t rows, int64_t K, void* out, int out_dtype, void* stream);

/* NVFP4 quantize + pack with block scales chosen by least squared weight
 * error ([MO] "NVFP4's own rules", the mse rule).
 *
 *  Arguments, layout, workspace, errors and the precondition as
 *  nvfp4_quantize; g is the same max|x| / 2688.  Each 16-block tries the
 *  126 positive finite E4M3 codes c (bytes 0x01..0x7E) as its scale: with
 *  d = s_c * g (binary32), every x is cast to E2M1 as nvfp4_quantize casts
 *  it (binary32 quotient x / d), the error (q * d - x) is formed exactly in
 *  double and the squares are summed over the block in column order by
 *  double fmas.  The block keeps the code with the least sum, the smallest
 *  code among equal sums (so an all-zero block takes 0x01), and its codes
 *  are E2M1(x / d) of that code (a zero x gives code 0).  A code whose d
 *  underflows to 0 is not a candidate.  An all-zero tensor gives the
 *  nvfp4_quantize output (g = 0, codes 0, block scales 1.0).
 *  The result is read back with nvfp4_dequantize. */
int nvfp4_quantize_mse(const void* x, int x_dtype, int64_t rows, int64_t K, void* packed,
                       void* block_scales, float* global_scale, void* workspace, void* stream);

/* Size of the library's own static device scratch used by
 * nvfp4_quantize_noalloc (bytes per GPU, held from library load to exit). */
#define MXQ_NOALLOC_SCRATCH_BYTES 256

/* nvfp4_quantize without a workspace argument and without allocating.
 *
 * No counterpart on the source pages: this entry point exists for callers
 * that own all device memory up front and may not allocate while they run,
 * for example an inference engine or a plugin whose memory pool is fixed at
 * start-up, where cudaMalloc would synchronize the device or fail once the
 * pool holds everything.  Such callers still pass inputs and outputs; the
 * 16 bytes of scratch the quantization needs (the tensor-wide maximum) come
 * from a static device array inside libmxq.so instead of a workspace.
 *
 * Arguments, results and errors are those of nvfp4_quantize without the
 * workspace.  The scratch need does not grow with the input (16 bytes for
 * any shape); a build whose need exceeded MXQ_NOALLOC_SCRATCH_BYTES would
 * return MXQ_ERR_UNSUPPORTED.  The first call on each device looks up the
 * array's device address (cudaGetSymbolAddress, with that device current)
 * and keeps it for the life of the process; make that first call before
 * capturing the stream into a graph.  Resetting a device (cudaDeviceReset)
 * after that first call is not supported: the kept address would then be
 * stale.  All calls
 * share the one array: the call clears it before use, and calls that overlap
 * on the GPU (for instance on two streams) race on it and must be
 * serialized by the caller.  Never allocates: no cudaMalloc, cudaFree or
 * allocating library routine is called. */
int nvfp4_quantize_noalloc(const void* x, int x_dtype, int64_t rows, int64_t K, void* packed,
                           void* block_scales, float* global_scale, void* stream);

/* Limit, in nanoseconds, after which a pipeline wait inside the grouped GEMM
 * gives up (the kernel then drains what it issued, frees its tensor memory
 * and reports MXQ_ERR_TIMEOUT through dev_status).  Default 2e9 (2 s); it
 * only ever matters if the GPU stops making progress.  Process-wide; applies
 * to launches made after the call.  Returns the previous limit. */
uint64_t mxq_set_wait_limit_ns(uint64_t ns);

/* Debug variant of the library (libmxq_debug.so, the same sources built
 * with MXQ_DEBUG_CHECKS; no counterpart on the source pages).  There every
 * kernel tests the element index of each global-memory access (and each
 * indexed shared-memory store of the GEMM epilogues and weight decode)
 * against the extent the launch was given; a failed test records the check
 * id, the index and the extent, and the access is skipped, so nothing traps
 * and no out-of-range address is touched.
 *
 * mxq_debug_checks: record (host, int64_t[3]) = {check id, index, extent} of
 *   the first failed check since the previous call, or zeros; the record is
 *   then cleared.  Synchronizes with the device (it copies the records
 *   back).  Returns MXQ_OK in the debug variant, MXQ_ERR_UNSUPPORTED (record
 *   zeroed) in the normal library; null record -> MXQ_ERR_INVALID_ARG.
 * mxq_debug_selftest: launches one checked store one element past the
 *   extent it declares into dev_words (device, two int32, 4-byte aligned;
 *   the store would land in the second word, which the check must leave
 *   untouched), so that the next mxq_debug_checks returns {99, 1, 1}.
 *   MXQ_ERR_UNSUPPORTED (no launch) in the normal library. */
int mxq_debug_checks(int64_t* record);
int mxq_debug_selftest(int32_t* dev_words, void* stream);

/* Human-readable name of a status code (static storage). */
const char* mxq_status_string(int status);

/* ABI version of this header (major * 100 + minor). */
int mxq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MXQ_H */
