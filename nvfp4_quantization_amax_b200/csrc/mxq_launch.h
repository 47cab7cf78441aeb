// Host-side launcher declarations shared by the ABI layer and the kernel
// translation units.  Arguments reaching these functions are validated.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace mxq {

// Number of SMs of the current device (cached per device).
int num_sms();
// CTAs of `kernel` that fit on one SM at `threads` threads and `smem` bytes
// of dynamic shared memory (occupancy query, cached per kernel and device;
// 1 if the query fails).
int resident_ctas(const void* kernel, int threads, size_t smem);
// Let `kernel` launch with `bytes` of dynamic shared memory on the current
// device (the attribute belongs to the device's context, so it is set once
// per kernel and device; the outcome is cached).
cudaError_t allow_dynamic_smem(const void* kernel, int bytes);
// Grid of a grid-stride streaming kernel: one CTA per per_cta units, at
// most one full wave (SMs x resident CTAs), so that no CTA waits for a
// second wave.
int wave_grid(const void* kernel, int threads, int64_t n_units, int64_t per_cta);

int launch_mx_quantize(const void* x, int dt, int64_t rows, int64_t K, void* packed, void* scales,
                       cudaStream_t st);
int launch_mx_dequantize(const void* packed, const void* scales, int64_t rows, int64_t K, void* out,
                         int dt, cudaStream_t st);
int launch_quantize_cache(const void* in, void* out, int dt, int64_t rows, int64_t C, int fmt,
                          int B, bool fast, cudaStream_t st);
int launch_quantize_cache_packed(const void* in, int dt, int64_t rows, int64_t C, int fmt, int B,
                                 void* codes, void* scales, bool fast, cudaStream_t st);
int launch_dequantize_cache_packed(const void* codes, const void* scales, int64_t rows, int64_t C,
                                   int fmt, int B, void* out, int dt, bool fast, cudaStream_t st);
int launch_nvfp4_quantize(const void* x, int dt, int64_t rows, int64_t K, void* packed,
                          void* block_scales, float* global_scale, uint32_t* amax_word,
                          cudaStream_t st);
// Clear *amax_word, then atomicMax into it the binary32 bits of max |x| over
// n_elems elements (n_elems % 8 == 0; 16-byte aligned x).
void launch_nvfp4_amax(const void* x, int dt, int64_t n_elems, uint32_t* amax_word,
                       cudaStream_t st);
int launch_nvfp4_quantize_mse(const void* x, int dt, int64_t rows, int64_t K, void* packed,
                              void* block_scales, float* global_scale, uint32_t* amax_word,
                              cudaStream_t st);
// Device address of the static scratch of the allocation-free entry point on
// the current device (looked up once per device), or nullptr on failure.
uint32_t* noalloc_scratch(size_t need_bytes, int* status);
int launch_nvfp4_dequantize(const void* packed, const void* block_scales, const float* global_scale,
                            int64_t rows, int64_t K, void* out, int dt, cudaStream_t st);
uint64_t set_wait_limit_ns(uint64_t ns);
uint64_t get_wait_limit_ns();
int launch_nvfp4_w4a4_grouped_mm(const void* xq, const void* xs, const float* xg,
                                 const void* packed, const void* scales, const float* wg,
                                 const int32_t* offs, int64_t T, int64_t E, int64_t N, int64_t K,
                                 void* y, int32_t* dev_status, uint64_t wait_limit_ns,
                                 cudaStream_t st);
int launch_w4a4_grouped_mm(const void* xq, const void* xs, const void* packed, const void* scales,
                           const int32_t* offs, int64_t T, int64_t E, int64_t N, int64_t K,
                           void* y, int32_t* dev_status, uint64_t wait_limit_ns, cudaStream_t st);
// Readers of each translation unit's debug check record (copy to out[3]
// and clear; MXQ_ERR_UNSUPPORTED in the normal build).
int check_record_elementwise(unsigned long long* out);
int check_record_cache_packed(unsigned long long* out);
int check_record_nvfp4(unsigned long long* out);
int check_record_nvfp4_mse(unsigned long long* out);
int check_record_grouped_mm_general(unsigned long long* out);
int check_record_grouped_mm_tc(unsigned long long* out);
int check_record_w4a4(unsigned long long* out);
int launch_grouped_mm(const void* a, const void* packed, const void* scales, const int32_t* offs,
                      int64_t T, int64_t E, int64_t N, int64_t K, int transpose_w, void* y,
                      int32_t* dev_status, cudaStream_t st);

}  // namespace mxq
