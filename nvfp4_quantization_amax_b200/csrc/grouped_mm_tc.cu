// Grouped GEMM dispatch (tensor-core kernel to follow).
#include "mxq.h"
#include "mxq_launch.h"

namespace mxq {

int launch_grouped_mm_general(const void* a, const void* packed, const void* scales,
                              const int32_t* offs, int64_t T, int64_t E, int64_t N, int64_t K,
                              int transpose_w, void* y, int32_t* dev_status, cudaStream_t st);

int launch_grouped_mm(const void* a, const void* packed, const void* scales, const int32_t* offs,
                      int64_t T, int64_t E, int64_t N, int64_t K, int transpose_w, void* y,
                      int32_t* dev_status, cudaStream_t st) {
  return launch_grouped_mm_general(a, packed, scales, offs, T, E, N, K, transpose_w, y,
                                   dev_status, st);
}

}  // namespace mxq
