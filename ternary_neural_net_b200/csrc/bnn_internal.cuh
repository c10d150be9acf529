// Internal helpers shared by the libbnn CUDA sources (not part of the ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "bnn.h"

namespace bnn {

// Records a failed CUDA call for bnn_last_cuda_error() and maps it to a status.
bnn_status cuda_fail(cudaError_t e);

inline bnn_status check_launch() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BNN_OK : cuda_fail(e);
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

__host__ __device__ inline int64_t words64(int64_t k) { return (k + 63) / 64; }
__host__ __device__ inline int64_t words10(int64_t k) { return (k + 9) / 10; }

// Number of SMs of the current device (cached per device).
int sm_count();

// Current device index (0 if the query fails).
int current_device();

// Raises a kernel's dynamic shared-memory limit to `bytes` once per kernel,
// device and process, so that later calls (including calls made while a
// stream is being captured into a CUDA graph) only launch.
cudaError_t ensure_smem_raw(const void* kernel, size_t bytes);

template <typename Kernel>
cudaError_t ensure_smem(Kernel kern, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return ensure_smem_raw(reinterpret_cast<const void*>(kern), bytes);
}

}  // namespace bnn

#define BNN_TRY(expr)                              \
  do {                                             \
    cudaError_t bnn_e_ = (expr);                   \
    if (bnn_e_ != cudaSuccess) return bnn::cuda_fail(bnn_e_); \
  } while (0)
