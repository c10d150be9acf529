// Internal helpers shared by the libbnn CUDA sources (not part of the ABI).
#pragma once

#include <cstdint>
#include <cuda.h>  // CUtensorMap and its enums (the encoder is fetched from the driver at run time)
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

// A unique non-zero id of the calling thread's current CUDA context (driver
// cuCtxGetId), 0 when there is none or the driver cannot say.  Per-context
// caches key on it: a device reset destroys the primary context, and the
// next one gets a new id, so nothing cached for the old one is reused.
uint64_t context_id();

// Stream-ordered scratch memory from a pool of this library (one per device
// and CUDA context) that keeps its memory between calls, where the default
// pool would hand it back to the driver at each synchronisation and map it
// again on the next call.  Free with cudaFreeAsync on the same stream.
cudaError_t scratch_alloc(void** p, size_t bytes, cudaStream_t s);

// Raises a kernel's dynamic shared-memory limit to `bytes` once per kernel
// and CUDA context, so that later calls (including calls made while a
// stream is being captured into a CUDA graph) only launch.
cudaError_t ensure_smem_raw(const void* kernel, size_t bytes);

template <typename Kernel>
cudaError_t ensure_smem(Kernel kern, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return ensure_smem_raw(reinterpret_cast<const void*>(kern), bytes);
}

// Fills a 2-D TMA descriptor for a row-major matrix of `rows` rows of `inner`
// elements, rows `row_bytes` apart, copied in boxes of box_inner x box_rows
// elements with the given shared-memory swizzle; elements outside the matrix
// read as zero.  False when the driver rejects it (alignment, sizes) or the
// encoder is unavailable.
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t inner, uint64_t rows,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle);

// Programmatic dependent launch.  A kernel launched with launch_pdl may start
// while the preceding kernel on the stream is still running; it must call
// pdl_wait() before it reads anything that kernel writes and before its own
// first global store.  pdl_trigger() lets the next such kernel start early (a
// no-op when the next kernel was launched normally).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, unsigned cluster_x,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster_x > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// Tensor-core (tcgen05 kind::mxf4) binary GEMM, in binary_gemm_tc.cu, with the
// optional layer epilogue: bias (may be null) and the sign-packed output for
// the next layer (next, may be null; ceil(n/64) words per row).
bnn_status binary_gemm_tc(const uint64_t* xp, const uint64_t* wp, const float* alpha, const float* bias, int64_t m,
                          int64_t n, int k, int kw, int32_t* dots, float* out, uint64_t* next, cudaStream_t s);

// Device address of the counter of bounded device-side waits that ran out
// (the one bnn_device_error_count reads), looked up once per CUDA context;
// nullptr when the lookup fails.
unsigned int* device_error_counter();

// Bounded waits that ran out in the ternary tensor-core kernel (reset != 0 clears).
int ternary_tc_error_count(int reset);

// Tensor-core (tcgen05 kind::f16) ternary GEMM, in ternary_gemm_tc.cu.
// Plan of the ternary kernel that decodes into tensor memory (one activation
// tile): rows of weights per CTA (32, 64, 96 or 128) and CTAs per cluster
// splitting the stages (1..4), for n weight rows of k trits (ceil(k / 256)
// stages), given how many clusters of each size fit the GPU at once
// (active[ks - 1]; 0 = unusable).  Host only.
void ternary_tmem_plan(int64_t n, int64_t k, const int active[4], int* rows, int* ks);
bnn_status ternary_gemm_tc(const uint16_t* x_bf16, const uint16_t* packed, const float* scale, const float* bias,
                           int64_t m, int64_t n, int64_t k, float* out, cudaStream_t s);

}  // namespace bnn

#define BNN_TRY(expr)                              \
  do {                                             \
    cudaError_t bnn_e_ = (expr);                   \
    if (bnn_e_ != cudaSuccess) return bnn::cuda_fail(bnn_e_); \
  } while (0)
