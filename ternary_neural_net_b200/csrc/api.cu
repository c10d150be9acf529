// Status strings, error bookkeeping and device queries for libbnn.
#include <mutex>

#include "bnn_internal.cuh"

namespace {
thread_local int g_last_cuda_error = 0;
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {0};
}  // namespace

namespace bnn {

bnn_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return BNN_ERR_CUDA;
}

namespace {
struct SmemEntry {
  const void* kernel;
  int device;
  size_t bytes;
};
constexpr int kMaxSmemEntries = 256;
SmemEntry g_smem[kMaxSmemEntries];
int g_smem_count = 0;
std::mutex g_smem_mu;
}  // namespace

cudaError_t ensure_smem_raw(const void* kernel, size_t bytes) {
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(g_smem_mu);
  for (int i = 0; i < g_smem_count; ++i)
    if (g_smem[i].kernel == kernel && g_smem[i].device == dev && g_smem[i].bytes >= bytes) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) return e;
  for (int i = 0; i < g_smem_count; ++i)
    if (g_smem[i].kernel == kernel && g_smem[i].device == dev) {
      g_smem[i].bytes = bytes;
      return cudaSuccess;
    }
  if (g_smem_count < kMaxSmemEntries) g_smem[g_smem_count++] = SmemEntry{kernel, dev, bytes};
  return cudaSuccess;
}

int current_device() {
  int dev = 0;
  return cudaGetDevice(&dev) == cudaSuccess ? dev : 0;
}

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (g_sm_count[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    g_sm_count[dev] = v;
  }
  return g_sm_count[dev];
}

}  // namespace bnn

extern "C" const char* bnn_status_string(bnn_status st) {
  switch (st) {
    case BNN_OK: return "BNN_OK";
    case BNN_ERR_INVALID_ARG: return "BNN_ERR_INVALID_ARG: a size is out of range or a required pointer is NULL";
    case BNN_ERR_MISALIGNED: return "BNN_ERR_MISALIGNED: a pointer is not aligned to its element size";
    case BNN_ERR_CUDA: return "BNN_ERR_CUDA: a CUDA call or kernel launch failed (see bnn_last_cuda_error)";
    case BNN_ERR_UNSUPPORTED: return "BNN_ERR_UNSUPPORTED: the device or the request is not supported";
  }
  return "BNN_ERR_UNKNOWN";
}

extern "C" int bnn_last_cuda_error(void) { return g_last_cuda_error; }
