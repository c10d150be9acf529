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
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;
std::once_flag g_ctx_once;

void* driver_entry(const char* name) {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
    return fn;
  return nullptr;
}
}  // namespace

uint64_t context_id() {
  std::call_once(g_ctx_once, [] {
    g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(driver_entry("cuCtxGetCurrent"));
    g_ctx_id = reinterpret_cast<CtxGetIdFn>(driver_entry("cuCtxGetId"));
  });
  if (!g_ctx_current || !g_ctx_id) return 0;
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  unsigned long long id = 0;
  if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return static_cast<uint64_t>(id) + 1;
}

namespace {
// One entry per (kernel, context): a context created after a device reset
// starts with default attributes, so it gets an entry of its own.
struct SmemEntry {
  const void* kernel;
  uint64_t ctx;
  size_t bytes;
};
constexpr int kMaxSmemEntries = 256;
SmemEntry g_smem[kMaxSmemEntries];
int g_smem_count = 0;
std::mutex g_smem_mu;
}  // namespace

cudaError_t ensure_smem_raw(const void* kernel, size_t bytes) {
  std::lock_guard<std::mutex> lock(g_smem_mu);
  uint64_t ctx = context_id();
  if (ctx != 0)
    for (int i = 0; i < g_smem_count; ++i)
      if (g_smem[i].kernel == kernel && g_smem[i].ctx == ctx && g_smem[i].bytes >= bytes) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) return e;
  ctx = context_id();  // the call above made the device's context current if it was not yet
  if (ctx == 0) return cudaSuccess;  // no context id available: set the attribute on every call
  for (int i = 0; i < g_smem_count; ++i)
    if (g_smem[i].kernel == kernel && g_smem[i].ctx == ctx) {
      g_smem[i].bytes = bytes;
      return cudaSuccess;
    }
  if (g_smem_count < kMaxSmemEntries) g_smem[g_smem_count++] = SmemEntry{kernel, ctx, bytes};
  return cudaSuccess;
}

namespace {
struct PoolSlot {
  uint64_t ctx;
  cudaMemPool_t pool;
};
constexpr int kPoolDevices = 64;
PoolSlot g_pool[kPoolDevices] = {};
std::mutex g_pool_mu;
}  // namespace

cudaError_t scratch_alloc(void** p, size_t bytes, cudaStream_t s) {
  const int dev = current_device();
  cudaMemPool_t pool = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_pool_mu);
    const uint64_t ctx = context_id();
    const bool cacheable = dev >= 0 && dev < kPoolDevices && ctx != 0;
    if (cacheable && g_pool[dev].ctx == ctx && g_pool[dev].pool) {
      pool = g_pool[dev].pool;
    } else {
      cudaMemPoolProps props = {};
      props.allocType = cudaMemAllocationTypePinned;
      props.location.type = cudaMemLocationTypeDevice;
      props.location.id = dev;
      cudaError_t e = cudaMemPoolCreate(&pool, &props);
      if (e != cudaSuccess) return e;
      uint64_t keep = ~uint64_t{0};  // never trim at synchronisation
      e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
      if (e != cudaSuccess) {
        cudaMemPoolDestroy(pool);
        return e;
      }
      if (cacheable) g_pool[dev] = PoolSlot{ctx, pool};
    }
  }
  return cudaMallocFromPoolAsync(p, bytes, pool, s);
}

namespace {
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiled g_encode = nullptr;
std::once_flag g_encode_once;
}  // namespace

bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t inner, uint64_t rows,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiled>(fn);
  });
  if (!g_encode || inner == 0 || rows == 0) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return g_encode(map, type, 2, const_cast<void*>(base), dims, strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
