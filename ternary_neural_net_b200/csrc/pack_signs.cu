// bnn_pack_signs: float32 rows -> packed sign words.
//
// "Binary Math Effectiveness -- why / how / when", section 1: bit 0 encodes
// +1, bit 1 encodes -1; "Edge cases": inputs <= 0 project to -1, pad bits are
// 0 (+1).  Element e of a row lands in bit (e mod 64) of word e/64.
//
// Design: memory-bound (reads 32 bits, writes 1 bit per element).  One warp
// emits 32 consecutive words of the flattened [rows, kw] output: for each word
// the 32 lanes read 2 x 32 consecutive floats (128-byte coalesced loads) and two
// __ballot_sync calls assemble the 64 bits; lane w keeps word w, so the warp
// finishes with one coalesced 256-byte store.  Loads of 8 words (16 per lane)
// are issued before their ballots to keep enough bytes in flight.
#include "bnn_internal.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 8;  // words whose loads are issued together

__global__ void __launch_bounds__(kThreads)
pack_signs_kernel(const float* __restrict__ x, int64_t k, int64_t kw, int64_t total_words,
                  uint64_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
  for (int64_t base = warp * 32; base < total_words; base += nwarps * 32) {
    // Lane l locates word base+l once; the others fetch it by shuffle.
    const int64_t g = base + lane;
    const int64_t r = g / kw;
    const int64_t e0_own = (g - r * kw) * 64;
    const int64_t rowoff_own = r * k;
    uint64_t mine = 0;
#pragma unroll
    for (int w0 = 0; w0 < 32; w0 += kBatch) {
      float a[kBatch], b[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int64_t e0 = __shfl_sync(0xffffffffu, e0_own, w0 + u);
        const int64_t rowoff = __shfl_sync(0xffffffffu, rowoff_own, w0 + u);
        const bool live = base + w0 + u < total_words;
        const int64_t lim = k - e0;  // logical elements left in this row from e0
        const float* p = x + rowoff + e0;
        // Elements past k read as +1 so that their bit stays 0.
        a[u] = (live && lane < lim) ? __ldg(p + lane) : 1.0f;
        b[u] = (live && lane + 32 < lim) ? __ldg(p + lane + 32) : 1.0f;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const unsigned lo = __ballot_sync(0xffffffffu, !(a[u] > 0.0f));
        const unsigned hi = __ballot_sync(0xffffffffu, !(b[u] > 0.0f));
        if (lane == w0 + u) mine = (static_cast<uint64_t>(hi) << 32) | lo;
      }
    }
    if (g < total_words) out[g] = mine;
  }
}

}  // namespace

extern "C" bnn_status bnn_pack_signs(const float* x, int64_t rows, int64_t k, uint64_t* out,
                                     cudaStream_t s) {
  if (rows < 0 || k < 0) return BNN_ERR_INVALID_ARG;
  if (rows == 0 || k == 0) return BNN_OK;
  if (!x || !out) return BNN_ERR_INVALID_ARG;
  if (!bnn::aligned(x, 4) || !bnn::aligned(out, 8)) return BNN_ERR_MISALIGNED;
  const int64_t kw = bnn::words64(k);
  if (rows > (INT64_MAX / 64) / kw) return BNN_ERR_INVALID_ARG;
  const int64_t total = rows * kw;
  const int64_t warps_needed = (total + 31) / 32;
  const int64_t blocks_needed = (warps_needed + (kThreads / 32) - 1) / (kThreads / 32);
  const int64_t cap = static_cast<int64_t>(bnn::sm_count()) * 8;
  const int grid = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
  pack_signs_kernel<<<grid, kThreads, 0, s>>>(x, k, kw, total, out);
  return bnn::check_launch();
}
