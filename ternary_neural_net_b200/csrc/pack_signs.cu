// bnn_pack_signs: float32 rows -> packed sign words.
//
// "Binary Math Effectiveness -- why / how / when", section 1: bit 0 encodes
// +1, bit 1 encodes -1; "Edge cases": inputs <= 0 project to -1, pad bits are
// 0 (+1).  Element e of a row lands in bit (e mod 64) of word e/64.
//
// Design: memory-bound (reads 32 bits, writes 1 bit per element).  The grid is
// 2-D: blockIdx.y walks rows, blockIdx.x covers kBlockWords consecutive words
// of a row, so no thread divides to find its row.  One warp emits kWords
// words: for each word the 32 lanes read 2 x 32 consecutive floats (128-byte
// coalesced loads), all 2*kWords loads of a lane are issued before any ballot,
// and two __ballot_sync calls assemble each 64-bit word; lane u < kWords
// stores word u (one 32-byte coalesced store).
#include "bnn_internal.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kWords = 4;                                  // words per warp
constexpr int kBlockWords = kWords * (kThreads / 32);      // words per block

__global__ void __launch_bounds__(kThreads)
pack_signs_kernel(const float* __restrict__ x, int64_t rows, int64_t k, int64_t kw,
                  uint64_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t j0 = static_cast<int64_t>(blockIdx.x) * kBlockWords + (threadIdx.x >> 5) * kWords;
  for (int64_t r = blockIdx.y; r < rows; r += gridDim.y) {
    const float* row = x + r * k;
    float a[kWords], b[kWords];
#pragma unroll
    for (int u = 0; u < kWords; ++u) {
      const int64_t e0 = (j0 + u) * 64;
      // Elements past k (and whole words past kw) read as +1 so that their bit stays 0.
      a[u] = e0 + lane < k ? __ldcs(row + e0 + lane) : 1.0f;
      b[u] = e0 + lane + 32 < k ? __ldcs(row + e0 + lane + 32) : 1.0f;
    }
    uint64_t mine = 0;
#pragma unroll
    for (int u = 0; u < kWords; ++u) {
      const unsigned lo = __ballot_sync(0xffffffffu, !(a[u] > 0.0f));
      const unsigned hi = __ballot_sync(0xffffffffu, !(b[u] > 0.0f));
      if (lane == u) mine = (static_cast<uint64_t>(hi) << 32) | lo;
    }
    if (lane < kWords && j0 + lane < kw) out[r * kw + j0 + lane] = mine;
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
  const int64_t gx = (kw + kBlockWords - 1) / kBlockWords;
  if (gx > 2147483647LL) return BNN_ERR_INVALID_ARG;
  const int64_t gy = rows < 65535 ? rows : 65535;
  pack_signs_kernel<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), kThreads, 0, s>>>(x, rows, k, kw,
                                                                                                     out);
  return bnn::check_launch();
}
