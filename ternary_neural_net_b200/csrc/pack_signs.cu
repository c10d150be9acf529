// bnn_pack_signs: float32 rows -> packed sign words.
//
// "Binary Math Effectiveness -- why / how / when", section 1: bit 0 encodes
// +1, bit 1 encodes -1; "Edge cases": inputs <= 0 project to -1, pad bits are
// 0 (+1).  Element e of a row lands in bit (e mod 64) of word e/64.
//
// Design: memory-bound (reads 32 bits, writes 1 bit per element).  A warp
// owns kWords consecutive words of one row at a time (a "unit"); units are
// numbered row-major and handed out grid-stride to a grid of a few CTAs per
// SM, so CTAs live long enough to keep many loads in flight.  For each word
// the 32 lanes read 2 x 32 consecutive floats (128-byte coalesced loads), the
// 2*kWords loads of two units are issued before any ballot, and two
// __ballot_sync calls assemble each 64-bit word; lane u < kWords stores word u.
#include "bnn_internal.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kWords = 4;    // words per unit
constexpr int kUnroll = 2;   // units whose loads are issued together

__global__ void __launch_bounds__(kThreads)
pack_signs_kernel(const float* __restrict__ x, int64_t k, int64_t kw, int64_t units_per_row, int64_t units,
                  uint64_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
  bnn::pdl_trigger();  // a matmul launched after this kernel may start its weight copies now
  for (int64_t u0 = warp; u0 < units; u0 += nwarps * kUnroll) {
    float a[kUnroll][kWords], b[kUnroll][kWords];
    int64_t row[kUnroll], j0[kUnroll];
#pragma unroll
    for (int q = 0; q < kUnroll; ++q) {
      const int64_t unit = u0 + q * nwarps;
      const bool live = unit < units;
      row[q] = live ? unit / units_per_row : 0;
      j0[q] = live ? (unit - row[q] * units_per_row) * kWords : kw;  // a dead unit covers no word
      const float* xr = x + row[q] * k;
#pragma unroll
      for (int u = 0; u < kWords; ++u) {
        const int64_t e0 = (j0[q] + u) * 64;
        // Elements past k (and words past kw) read as +1 so that their bit stays 0.
        a[q][u] = e0 + lane < k ? __ldcs(xr + e0 + lane) : 1.0f;
        b[q][u] = e0 + lane + 32 < k ? __ldcs(xr + e0 + lane + 32) : 1.0f;
      }
    }
#pragma unroll
    for (int q = 0; q < kUnroll; ++q) {
      uint64_t mine = 0;
#pragma unroll
      for (int u = 0; u < kWords; ++u) {
        const unsigned lo = __ballot_sync(0xffffffffu, !(a[q][u] > 0.0f));
        const unsigned hi = __ballot_sync(0xffffffffu, !(b[q][u] > 0.0f));
        if (lane == u) mine = (static_cast<uint64_t>(hi) << 32) | lo;
      }
      if (lane < kWords && j0[q] + lane < kw) out[row[q] * kw + j0[q] + lane] = mine;
    }
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
  const int64_t units_per_row = (kw + kWords - 1) / kWords;
  const int64_t units = rows * units_per_row;
  const int64_t warps_per_block = kThreads / 32;
  const int64_t blocks_needed = (units + warps_per_block * kUnroll - 1) / (warps_per_block * kUnroll);
  const int64_t cap = static_cast<int64_t>(bnn::sm_count()) * 8;
  const int grid = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
  pack_signs_kernel<<<grid, kThreads, 0, s>>>(x, k, kw, units_per_row, units, out);
  return bnn::check_launch();
}
