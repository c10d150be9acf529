// Index + sign sparse ternary layers: encode the base-3 packed weights into
// per-row lists of non-zero positions and run the layer over those lists.
//
// "BalancedTernaryEngine" README, "Features" (sparse encoding: an index + sign
// format for high-sparsity layers) and "Module Overview" (Packer.pack_sparse).
// Format: row j's entries are entries[row_ptr[j] .. row_ptr[j+1]), one 16-bit
// entry per non-zero trit in increasing position order, the position in bits
// 0..14 and bit 15 set for -1.
//
// Design: every kernel gives one warp to one weight row.
//   - count: the lanes walk the row's packed words, take each word's ten
//     base-3 digits with the fixed-point fraction (__umulhi by 3), count the
//     digits that are not 1 (trit != 0) at positions < k and add the counts
//     across the warp; a single-CTA scan then turns the counts into row_ptr.
//   - encode: per 32 words, each lane builds the non-zero and negative masks of
//     its word, a warp prefix sum of the mask popcounts gives each lane its
//     first slot, and the lane writes its entries in position order.
//   - layer: the lanes stride over the row's entries (64-byte coalesced
//     loads), gather x at each position and add or subtract it in float32;
//     the warp sum is scaled (and biased) once.  At m = 1, x is staged in
//     shared memory as float32 and the next row's entries load while this
//     row's are gathered; for m > 1 the gathers read bf16 x through L1.
//     Launched with programmatic dependent launch: the row's first entries
//     are read before waiting for the kernel that produced x.
#include "bnn_internal.cuh"

namespace {

constexpr uint32_t kFix = 72736u;  // ceil(2^32 / 3^10)
constexpr int kWarpsPerBlock = 8;

// masks of the non-zero and the negative trits of one packed word (bit i = trit
// 10j + i), restricted to positions < k
__device__ __forceinline__ void word_masks(uint32_t w, int64_t pos0, int64_t k, uint32_t& nz, uint32_t& neg) {
  uint32_t F = w * kFix;
  nz = 0;
  neg = 0;
#pragma unroll
  for (int s = 0; s < 10; ++s) {
    const uint32_t d = __umulhi(F, 3u);  // most significant remaining digit: trit 9 - s
    F *= 3u;
    const int i = 9 - s;
    if (d != 1u) nz |= 1u << i;
    if (d == 0u) neg |= 1u << i;
  }
  const int64_t left = k - pos0;
  if (left < 10) {
    const uint32_t keep = left <= 0 ? 0u : ((1u << left) - 1u);
    nz &= keep;
    neg &= keep;
  }
}

__global__ void __launch_bounds__(kWarpsPerBlock * 32)
sparse_count_kernel(const uint16_t* __restrict__ packed, int64_t n, int64_t k, int64_t kt,
                    int64_t* __restrict__ row_ptr) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  if (blockIdx.x == 0 && threadIdx.x == 0) row_ptr[0] = 0;
  for (int64_t r = warp; r < n; r += nwarps) {
    int c = 0;
    for (int64_t j = lane; j < kt; j += 32) {
      uint32_t nz, neg;
      word_masks(__ldg(packed + r * kt + j), 10 * j, k, nz, neg);
      c += __popc(nz);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
    if (lane == 0) row_ptr[r + 1] = c;
  }
}

// In-place inclusive scan of row_ptr[1 .. n] by one CTA of kScanThreads threads:
// each thread sums a contiguous chunk, the chunk sums are scanned, and every
// chunk is rewritten with its running prefix.
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) sparse_scan_kernel(int64_t* __restrict__ row_ptr, int64_t n) {
  __shared__ int64_t warp_sums[kScanThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t chunk = (n + kScanThreads - 1) / kScanThreads;
  const int64_t b = 1 + tid * chunk, e = b + chunk < n + 1 ? b + chunk : n + 1;
  int64_t local = 0;
  for (int64_t i = b; i < e; ++i) local += row_ptr[i];
  // inclusive scan of the thread sums: within the warp, then across warps
  int64_t incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int64_t v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int64_t w = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int64_t v = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += v;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  int64_t run = incl - local + (warp > 0 ? warp_sums[warp - 1] : 0);
  for (int64_t i = b; i < e; ++i) {
    run += row_ptr[i];
    row_ptr[i] = run;
  }
}

__global__ void __launch_bounds__(kWarpsPerBlock * 32)
sparse_encode_kernel(const uint16_t* __restrict__ packed, int64_t n, int64_t k, int64_t kt,
                     const int64_t* __restrict__ row_ptr, uint16_t* __restrict__ entries) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = warp; r < n; r += nwarps) {
    int64_t base = row_ptr[r];
    const int64_t row_end = row_ptr[r + 1];  // entries past it are never written
    for (int64_t j0 = 0; j0 < kt; j0 += 32) {
      const int64_t j = j0 + lane;
      uint32_t nz = 0, neg = 0;
      if (j < kt) word_masks(__ldg(packed + r * kt + j), 10 * j, k, nz, neg);
      const int cnt = __popc(nz);
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      int64_t at = base + (incl - cnt);
      while (nz) {
        const int i = __ffs(nz) - 1;  // lowest remaining position first
        nz &= nz - 1;
        if (at < row_end) entries[at] = static_cast<uint16_t>((10 * j + i) | (((neg >> i) & 1u) << 15));
        ++at;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
}

template <int MT>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
sparse_gemm_kernel(const uint16_t* __restrict__ x, const int64_t* __restrict__ row_ptr,
                   const uint16_t* __restrict__ entries, const float* __restrict__ scale,
                   const float* __restrict__ bias, int64_t m, int64_t n, int64_t k, float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  bnn::pdl_trigger();
  bool waited = false;
  for (int64_t r = warp; r < n; r += nwarps) {
    const int64_t b = row_ptr[r], e = row_ptr[r + 1];
    for (int64_t t0 = 0; t0 < m; t0 += MT) {
      float acc[MT];
#pragma unroll
      for (int t = 0; t < MT; ++t) acc[t] = 0.0f;
      for (int64_t q0 = b; q0 < e; q0 += 4 * 32) {
        // four entries per lane in flight before the gathers
        uint32_t ent[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int64_t q = q0 + u * 32 + lane;
          ent[u] = q < e ? static_cast<uint32_t>(__ldg(entries + q)) : 0xFFFFFFFFu;
        }
        if (!waited) {
          bnn::pdl_wait();  // x may come from the preceding kernel
          waited = true;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int64_t pos = ent[u] & 0x7FFFu;
          if (ent[u] != 0xFFFFFFFFu && pos < k) {  // positions >= k are malformed: skipped
            const bool minus = (ent[u] >> 15) != 0u;
#pragma unroll
            for (int t = 0; t < MT; ++t) {
              if (t0 + t < m) {
                const float v = __uint_as_float(static_cast<uint32_t>(__ldg(x + (t0 + t) * k + pos)) << 16);
                acc[t] += minus ? -v : v;
              }
            }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < MT; ++t)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], off);
      if (!waited) {
        bnn::pdl_wait();  // the outputs are written after the preceding kernel
        waited = true;
      }
      if (lane == 0) {
        const float sc = __ldg(scale + r), bv = bias ? __ldg(bias + r) : 0.0f;
#pragma unroll
        for (int t = 0; t < MT; ++t)
          if (t0 + t < m) out[(t0 + t) * n + r] = bias ? sc * acc[t] + bv : sc * acc[t];
      }
    }
  }
}

// The layer at m = 1: x staged once per CTA in shared memory as float32 (k
// floats, k <= 32768), so every gather is a shared-memory load.  Two CTAs of
// 512 threads per SM (one where k leaves room for only one) each take a
// contiguous block of rows, in chunks of kSpChunk = 48: the chunk's row_ptr
// values are read into shared memory once, and warp w takes rows w, w + 16
// and w + 32 of it.  (With two CTAs per SM, the next launch's CTAs start
// their row_ptr and entry loads while this launch's last CTAs finish: 5.8
// against 6.2 µs for one 1024-thread CTA per SM at 11008 x 4096, 10% of the
// trits non-zero; four 256-thread CTAs lost on long rows.)  A warp issues the loads of all its rows' first
// 511..512 entries at once, before the programmatic-launch wait and the
// staging of x (each lane eight 32-bit entry pairs per row, 128-byte coalesced
// loads from the even entry at or below the row's first), so the whole
// chunk's entries are in flight together.  A pair's halves outside the row
// contribute nothing (the gathered value is masked in the same logic op that
// applies the sign).  Longer rows take further passes of 512 entries.  The
// row's sum is added by a shuffle tree (a fixed order), scaled once (and
// biased).  VEC: entries 4-byte aligned (one 32-bit load per pair), else two
// 16-bit loads.
constexpr int kSpThreads = 512;
constexpr int kSpWarps = kSpThreads / 32;
constexpr int kSpPerSm = 2;                     // CTAs per SM (register budget: 64 per thread)
constexpr int kSpR = 3;                         // rows per warp and chunk
constexpr int kSpChunk = kSpWarps * kSpR;
static_assert(kSpChunk + 1 <= kSpThreads, "one thread per row_ptr value of a chunk");
constexpr int kSpW = 8;                         // entry pairs per lane per pass

// entries q, q + 1 (bits 0..15 and 16..31; q even relative to the row's pass
// start); entries at or past e are not read (their halves are masked off, and
// e may be the end of the array)
template <bool VEC>
__device__ __forceinline__ uint32_t sp_pair(const uint16_t* __restrict__ entries, int64_t q, int64_t e) {
  if (q >= e) return 0u;
  if (VEC && q + 1 < e) return __ldcs(reinterpret_cast<const uint32_t*>(entries + q));
  const uint32_t lo = __ldcs(entries + q);
  return q + 1 < e ? lo | (static_cast<uint32_t>(__ldcs(entries + q + 1)) << 16) : lo;
}

// the contributions of one pass of a row: pairs v[i] hold entries a + 2 (32 i
// + lane) and the one after; only those in [b, e) count (offsets within the
// pass are 32-bit: 0 <= max(b - a, 0) and min(e - a, 64 W) <= 64 W)
template <int W>
__device__ __forceinline__ float sp_gather(const float* xs, const uint32_t (&v)[W], int64_t a, int64_t b, int64_t e,
                                           int lane, uint32_t kk) {
  const int lo = b > a ? static_cast<int>(b - a) : 0;
  const int hi = e - a < 64 * W ? static_cast<int>(e - a) : 64 * W;
  const int span = hi > lo ? hi - lo : 0;  // entries of the row in this pass
  const int base = 2 * lane - lo;    // offset of pair 0's first entry from the row's first in the pass
  float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
  for (int i = 0; i < W; ++i) {
    const uint32_t d = static_cast<uint32_t>(base + 64 * i);
    const uint32_t p0 = min(v[i] & 0x7FFFu, kk), p1 = min((v[i] >> 16) & 0x7FFFu, kk);  // >= k: the zero slot
    const float t0 = __uint_as_float(__float_as_uint(xs[p0]) ^ ((v[i] << 16) & 0x80000000u));  // sign: bit 15
    const float t1 = __uint_as_float(__float_as_uint(xs[p1]) ^ (v[i] & 0x80000000u));          // sign: bit 31
    if (d < static_cast<uint32_t>(span)) acc0 += t0;
    if (d + 1u < static_cast<uint32_t>(span)) acc1 += t1;
  }
  return acc0 + acc1;
}

template <bool VEC>
__global__ void __launch_bounds__(kSpThreads, kSpPerSm)
sparse_gemv_smem_kernel(const uint16_t* __restrict__ x, const int64_t* __restrict__ row_ptr,
                        const uint16_t* __restrict__ entries, const float* __restrict__ scale,
                        const float* __restrict__ bias, int64_t n, int k, float* __restrict__ out) {
  extern __shared__ float xs[];  // [k + 1]: x as float32, then xs[k] = 0
  __shared__ int64_t rp[kSpChunk + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t r_begin = n * blockIdx.x / gridDim.x, r_end = n * (blockIdx.x + 1) / gridDim.x;
  const uint32_t kk = static_cast<uint32_t>(k);
  bnn::pdl_trigger();
  bool staged = false;
  for (int64_t cb = r_begin; cb < r_end; cb += kSpChunk) {
    const int rows = static_cast<int>(r_end - cb < kSpChunk ? r_end - cb : kSpChunk);
    if (tid <= rows) rp[tid] = row_ptr[cb + tid];
    __syncthreads();
    // every row's first pass, in flight together
    uint32_t v[kSpR][kSpW];
#pragma unroll
    for (int j = 0; j < kSpR; ++j) {
      const int rl = warp + kSpWarps * j;
      const int64_t b = rl < rows ? rp[rl] : 0, e = rl < rows ? rp[rl + 1] : 0;
      const int64_t a = b & ~int64_t{1};
#pragma unroll
      for (int i = 0; i < kSpW; ++i) v[j][i] = sp_pair<VEC>(entries, a + 2 * (32 * i + lane), e);
    }
    if (!staged) {
      bnn::pdl_wait();  // x may come from the kernel ahead
      for (int i = tid; i < k; i += kSpThreads) xs[i] = __uint_as_float(static_cast<uint32_t>(__ldg(x + i)) << 16);
      if (tid == 0) xs[k] = 0.0f;
      __syncthreads();
      staged = true;
    }
#pragma unroll
    for (int j = 0; j < kSpR; ++j) {
      const int rl = warp + kSpWarps * j;
      if (rl >= rows) break;
      const int64_t b = rp[rl], e = rp[rl + 1];
      int64_t a = b & ~int64_t{1};
      float sum = sp_gather<kSpW>(xs, v[j], a, b, e, lane, kk);
      for (a += 64 * kSpW; a < e; a += 64 * kSpW) {  // rows of more than one pass
        uint32_t w[kSpW];
#pragma unroll
        for (int i = 0; i < kSpW; ++i) w[i] = sp_pair<VEC>(entries, a + 2 * (32 * i + lane), e);
        sum += sp_gather<kSpW>(xs, w, a, b, e, lane, kk);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      const int64_t r = cb + rl;
      if (lane == 0) out[r] = bias ? __ldg(scale + r) * sum + __ldg(bias + r) : __ldg(scale + r) * sum;
    }
    __syncthreads();  // rp is refilled by the next chunk
  }
}

int warp_grid(int64_t rows) {
  const int64_t need = (rows + kWarpsPerBlock - 1) / kWarpsPerBlock;
  const int64_t cap = static_cast<int64_t>(bnn::sm_count()) * 8;
  return static_cast<int>(need < cap ? (need > 0 ? need : 1) : cap);
}

}  // namespace

extern "C" bnn_status bnn_ternary_sparse_count(const uint16_t* packed, int64_t n, int64_t k, int64_t* row_ptr,
                                               cudaStream_t s) {
  if (n < 0 || k < 0 || k > BNN_MAX_K_SPARSE || !row_ptr) return BNN_ERR_INVALID_ARG;
  if (n > 0 && k > 0 && !packed) return BNN_ERR_INVALID_ARG;
  if ((packed && !bnn::aligned(packed, 2)) || !bnn::aligned(row_ptr, 8)) return BNN_ERR_MISALIGNED;
  if (n == 0 || k == 0) {
    BNN_TRY(cudaMemsetAsync(row_ptr, 0, static_cast<size_t>(n + 1) * sizeof(int64_t), s));
    return BNN_OK;
  }
  const int64_t kt = bnn::words10(k);
  sparse_count_kernel<<<warp_grid(n), kWarpsPerBlock * 32, 0, s>>>(packed, n, k, kt, row_ptr);
  BNN_TRY(cudaGetLastError());
  sparse_scan_kernel<<<1, kScanThreads, 0, s>>>(row_ptr, n);
  return bnn::check_launch();
}

extern "C" bnn_status bnn_ternary_sparse_encode(const uint16_t* packed, int64_t n, int64_t k, const int64_t* row_ptr,
                                                uint16_t* entries, cudaStream_t s) {
  if (n < 0 || k < 0 || k > BNN_MAX_K_SPARSE || !row_ptr) return BNN_ERR_INVALID_ARG;
  if (n == 0 || k == 0) return BNN_OK;
  if (!packed || !entries) return BNN_ERR_INVALID_ARG;
  if (!bnn::aligned(packed, 2) || !bnn::aligned(row_ptr, 8) || !bnn::aligned(entries, 2)) return BNN_ERR_MISALIGNED;
  sparse_encode_kernel<<<warp_grid(n), kWarpsPerBlock * 32, 0, s>>>(packed, n, k, bnn::words10(k), row_ptr, entries);
  return bnn::check_launch();
}

extern "C" bnn_status bnn_ternary_sparse_gemm(const uint16_t* x_bf16, const int64_t* row_ptr,
                                              const uint16_t* entries, const float* scale, const float* bias,
                                              int64_t m, int64_t n, int64_t k, float* out, cudaStream_t s) {
  if (m < 0 || n < 0 || k < 0 || k > BNN_MAX_K_SPARSE) return BNN_ERR_INVALID_ARG;
  if (m == 0 || n == 0) return BNN_OK;
  if (!row_ptr || !scale || !out || (k > 0 && !x_bf16)) return BNN_ERR_INVALID_ARG;
  if ((x_bf16 && !bnn::aligned(x_bf16, 2)) || !bnn::aligned(row_ptr, 8) || (entries && !bnn::aligned(entries, 2)) ||
      !bnn::aligned(scale, 4) || (bias && !bnn::aligned(bias, 4)) || !bnn::aligned(out, 4))
    return BNN_ERR_MISALIGNED;
  if (m == 1 && k > 0) {
    const size_t smem = static_cast<size_t>(k + 1) * sizeof(float);
    // two CTAs per SM where their x copies fit one SM's shared memory together
    const int per_sm = 2 * (smem + 2048) <= 228u * 1024u ? kSpPerSm : 1;
    const int64_t slots = bnn::sm_count() * static_cast<int64_t>(per_sm);
    const int grid = static_cast<int>(n < slots ? n : slots);
    if (entries && bnn::aligned(entries, 4)) {
      BNN_TRY(bnn::ensure_smem(sparse_gemv_smem_kernel<true>, smem));
      BNN_TRY(bnn::launch_pdl(sparse_gemv_smem_kernel<true>, dim3(grid), dim3(kSpThreads), smem, s, 1, x_bf16,
                              row_ptr, entries, scale, bias, n, static_cast<int>(k), out));
    } else {
      BNN_TRY(bnn::ensure_smem(sparse_gemv_smem_kernel<false>, smem));
      BNN_TRY(bnn::launch_pdl(sparse_gemv_smem_kernel<false>, dim3(grid), dim3(kSpThreads), smem, s, 1, x_bf16,
                              row_ptr, entries, scale, bias, n, static_cast<int>(k), out));
    }
    return bnn::check_launch();
  }
  const dim3 grid(warp_grid(n)), block(kWarpsPerBlock * 32);
  cudaError_t e;
  if (m == 1)
    e = bnn::launch_pdl(sparse_gemm_kernel<1>, grid, block, 0, s, 1, x_bf16, row_ptr, entries, scale, bias, m, n, k,
                        out);
  else if (m <= 4)
    e = bnn::launch_pdl(sparse_gemm_kernel<4>, grid, block, 0, s, 1, x_bf16, row_ptr, entries, scale, bias, m, n, k,
                        out);
  else
    e = bnn::launch_pdl(sparse_gemm_kernel<8>, grid, block, 0, s, 1, x_bf16, row_ptr, entries, scale, bias, m, n, k,
                        out);
  if (e != cudaSuccess) return bnn::cuda_fail(e);
  return bnn::check_launch();
}
