// Balanced ternary: TWN ternarisation + base-3 packing, and the ternary matmul.
//
// "BalancedTernaryEngine" README, section "Features": TWN threshold
// Delta = 0.7 * mean|W|, least-squares per-channel scale, 10 trits per 16-bit
// word in base 3; "Module Overview": Layer.forward (activations times trits,
// times the channel scale).
//
// Base-3 word j of a row holds trits 10j..10j+9 with digit (trit + 1) at weight
// 3^i.  Decoding uses one fixed-point multiply instead of ten divisions: with
// F = w * ceil(2^32 / 3^10) (fits in 32 bits for w < 3^10), F / 2^32 lies in
// [w / 3^10, w / 3^10 + 1/3^10), so repeatedly taking the high word of 3F
// yields the digits most significant first, exactly, for every valid word
// (base 9 works the same way with 9F, giving trit pairs).
#include <cuda_bf16.h>

#include <mutex>

#include "bnn_internal.cuh"

namespace {

constexpr uint32_t kFixMul = 72736u;  // ceil(2^32 / 3^10)

// ---------------------------------------------------------------------------
// Ternarisation + packing
// ---------------------------------------------------------------------------
constexpr int kRedThreads = 256;
constexpr int64_t kChunk = 65536;  // weights per partial sum

// Fixed-order block reduction of a double (deterministic for a given blockDim).
__device__ double block_sum_f64(double v, double* sh) {
  const int tid = threadIdx.x;
  sh[tid] = v;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (tid < s) sh[tid] += sh[tid + s];
    __syncthreads();
  }
  const double r = sh[0];
  __syncthreads();
  return r;
}

__device__ long long block_sum_i64(long long v, long long* sh) {
  const int tid = threadIdx.x;
  sh[tid] = v;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (tid < s) sh[tid] += sh[tid + s];
    __syncthreads();
  }
  const long long r = sh[0];
  __syncthreads();
  return r;
}

// partial[b] = sum of |w| over weights [b*kChunk, (b+1)*kChunk), float64.
__global__ void __launch_bounds__(kRedThreads)
twn_abs_partial_kernel(const float* __restrict__ w, int64_t total, double* __restrict__ partial) {
  __shared__ double sh[kRedThreads];
  const int64_t begin = static_cast<int64_t>(blockIdx.x) * kChunk;
  const int64_t end = begin + kChunk < total ? begin + kChunk : total;
  double acc = 0.0;
  for (int64_t e = begin + threadIdx.x; e < end; e += kRedThreads) acc += fabs(static_cast<double>(__ldg(w + e)));
  const double s = block_sum_f64(acc, sh);
  if (threadIdx.x == 0) partial[blockIdx.x] = s;
}

// Every block derives Delta from the partial sums (same order in every block),
// then ternarises, scales and packs whole rows.
__global__ void __launch_bounds__(kRedThreads)
twn_pack_rows_kernel(const float* __restrict__ w, int64_t n, int64_t k, const double* __restrict__ partial,
                     int64_t nparts, int64_t total, uint16_t* __restrict__ packed, float* __restrict__ scale,
                     float* __restrict__ delta_out) {
  __shared__ double shd[kRedThreads];
  __shared__ long long shl[kRedThreads];
  double ps = 0.0;
  for (int64_t i = threadIdx.x; i < nparts; i += kRedThreads) ps += partial[i];
  const double sum_abs = block_sum_f64(ps, shd);
  const double mean_abs = total > 0 ? sum_abs / static_cast<double>(total) : 0.0;
  const float delta = __double2float_rn(0.7 * mean_abs);
  if (blockIdx.x == 0 && threadIdx.x == 0) *delta_out = delta;

  const int64_t kt = bnn::words10(k);
  for (int64_t r = blockIdx.x; r < n; r += gridDim.x) {
    const float* row = w + r * k;
    double kept = 0.0;
    long long nz = 0;
    for (int64_t j = threadIdx.x; j < kt; j += kRedThreads) {
      uint32_t word = 0, weight = 1;
#pragma unroll
      for (int i = 0; i < 10; ++i) {
        const int64_t e = 10 * j + i;
        uint32_t digit = 1;  // trit 0
        if (e < k) {
          const float v = __ldg(row + e);
          const float a = fabsf(v);
          if (a > delta) {
            digit = v > 0.0f ? 2u : 0u;
            kept += static_cast<double>(a);
            ++nz;
          }
        }
        word += digit * weight;
        weight *= 3u;
      }
      packed[r * kt + j] = static_cast<uint16_t>(word);
    }
    const double kept_sum = block_sum_f64(kept, shd);
    const long long nz_sum = block_sum_i64(nz, shl);
    if (threadIdx.x == 0)
      scale[r] = nz_sum > 0 ? __double2float_rn(kept_sum / static_cast<double>(nz_sum)) : 0.0f;
  }
}

// ---------------------------------------------------------------------------
// Ternary GEMV (small m): one warp per weight row, fp32 accumulation.
// ---------------------------------------------------------------------------
// Accumulates sum_i x[i] * t_i over the 10 trits of `word`, x given as 10 floats.
__device__ __forceinline__ float dot_word(uint32_t word, const float* x) {
  uint32_t F = word * kFixMul;
  float acc = 0.0f;
#pragma unroll
  for (int i = 9; i >= 0; --i) {
    const uint32_t d = __umulhi(F, 3u);
    F *= 3u;
    const float t = d == 0u ? -1.0f : (d == 2u ? 1.0f : 0.0f);
    acc = fmaf(x[i], t, acc);
  }
  return acc;
}

template <int MT>
__global__ void __launch_bounds__(256)
ternary_gemv_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ packed,
                    const float* __restrict__ scale, int m, int64_t n, int64_t k, int64_t kt,
                    float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = warp; r < n; r += nwarps) {
    float acc[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) acc[t] = 0.0f;
    for (int64_t j = lane; j < kt; j += 32) {
      const uint32_t word = __ldcs(packed + r * kt + j);
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        if (t < m) {
          float xv[10];
          const uint16_t* xr = x + static_cast<int64_t>(t) * k + 10 * j;
#pragma unroll
          for (int i = 0; i < 10; ++i) {
            const int64_t e = 10 * j + i;
            xv[i] = e < k ? __uint_as_float(static_cast<uint32_t>(__ldg(xr + i)) << 16) : 0.0f;
          }
          acc[t] += dot_word(word, xv);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < MT; ++t)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], off);
    if (lane == 0) {
      const float s = __ldg(scale + r);
#pragma unroll
      for (int t = 0; t < MT; ++t)
        if (t < m) out[static_cast<int64_t>(t) * n + r] = s * acc[t];
    }
  }
}


// ---------------------------------------------------------------------------
// Ternary GEMV, m = 1: activation pair tables + base-9 digits.
//
// Each base-9 digit v of a word (v = d_{2q} + 3 d_{2q+1}, q = 0..4) covers two
// consecutive trits, so for the activation pair (x_{2P}, x_{2P+1}) at pair
// index P = 5j + q a 9-entry table T_P[v] = x_{2P} (v mod 3 - 1) + x_{2P+1}
// (v div 3 - 1) turns two multiply-adds into one shared-memory load and one
// add.  The digit is the high word of 9F and the next fraction its low word
// (taken with __umulhi and a 32-bit multiply).
// Lanes of a half-warp own 16 consecutive weight rows and walk the same word
// index, so the 16 lanes read within one 9-entry table (at most 9 distinct
// addresses, one per bank: no bank conflicts); the two half-warps work on
// K-slices whose tables sit in disjoint banks.  The 16-row chunk of packed
// words is contiguous in memory and is brought into shared memory with
// 16-byte cp.async (double-buffered across the chunks this CTA owns); the
// per-slice partial sums are added in a fixed order, then scaled once.  The
// chunk copies run kLutStages - 1 chunks ahead of the compute (the copy
// latency from HBM is several times one chunk's compute).
// ---------------------------------------------------------------------------
constexpr int kLutRows = 16;
constexpr int kLutStages = 4;

template <int SLICES>
__global__ void __launch_bounds__(kLutRows * SLICES, 1)
ternary_gemv_lut_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ packed,
                        const float* __restrict__ scale, int64_t n, int k, int kt, int slice_words,
                        float* __restrict__ out) {
  constexpr int THREADS = kLutRows * SLICES;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int npairs = 5 * kt;
  float* T = reinterpret_cast<float*>(smem_raw);                                   // [npairs][9]
  const size_t t_bytes = (static_cast<size_t>(npairs) * 9 * sizeof(float) + 15) & ~static_cast<size_t>(15);
  const size_t chunk_bytes = (static_cast<size_t>(kLutRows) * kt * 2 + 15) & ~static_cast<size_t>(15);
  uint16_t* const buf0 = reinterpret_cast<uint16_t*>(smem_raw + t_bytes);         // [kLutStages][chunk]
  const size_t chunk_elems = chunk_bytes / 2;
  float* red = reinterpret_cast<float*>(smem_raw + t_bytes + kLutStages * chunk_bytes);  // [SLICES][kLutRows]

  const int tid = threadIdx.x;
  const int64_t nchunks = (n + kLutRows - 1) / kLutRows;

  auto issue_chunk = [&](int64_t c, uint16_t* dst) {
    const int64_t rows = n - c * kLutRows < kLutRows ? n - c * kLutRows : kLutRows;
    const int64_t bytes = rows * kt * 2;
    const unsigned char* src = reinterpret_cast<const unsigned char*>(packed + c * kLutRows * kt);
    for (int64_t off = static_cast<int64_t>(tid) * 16; off < bytes; off += THREADS * 16) {
      const int64_t left = bytes - off;
      const int sz = left < 16 ? static_cast<int>(left) : 16;
      const unsigned saddr = static_cast<unsigned>(__cvta_generic_to_shared(reinterpret_cast<unsigned char*>(dst) + off));
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(saddr), "l"(src + off), "r"(sz));
    }
  };

  // Prefetch the first kLutStages - 1 chunks of this CTA (one commit group each).
#pragma unroll
  for (int st = 0; st < kLutStages - 1; ++st) {
    const int64_t cc = blockIdx.x + static_cast<int64_t>(st) * gridDim.x;
    if (cc < nchunks) issue_chunk(cc, buf0 + st * chunk_elems);
    asm volatile("cp.async.commit_group;\n" ::);
  }
  int64_t c = blockIdx.x;

  // Pair tables from the activation row (exact products, one rounding per entry).
  for (int p = tid; p < npairs; p += THREADS) {
    const float x0 = 2 * p < k ? __uint_as_float(static_cast<uint32_t>(__ldg(x + 2 * p)) << 16) : 0.0f;
    const float x1 = 2 * p + 1 < k ? __uint_as_float(static_cast<uint32_t>(__ldg(x + 2 * p + 1)) << 16) : 0.0f;
#pragma unroll
    for (int v = 0; v < 9; ++v)
      T[p * 9 + v] = x0 * static_cast<float>(v % 3 - 1) + x1 * static_cast<float>(v / 3 - 1);
  }

  const int row = tid % kLutRows;
  const int sl = tid / kLutRows;
  const int j0 = sl * slice_words;
  const int j1 = j0 + slice_words < kt ? j0 + slice_words : kt;

  for (int it = 0; c < nchunks; c += gridDim.x, ++it) {
    // chunk `it` was the (it+1)-th commit group: allow the kLutStages-2 newer ones to be pending
    asm volatile("cp.async.wait_group %0;\n" ::"n"(kLutStages - 2));
    __syncthreads();

    const uint16_t* rowp = buf0 + (it % kLutStages) * chunk_elems + row * kt;
    float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll 2
    for (int j = j0; j < j1; ++j) {
      uint32_t F = static_cast<uint32_t>(rowp[j]) * kFixMul;
      const float* Tj = T + (5 * j) * 9;
#pragma unroll
      for (int q = 4; q >= 0; --q) {
        // high and low words of 9F: the digit and the next fraction
        const uint32_t v = __umulhi(F, 9u);
        F *= 9u;
        if (q & 1) acc1 += Tj[q * 9 + v]; else acc0 += Tj[q * 9 + v];
      }
    }
    red[sl * kLutRows + row] = acc0 + acc1;
    __syncthreads();
    if (tid < kLutRows) {
      const int64_t r = c * kLutRows + tid;
      if (r < n) {
        float s = 0.0f;
#pragma unroll 4
        for (int q = 0; q < SLICES; ++q) s += red[q * kLutRows + tid];
        out[r] = __ldg(scale + r) * s;
      }
    }
    // The buffer of chunk it + kLutStages - 1 (the one computed in the previous
    // iteration) and red are rewritten only after this barrier.
    __syncthreads();
    const int64_t cn = c + static_cast<int64_t>(kLutStages - 1) * gridDim.x;
    if (cn < nchunks) issue_chunk(cn, buf0 + ((it + kLutStages - 1) % kLutStages) * chunk_elems);
    asm volatile("cp.async.commit_group;\n" ::);
  }
  asm volatile("cp.async.wait_group 0;\n" ::);
}

constexpr int kLutSlices = 32;

size_t lut_smem_bytes(int64_t kt) {
  const size_t t_bytes = (static_cast<size_t>(5 * kt) * 9 * sizeof(float) + 15) & ~static_cast<size_t>(15);
  const size_t chunk_bytes = (static_cast<size_t>(kLutRows) * kt * 2 + 15) & ~static_cast<size_t>(15);
  return t_bytes + kLutStages * chunk_bytes + static_cast<size_t>(kLutSlices) * kLutRows * sizeof(float);
}

// ---------------------------------------------------------------------------
// Ternary GEMM (m > 8): decode trits to bf16 tiles in shared memory, bf16
// mma.sync m16n8k16 with fp32 accumulation.
// ---------------------------------------------------------------------------
constexpr int kTBM = 64;           // activation rows per CTA
constexpr int kTBN = 64;           // weight rows per CTA
constexpr int kTBKW = 16;          // base-3 words per K chunk
constexpr int kTBK = 10 * kTBKW;   // 160 trits per chunk (a multiple of 16)
constexpr int kTPitch = kTBK + 8;  // bf16 elements per smem row (336 bytes)

__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                            const void* p) {
  const unsigned a = static_cast<unsigned>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(a));
}
__device__ __forceinline__ void ldmatrix_x2(uint32_t& r0, uint32_t& r1, const void* p) {
  const unsigned a = static_cast<unsigned>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n" : "=r"(r0), "=r"(r1) : "r"(a));
}
__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__global__ void __launch_bounds__(256)
ternary_gemm_mma_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ packed,
                        const float* __restrict__ scale, int64_t m, int64_t n, int64_t k, int64_t kt,
                        float* __restrict__ out) {
  __shared__ __align__(16) uint16_t Xs[kTBM * kTPitch];
  __shared__ __align__(16) uint16_t Ws[kTBN * kTPitch];
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int wm = warp & 1;   // 2 warps along M (32 rows each)
  const int wn = warp >> 1;  // 4 warps along N (16 cols each)
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kTBM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kTBN;

  float acc[2][2][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][b][c] = 0.0f;

  const int64_t nchunks = (kt + kTBKW - 1) / kTBKW;
  for (int64_t ch = 0; ch < nchunks; ++ch) {
    const int64_t kbase = ch * kTBK;
    // Activations: kTBM rows x kTBK bf16, zero outside [m) x [k).
    for (int idx = tid; idx < kTBM * kTBK; idx += 256) {
      const int row = idx / kTBK, col = idx % kTBK;
      const int64_t gm = m0 + row, gk = kbase + col;
      Xs[row * kTPitch + col] = (gm < m && gk < k) ? __ldg(x + gm * k + gk) : static_cast<uint16_t>(0);
    }
    // Weights: kTBN rows x kTBKW words, each decoded to 10 bf16 trits.
    for (int idx = tid; idx < kTBN * kTBKW; idx += 256) {
      const int row = idx / kTBKW, wj = idx % kTBKW;
      const int64_t gn = n0 + row, gj = ch * kTBKW + wj;
      uint16_t* dst = Ws + row * kTPitch + 10 * wj;
      if (gn < n && gj < kt) {
        uint32_t F = static_cast<uint32_t>(__ldg(packed + gn * kt + gj)) * kFixMul;
#pragma unroll
        for (int i = 9; i >= 0; --i) {
          const uint32_t d = __umulhi(F, 3u);
          F *= 3u;
          dst[i] = d == 0u ? static_cast<uint16_t>(0xBF80u) : (d == 2u ? static_cast<uint16_t>(0x3F80u) : static_cast<uint16_t>(0));
        }
      } else {
#pragma unroll
        for (int i = 0; i < 10; ++i) dst[i] = 0;
      }
    }
    __syncthreads();
#pragma unroll
    for (int ks = 0; ks < kTBK; ks += 16) {
      uint32_t af[2][4], bfr[2][2];
#pragma unroll
      for (int mi = 0; mi < 2; ++mi) {
        const int row = wm * 32 + mi * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int col = ks + 8 * (lane >> 4);
        ldmatrix_x4(af[mi][0], af[mi][1], af[mi][2], af[mi][3], Xs + row * kTPitch + col);
      }
#pragma unroll
      for (int ni = 0; ni < 2; ++ni) {
        const int row = wn * 16 + ni * 8 + (lane & 7);
        const int col = ks + 8 * ((lane >> 3) & 1);
        ldmatrix_x2(bfr[ni][0], bfr[ni][1], Ws + row * kTPitch + col);
      }
#pragma unroll
      for (int mi = 0; mi < 2; ++mi)
#pragma unroll
        for (int ni = 0; ni < 2; ++ni) mma_bf16_16816(acc[mi][ni], af[mi], bfr[ni]);
    }
    __syncthreads();
  }

  const int g = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int ni = 0; ni < 2; ++ni)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t gm = m0 + wm * 32 + mi * 16 + g + 8 * h;
        if (gm >= m) continue;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int64_t gn = n0 + wn * 16 + ni * 8 + 2 * tq + c;
          if (gn < n) out[gm * n + gn] = __ldg(scale + gn) * acc[mi][ni][2 * h + c];
        }
      }
}

}  // namespace

extern "C" bnn_status bnn_ternary_pack(const float* w, int64_t n, int64_t k, uint16_t* packed,
                                       float* scale, float* delta, cudaStream_t s) {
  if (n < 0 || k < 0) return BNN_ERR_INVALID_ARG;
  if (!delta) return BNN_ERR_INVALID_ARG;
  if (n > 0 && !scale) return BNN_ERR_INVALID_ARG;
  if (n > 0 && k > 0 && (!w || !packed)) return BNN_ERR_INVALID_ARG;
  if (k > 0 && n > (int64_t(1) << 40) / k) return BNN_ERR_INVALID_ARG;
  if ((w && !bnn::aligned(w, 4)) || (packed && !bnn::aligned(packed, 2)) || (scale && !bnn::aligned(scale, 4)) ||
      !bnn::aligned(delta, 4))
    return BNN_ERR_MISALIGNED;
  const int64_t total = n * k;
  const int64_t nparts = (total + kChunk - 1) / kChunk;
  double* partial = nullptr;
  if (nparts > 0) {
    BNN_TRY(cudaMallocAsync(reinterpret_cast<void**>(&partial), static_cast<size_t>(nparts) * sizeof(double), s));
    twn_abs_partial_kernel<<<static_cast<unsigned>(nparts), kRedThreads, 0, s>>>(w, total, partial);
    const bnn_status st = bnn::check_launch();
    if (st != BNN_OK) {
      cudaFreeAsync(partial, s);
      return st;
    }
  }
  const int64_t cap = static_cast<int64_t>(bnn::sm_count()) * 8;
  const int grid = static_cast<int>(n < 1 ? 1 : (n < cap ? n : cap));
  twn_pack_rows_kernel<<<grid, kRedThreads, 0, s>>>(w, n, k, partial, nparts, total, packed, scale, delta);
  bnn_status st = bnn::check_launch();
  if (partial) {
    const cudaError_t e = cudaFreeAsync(partial, s);
    if (st == BNN_OK && e != cudaSuccess) st = bnn::cuda_fail(e);
  }
  return st;
}

extern "C" bnn_status bnn_ternary_gemm(const uint16_t* x_bf16, const uint16_t* packed, const float* scale,
                                       int64_t m, int64_t n, int64_t k, float* out, cudaStream_t s) {
  if (m < 0 || n < 0 || k < 0) return BNN_ERR_INVALID_ARG;
  if (m == 0 || n == 0) return BNN_OK;
  if (!scale || !out || (k > 0 && (!x_bf16 || !packed))) return BNN_ERR_INVALID_ARG;
  if ((x_bf16 && !bnn::aligned(x_bf16, 2)) || (packed && !bnn::aligned(packed, 2)) || !bnn::aligned(scale, 4) ||
      !bnn::aligned(out, 4))
    return BNN_ERR_MISALIGNED;
  const int64_t kt = bnn::words10(k);
  if (m == 1 && kt > 0 && bnn::aligned(packed, 16) && lut_smem_bytes(kt) <= 200 * 1024) {
    const size_t smem = lut_smem_bytes(kt);
    auto kern = ternary_gemv_lut_kernel<kLutSlices>;
    BNN_TRY(bnn::ensure_smem(kern, smem));
    int slice_words = static_cast<int>((kt + kLutSlices - 1) / kLutSlices);
    const int64_t nchunks = (n + kLutRows - 1) / kLutRows;
    const int grid = static_cast<int>(nchunks < bnn::sm_count() ? nchunks : bnn::sm_count());
    kern<<<grid, kLutRows * kLutSlices, smem, s>>>(x_bf16, packed, scale, n, static_cast<int>(k), static_cast<int>(kt),
                                                  slice_words, out);
    return bnn::check_launch();
  }
  if (m <= 8) {
    const int64_t warps_per_block = 8;
    const int64_t blocks_needed = (n + warps_per_block - 1) / warps_per_block;
    const int64_t cap = static_cast<int64_t>(bnn::sm_count()) * 8;
    const int grid = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
    if (m == 1) ternary_gemv_kernel<1><<<grid, 256, 0, s>>>(x_bf16, packed, scale, 1, n, k, kt, out);
    else if (m <= 4) ternary_gemv_kernel<4><<<grid, 256, 0, s>>>(x_bf16, packed, scale, static_cast<int>(m), n, k, kt, out);
    else ternary_gemv_kernel<8><<<grid, 256, 0, s>>>(x_bf16, packed, scale, static_cast<int>(m), n, k, kt, out);
    return bnn::check_launch();
  }
  const int64_t gx = (n + kTBN - 1) / kTBN, gy = (m + kTBM - 1) / kTBM;
  if (gx > 2147483647LL || gy > 65535) return BNN_ERR_INVALID_ARG;
  ternary_gemm_mma_kernel<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), 256, 0, s>>>(
      x_bf16, packed, scale, m, n, k, kt, out);
  return bnn::check_launch();
}

// ---------------------------------------------------------------------------
// bnn_ternary_pack_noalloc: the same TWN pack with its scratch in a fixed
// device array instead of memory taken from an allocator.
//
// The float64 partial sums of |W| (one per 65536 weights) live in the
// file-scope array below, which every GPU that loads this library holds
// until the process exits.  Its host-side name is only a stand-in for the
// symbol; the device address comes from cudaGetSymbolAddress, looked up once
// per device (with that device current) on the first call and cached.
// ---------------------------------------------------------------------------
constexpr int64_t kNoAllocMaxParts = 8192;  // 64 KiB of float64: up to 8192 * 65536 = 2^29 weights

static __device__ __align__(256) double g_twn_noalloc_partials[kNoAllocMaxParts];

namespace {

constexpr int kNoAllocMaxDevices = 64;
double* g_noalloc_ptr[kNoAllocMaxDevices] = {nullptr};
std::mutex g_noalloc_mu;

// Device address of g_twn_noalloc_partials on the current device.
bnn_status noalloc_scratch(double** out) {
  int dev = -1;
  BNN_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNoAllocMaxDevices) return BNN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_twn_noalloc_partials);
    if (e != cudaSuccess) return bnn::cuda_fail(e);
    g_noalloc_ptr[dev] = static_cast<double*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return BNN_OK;
}

}  // namespace

extern "C" bnn_status bnn_ternary_pack_noalloc(const float* w, int64_t n, int64_t k, uint16_t* packed,
                                               float* scale, float* delta, cudaStream_t s) {
  if (n < 0 || k < 0) return BNN_ERR_INVALID_ARG;
  if (!delta) return BNN_ERR_INVALID_ARG;
  if (n > 0 && !scale) return BNN_ERR_INVALID_ARG;
  if (n > 0 && k > 0 && (!w || !packed)) return BNN_ERR_INVALID_ARG;
  if (k > 0 && n > (int64_t(1) << 40) / k) return BNN_ERR_INVALID_ARG;
  if ((w && !bnn::aligned(w, 4)) || (packed && !bnn::aligned(packed, 2)) || (scale && !bnn::aligned(scale, 4)) ||
      !bnn::aligned(delta, 4))
    return BNN_ERR_MISALIGNED;
  const int64_t total = n * k;
  const int64_t nparts = (total + kChunk - 1) / kChunk;
  if (nparts > kNoAllocMaxParts) return BNN_ERR_INVALID_ARG;  // more than 2^29 weights
  double* partial = nullptr;
  if (nparts > 0) {
    const bnn_status st = noalloc_scratch(&partial);
    if (st != BNN_OK) return st;
    // Every slot the second kernel reads is written by the first kernel of the
    // same call, so nothing left by an earlier call needs clearing.
    twn_abs_partial_kernel<<<static_cast<unsigned>(nparts), kRedThreads, 0, s>>>(w, total, partial);
    const bnn_status st2 = bnn::check_launch();
    if (st2 != BNN_OK) return st2;
  }
  const int64_t cap = static_cast<int64_t>(bnn::sm_count()) * 8;
  const int grid = static_cast<int>(n < 1 ? 1 : (n < cap ? n : cap));
  twn_pack_rows_kernel<<<grid, kRedThreads, 0, s>>>(w, n, k, partial, nparts, total, packed, scale, delta);
  return bnn::check_launch();
}
