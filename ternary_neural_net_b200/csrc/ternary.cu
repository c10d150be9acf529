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
#include <cooperative_groups.h>
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

// Ternarisation rules (BNN_TERNARY_* in bnn.h):
//   TWN:     Delta = float32(0.7 mean|W|), trit = sign(w) where |w| > Delta;
//   ABSMEAN: gamma = float32(mean|W|), trit = clamp(round-half-even(w / gamma), -1, 1)
//            ("Binary Math Effectiveness", section 5; BitNet b1.58), i.e.
//            sign(w) where |w / gamma| > 0.5, 0 at or below (ties round to 0);
//   DELTA:   a given threshold F, trit = sign(w) where |w| > F.
// Every mode takes the per-row least-squares scale.
enum { kModeTWN = 0, kModeAbsmean = 1, kModeDelta = 2 };

// Every block derives the threshold from the partial sums (same order in every
// block), then ternarises, scales and packs whole rows.
template <int MODE>
__global__ void __launch_bounds__(kRedThreads)
twn_pack_rows_kernel(const float* __restrict__ w, int64_t n, int64_t k, const double* __restrict__ partial,
                     int64_t nparts, int64_t total, uint16_t* __restrict__ packed, float* __restrict__ scale,
                     float* __restrict__ delta_out, float fixed_threshold = 0.0f) {
  __shared__ double shd[kRedThreads];
  __shared__ long long shl[kRedThreads];
  float delta = fixed_threshold;
  if constexpr (MODE != kModeDelta) {
    double ps = 0.0;
    for (int64_t i = threadIdx.x; i < nparts; i += kRedThreads) ps += partial[i];
    const double sum_abs = block_sum_f64(ps, shd);
    const double mean_abs = total > 0 ? sum_abs / static_cast<double>(total) : 0.0;
    delta = __double2float_rn(MODE == kModeTWN ? 0.7 * mean_abs : mean_abs);
  }
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
          bool keep;
          if constexpr (MODE == kModeAbsmean) {
            keep = delta > 0.0f && fabsf(__fdiv_rn(v, delta)) > 0.5f;  // |round-half-even(q)| >= 1
          } else {
            keep = a > delta;
          }
          if (keep) {
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
                    float* __restrict__ out, const float* __restrict__ bias) {
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
        if (t < m) out[static_cast<int64_t>(t) * n + r] = bias ? s * acc[t] + __ldg(bias + r) : s * acc[t];
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
// One CTA per SM builds the tables once and takes a contiguous block of
// weight rows; each warp takes one row at a time, its lanes walking the row's
// words (lane l: words l, l + 32, ... -- 64-byte coalesced loads, the next
// row's words prefetched in registers while this row is decoded).  The tables
// are stored entry-major, word-minor: entry (q, v) of word j sits at
// (9q + v) * ktp + j with ktp a multiple of 32, so the 32 lanes (32
// consecutive words) always hit 32 different banks whatever digits they
// decode.  The lanes' sums are added by a shuffle tree (a fixed order) and
// scaled once.  No block barrier after the table build.  Launched with
// programmatic dependent launch: the first row's words are read before
// waiting for the kernel that produced x.
// ---------------------------------------------------------------------------
constexpr int kRowThreads = 1024;
constexpr int kRowWords = 16;  // words per lane per pass over a row (512 words per warp pass)

__host__ __device__ constexpr int table_pitch(int kt) { return (kt + 31) & ~31; }

__global__ void __launch_bounds__(kRowThreads, 1)
ternary_gemv_rows_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ packed,
                         const float* __restrict__ scale, int64_t n, int k, int kt, float* __restrict__ out,
                         const float* __restrict__ bias) {
  extern __shared__ float T[];  // [45][ktp]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = kRowThreads / 32;
  constexpr int kPassWords = 32 * kRowWords;
  const int ktp = table_pitch(kt);
  const int64_t r_begin = n * blockIdx.x / gridDim.x, r_end = n * (blockIdx.x + 1) / gridDim.x;
  bnn::pdl_trigger();

  // the words of (row r, pass p) for this lane (words p * kPassWords + lane + 32 i), 0xFFFF past the row
  auto fetch = [&](int64_t r, int p, uint32_t (&w)[kRowWords]) {
    const bool live = r < r_end;
    const int lim = live ? kt - p * kPassWords - lane : 0;
    const uint16_t* src = packed + (live ? r : r_begin) * kt + p * kPassWords + lane;
#pragma unroll
    for (int i = 0; i < kRowWords; ++i) {
      w[i] = 0xFFFFu;
      if (32 * i < lim) w[i] = __ldcs(src + 32 * i);
    }
  };
  const int passes = (kt + kPassWords - 1) / kPassWords;
  int64_t r = r_begin + warp;
  int p = 0;
  uint32_t cur[kRowWords];
  fetch(r, p, cur);  // weights do not depend on the preceding kernel

  bnn::pdl_wait();  // x may come from it
  for (int e = tid; e < 5 * kt; e += kRowThreads) {
    const int q = e / kt, j = e - q * kt;  // consecutive threads: consecutive words, distinct banks
    const int P = 5 * j + q;
    const float x0 = 2 * P < k ? __uint_as_float(static_cast<uint32_t>(__ldg(x + 2 * P)) << 16) : 0.0f;
    const float x1 = 2 * P + 1 < k ? __uint_as_float(static_cast<uint32_t>(__ldg(x + 2 * P + 1)) << 16) : 0.0f;
#pragma unroll
    for (int v = 0; v < 9; ++v)
      T[(9 * q + v) * ktp + j] = x0 * static_cast<float>(v % 3 - 1) + x1 * static_cast<float>(v / 3 - 1);
  }
  __syncthreads();

  // shared-memory byte addresses: entry (q, v) of word j at tq[q] + v * stride + 4 j'
  const uint32_t stride = 4u * static_cast<uint32_t>(ktp);
  const uint32_t t0 = static_cast<uint32_t>(__cvta_generic_to_shared(T)) + 4u * static_cast<uint32_t>(lane);
  float acc0 = 0.0f, acc1 = 0.0f;
  while (r < r_end) {
    // the next (row, pass) while this one is decoded
    const int pn = p + 1 < passes ? p + 1 : 0;
    const int64_t rn = p + 1 < passes ? r : r + kWarps;
    uint32_t nxt[kRowWords];
    fetch(rn, pn, nxt);
    uint32_t tq[5];
#pragma unroll
    for (int q = 0; q < 5; ++q) tq[q] = t0 + 4u * static_cast<uint32_t>(p * kPassWords) + 9u * q * stride;
#pragma unroll
    for (int i = 0; i < kRowWords; ++i) {
      if (cur[i] != 0xFFFFu) {
        uint32_t F = cur[i] * kFixMul;
#pragma unroll
        for (int q = 4; q >= 0; --q) {
          // base-9 digit q (trits 2q, 2q+1) in the high word of 9F, the rest in the low word
          const uint64_t P9 = static_cast<uint64_t>(F) * 9u;
          const uint32_t v = static_cast<uint32_t>(P9 >> 32);
          F = static_cast<uint32_t>(P9);
          float t;
          asm volatile("ld.shared.f32 %0, [%1];\n" : "=f"(t) : "r"(tq[q] + v * stride + 128u * i));
          if (q & 1) acc1 += t; else acc0 += t;
        }
      }
    }
    if (pn == 0) {  // the row is complete
      float sum = acc0 + acc1;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      if (lane == 0) out[r] = bias ? __ldg(scale + r) * sum + __ldg(bias + r) : __ldg(scale + r) * sum;
      acc0 = acc1 = 0.0f;
    }
    r = rn;
    p = pn;
#pragma unroll
    for (int i = 0; i < kRowWords; ++i) cur[i] = nxt[i];
  }
}

size_t rows_smem_bytes(int64_t kt) {
  return static_cast<size_t>(45) * static_cast<size_t>((kt + 31) & ~int64_t{31}) * sizeof(float);
}

// ---------------------------------------------------------------------------
// Ternary GEMV, m = 1, k <= 4800: 5 + 5-trit activation tables, the row
// length split over a cluster of kC5 CTAs.
//
// A word's low five digits (w mod 243) and high five (w div 243, one exact
// multiply-shift) index two 243-entry tables of word position j: lo_j[e] =
// sum_{i<5} x[10j+i] (d_i(e) - 1) and hi_j[e] the same over x[10j+5..10j+9], so
// a word costs two shared-memory loads and two adds.  The tables of a whole row
// do not fit one SM (2 x 243 entries per word), so the kC5 CTAs of a cluster
// take one slice of at most 96 word positions each and hold only that slice's
// tables (two [243][96] float arrays, 182 KiB); every CTA of the cluster runs
// over the cluster's contiguous range of rows.
//
// Lanes and columns: in one row, lane l holds the words of slice columns 2l and
// 2l + 1 (one 32-bit load where kt and the slice start are even, else two
// 16-bit loads) and of column 64 + l (a 16-bit load).  Table rows store column
// c < 64 at position (c & 1) * 32 + c / 2 and column c >= 64 at c, so each of
// the six lookups of a row reads 32 consecutive positions of one table row
// chosen per lane: 32 different banks, whatever the words are.  Columns past
// the slice hold x = 0 (all entries 0); lanes there read the row's first
// word(s) instead and look them up in those zero columns.
//
// A warp takes 16 consecutive rows per round (four without 32-bit pairs) and
// holds the words of two rounds: the first two are loaded before the
// programmatic-launch wait, while x is staged and the tables are built (for a
// cluster's first 512 rows, every word it reads), and each round's registers
// are refilled with the round two ahead once its lookups are done.  Rows past
// the cluster's last are read as that last row and dropped, so nothing in the
// loop is predicated per row.  The rows' lane sums are added in one transposed
// shuffle tree (16 shuffles for 16 rows) and stored as the CTA's slice
// sums; at the end of each chunk of kC5Rows rows, after a cluster barrier, CTA q
// adds for its share of the chunk the kC5 slice sums in rank order through
// distributed shared memory, scales once and writes.  Deterministic for a given launch shape.
// ---------------------------------------------------------------------------
constexpr int kC5 = 5;                 // CTAs per cluster (slices of the row)
constexpr int kC5Threads = 512;
constexpr int kC5Warps = kC5Threads / 32;
constexpr int kC5Pitch = 96;           // table positions per slice (64 in pairs + 32 single)
constexpr int kC5Rows = 1024;          // rows of a chunk (slice sums held at once)
// rows per warp round: 16 with 32-bit word pairs (2 registers a row), 4 with
// three 16-bit words (3 registers a row); two rounds of words are held at once
template <bool VEC>
constexpr int c5_rows_per_warp() { return VEC ? 16 : 4; }
static_assert(kC5Rows % (2 * kC5Warps * 16) == 0 && kC5Rows % (2 * kC5Warps * 4) == 0,
              "a chunk is an even number of rounds");
constexpr uint32_t kDiv243Hi = 17674763u;   // ceil(2^32 / 243): floor(w / 243) = high word of w * kDiv243Hi
constexpr uint32_t kC5HiOff = 243u * kC5Pitch * 4u;  // bytes from the lo table to the hi table

constexpr bool div243_exact() {
  for (uint64_t w = 0; w < 59049u; ++w)
    if (((w * kDiv243Hi) >> 32) != w / 243u) return false;
  return true;
}
static_assert(div243_exact(), "multiply-high division by 243");

// floats: lo [243][96], hi [243][96], slice sums [kC5Rows], x [10][96] by table position
size_t c5_smem_bytes() { return (2u * 243u * kC5Pitch + kC5Rows + 10u * kC5Pitch) * sizeof(float); }

// slice column of table position p
__device__ __forceinline__ int c5_column(int p) { return p < 64 ? (p < 32 ? 2 * p : 2 * (p - 32) + 1) : p; }

// The words of one row at this lane's three columns: VEC, one 32-bit load for
// columns 2l, 2l + 1 (w[0]) and one 16-bit load for column 64 + l (w[1]);
// else three 16-bit loads.  pa, pb, pc point at the lane's columns in the
// cluster's first row (at that row's first word where a column lies past the
// slice: the lane then looks up a real word in a table column of zeros), ro is
// the row's offset from there in 16-bit words.
template <bool VEC>
struct C5Words {
  uint32_t w[VEC ? 2 : 3];
};

template <bool VEC>
__device__ __forceinline__ void c5_fetch(const uint16_t* __restrict__ pa, const uint16_t* __restrict__ pb,
                                         const uint16_t* __restrict__ pc, uint32_t ro, C5Words<VEC>& v) {
  if constexpr (VEC) {
    v.w[0] = __ldcs(reinterpret_cast<const uint32_t*>(pa + ro));
    v.w[1] = static_cast<uint32_t>(__ldcs(pc + ro));
  } else {
    v.w[0] = static_cast<uint32_t>(__ldcs(pa + ro));
    v.w[1] = static_cast<uint32_t>(__ldcs(pb + ro));
    v.w[2] = static_cast<uint32_t>(__ldcs(pc + ro));
  }
}

// lo_p[ql] + hi_p[qh] of one word; t = this lane's lo-table position (bytes),
// plus 128 per 32 positions; the hi table sits kC5HiOff bytes above.
__device__ __forceinline__ float c5_lookup(uint32_t w, uint32_t t) {
  const uint32_t qh = __umulhi(w, kDiv243Hi);  // digits 5..9
  const uint32_t ql = w - 243u * qh;          // digits 0..4
  float a, b;
  asm volatile("ld.shared.f32 %0, [%1];\n" : "=f"(a) : "r"(t + ql * (4u * kC5Pitch)));
  asm volatile("ld.shared.f32 %0, [%1+%2];\n" : "=f"(b) : "r"(t + qh * (4u * kC5Pitch)), "n"(kC5HiOff));
  return a + b;
}

// One row's three words at this lane.  Words are clamped to 3^10 - 1 first, so
// a word outside the format (its result unspecified) still looks up inside the
// tables.
template <bool VEC>
__device__ __forceinline__ float c5_row(const C5Words<VEC>& v, uint32_t t) {
  constexpr uint32_t kMaxWord = 59048u;
  float s;
  if constexpr (VEC) {
    const uint32_t pr = __vminu2(v.w[0], kMaxWord | (kMaxWord << 16));
    s = c5_lookup(pr & 0xFFFFu, t) + c5_lookup(pr >> 16, t + 128u);
    s += c5_lookup(min(v.w[1], kMaxWord), t + 256u);
  } else {
    s = c5_lookup(min(v.w[0], kMaxWord), t) + c5_lookup(min(v.w[1], kMaxWord), t + 128u);
    s += c5_lookup(min(v.w[2], kMaxWord), t + 256u);
  }
  return s;
}

// Sums of D rows (a[j] = this lane's part of row j) over the warp: D / 2 + ... +
// 1 shuffles exchange halves of the rows (masks 16, 8, ...), after which lane l
// holds a part of row l >> (5 - log2 D); plain shuffles finish the sum.  The
// result is row (lane >> (5 - log2 D))'s total, in every lane of its group.
template <int D>
__device__ __forceinline__ float c5_reduce(float (&a)[D], int lane) {
#pragma unroll
  for (int h = D / 2, mask = 16; h >= 1; h /= 2, mask >>= 1) {
    const bool up = (lane & mask) != 0;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float keep = up ? a[h + i] : a[i];
      const float send = up ? a[i] : a[h + i];
      a[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
    }
  }
  float v = a[0];
#pragma unroll
  for (int mask = 16 / D; mask >= 1; mask >>= 1) v += __shfl_xor_sync(0xffffffffu, v, mask);
  return v;
}

// base + x0 (d0 - 1) + x1 (d1 - 1) for the digits d0 = a % 3, d1 = a / 3 (a is
// a compile-time constant once the caller's loop is unrolled: one add)
__device__ __forceinline__ float c5_entry(int a, float base, float x0, float x1) {
  switch (a) {
    case 0: return base - (x0 + x1);
    case 1: return base - x1;
    case 2: return base + (x0 - x1);
    case 3: return base - x0;
    case 4: return base;
    case 5: return base + x0;
    case 6: return base - (x0 - x1);
    case 7: return base + x1;
    default: return base + (x0 + x1);
  }
}

template <bool VEC>
__global__ void __launch_bounds__(kC5Threads, 1)
ternary_gemv_c5_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ packed,
                       const float* __restrict__ scale, int64_t n, int k, int kt, int slice,
                       float* __restrict__ out, const float* __restrict__ bias) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) float c5sm[];
  float* const lo = c5sm;
  float* const hi = c5sm + 243 * kC5Pitch;
  float* const psum = c5sm + 2 * 243 * kC5Pitch;
  float* const xs = psum + kC5Rows;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = static_cast<int>(cluster.block_rank());
  const int64_t cl = blockIdx.x / kC5, ncl = gridDim.x / kC5;
  const int w0 = rank * slice;                                            // this CTA's first word position
  const int sw = kt - w0 < slice ? (kt - w0 > 0 ? kt - w0 : 0) : slice;  // its word count (<= kC5Pitch)
  const int64_t c0 = n * cl / ncl, c1 = n * (cl + 1) / ncl;              // the cluster's rows
  constexpr int D = c5_rows_per_warp<VEC>();  // rows per warp round
  constexpr int R = kC5Warps * D;             // rows per CTA round
  constexpr int kRoundsPerChunk = kC5Rows / R;
  const int rows_c = static_cast<int>(c1 - c0);
  const int rounds = (rows_c + R - 1) / R;
  bnn::pdl_trigger();

  // Row offsets are 32-bit (the launch keeps n * kt below 2^31).  A warp's rows
  // of round i are the local rows R i + D warp + j; rows past the cluster's
  // last are read as that last row (their sums are dropped), and a warp whose
  // D rows all lie past it skips the round.
  const uint32_t ktu = static_cast<uint32_t>(kt);
  const uint16_t* const row0 = packed + c0 * static_cast<int64_t>(kt);
  const uint16_t* const pa = row0 + (2 * lane < sw ? w0 + 2 * lane : 0);
  const uint16_t* const pb = row0 + (2 * lane + 1 < sw ? w0 + 2 * lane + 1 : 0);
  const uint16_t* const pc = row0 + (64 + lane < sw ? w0 + 64 + lane : 0);
  auto fetch_round = [&](int i, C5Words<VEC> (&buf)[D]) {
    const int rb = i * R + warp * D;
#pragma unroll
    for (int j = 0; j < D; ++j) {
      const uint32_t rl = static_cast<uint32_t>(rb + j < rows_c ? rb + j : rows_c - 1);
      c5_fetch<VEC>(pa, pb, pc, rl * ktu, buf[j]);
    }
  };
  // rounds 0 and 1 are loaded before the programmatic-launch wait, while x is
  // staged and the tables are built
  C5Words<VEC> bufA[D], bufB[D];
  if (warp * D < rows_c) fetch_round(0, bufA);
  if (R + warp * D < rows_c) fetch_round(1, bufB);

  bnn::pdl_wait();  // x may come from the kernel ahead
  // x of the slice as float32, [digit i][table position p]
  for (int f = tid; f < 10 * kC5Pitch; f += kC5Threads) {
    const int i = f / kC5Pitch, p = f - kC5Pitch * i, c = c5_column(p), e = 10 * (w0 + c) + i;
    xs[f] = (c < sw && e < k) ? __uint_as_float(static_cast<uint32_t>(__ldg(x + e)) << 16) : 0.0f;
  }
  __syncthreads();
  // Tables: task = (table t, digits 2..4 of the five as b, four table positions
  // 4q..4q+3); the nine entries 9b + a (a = digits 0, 1) of each position, one
  // add each, stored four positions at a time.
  for (int f = tid; f < 2 * 27 * (kC5Pitch / 4); f += kC5Threads) {
    const int q = f % (kC5Pitch / 4), g = f / (kC5Pitch / 4), t = g / 27, b = g - 27 * t;
    const float4* xq = reinterpret_cast<const float4*>(xs + (5 * t) * kC5Pitch) + q;
    const float4 x0 = xq[0], x1 = xq[kC5Pitch / 4], x2 = xq[2 * kC5Pitch / 4], x3 = xq[3 * kC5Pitch / 4],
                 x4 = xq[4 * kC5Pitch / 4];
    const float c2 = static_cast<float>(b % 3 - 1), c3 = static_cast<float>((b / 3) % 3 - 1),
                c4 = static_cast<float>(b / 9 - 1);
    const float bx = x2.x * c2 + x3.x * c3 + x4.x * c4, by = x2.y * c2 + x3.y * c3 + x4.y * c4,
                bz = x2.z * c2 + x3.z * c3 + x4.z * c4, bw = x2.w * c2 + x3.w * c3 + x4.w * c4;
    float4* dst = reinterpret_cast<float4*>((t == 0 ? lo : hi) + (9 * b) * kC5Pitch) + q;
#pragma unroll
    for (int a = 0; a < 9; ++a) {
      float4 v;
      v.x = c5_entry(a, bx, x0.x, x1.x);
      v.y = c5_entry(a, by, x0.y, x1.y);
      v.z = c5_entry(a, bz, x0.z, x1.z);
      v.w = c5_entry(a, bw, x0.w, x1.w);
      dst[a * (kC5Pitch / 4)] = v;
    }
  }
  __syncthreads();

  const uint32_t tl = static_cast<uint32_t>(__cvta_generic_to_shared(lo)) + 4u * static_cast<uint32_t>(lane);
  // round i from the words in cur; round i + 2 is then loaded into cur
  auto step = [&](int i, C5Words<VEC> (&cur)[D]) {
    const int rl0 = i * R + warp * D;  // local row of cur[0]
    if (rl0 >= rows_c) return;
    float acc[D];
#pragma unroll
    for (int j = 0; j < D; ++j) acc[j] = c5_row<VEC>(cur[j], tl);
    if (rl0 + 2 * R < rows_c) fetch_round(i + 2, cur);
    const float v = c5_reduce<D>(acc, lane);
    const int j = lane / (32 / D);
    if ((lane & (32 / D - 1)) == 0 && rl0 + j < rows_c) psum[(rl0 + j) & (kC5Rows - 1)] = v;  // chunks start at multiples of kC5Rows
  };
  for (int cb = 0, i0 = 0; i0 < rounds; cb += kC5Rows, i0 += kRoundsPerChunk) {
    const int i1 = i0 + kRoundsPerChunk < rounds ? i0 + kRoundsPerChunk : rounds;
    for (int i = i0; i < i1; i += 2) {  // chunks hold an even number of rounds: round i's words are in bufA
      step(i, bufA);
      if (i + 1 < i1) step(i + 1, bufB);
    }
    // end of a chunk: its slice sums added in rank order by the CTA that owns the row
    cluster.sync();
    const int rows = rows_c - cb < kC5Rows ? rows_c - cb : kC5Rows;
    const int q0 = rows * rank / kC5, q1 = rows * (rank + 1) / kC5;
    for (int rl = q0 + tid; rl < q1; rl += kC5Threads) {
      float sum = 0.0f;
#pragma unroll
      for (int q = 0; q < kC5; ++q) sum += cluster.map_shared_rank(psum, q)[rl];
      const int64_t r = c0 + cb + rl;
      out[r] = bias ? __ldg(scale + r) * sum + __ldg(bias + r) : __ldg(scale + r) * sum;
    }
    cluster.sync();  // slice sums read before the next chunk overwrites them (and before any CTA exits)
  }
}

// ---------------------------------------------------------------------------
// Ternary GEMM (m > 8): trits decoded to bf16 tiles in shared memory, bf16
// mma.sync m16n8k16 with fp32 accumulation.
//
// A cluster of kTK CTAs computes one kTBM x kTBN output tile; CTA r of the
// cluster takes the r-th quarter of the packed words, so four times as many
// CTAs share the GPU and each reads only its quarter of the activations.  The
// partial tiles are added through distributed shared memory in rank order
// (0 + 1 + 2 + 3) by rank 0, which applies the scale once and writes out.
// Per 8-word (80-trit, 5 x k16) chunk: the activation tile is copied with
// 16-byte cp.async (double-buffered), and each weight word is decoded by one
// thread: five base-9 digits, each a 9-entry table lookup giving the bf16
// pair (t_2q, t_2q+1), stored as one 32-bit word.
// ---------------------------------------------------------------------------
constexpr int kTBM = 64;             // activation rows per CTA
constexpr int kTBN = 64;             // weight rows per CTA
constexpr int kTK = 4;               // CTAs per cluster, splitting the packed words
constexpr int kTCW = 8;              // words per chunk (80 trits = 5 k16 steps)
constexpr int kTCK = 10 * kTCW;      // 80 trits per chunk
constexpr int kTPitch = kTCK + 8;    // bf16 per smem row: 176 bytes, an odd multiple of 16
constexpr int kTThreads = 256;

__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                            const void* p) {
  const unsigned a = static_cast<unsigned>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(a));
}
__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

template <bool VECX>
__global__ void __cluster_dims__(kTK, 1, 1) __launch_bounds__(kTThreads)
ternary_gemm_mma_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ packed,
                        const float* __restrict__ scale, int64_t m, int64_t n, int64_t k, int64_t kt,
                        int64_t slice_words, float* __restrict__ out, const float* __restrict__ bias) {
  extern __shared__ __align__(16) uint16_t tsm[];
  uint16_t (*Xs)[kTBM * kTPitch] = reinterpret_cast<uint16_t (*)[kTBM * kTPitch]>(tsm);                // [2]
  uint16_t (*Ws)[kTBN * kTPitch] = reinterpret_cast<uint16_t (*)[kTBN * kTPitch]>(tsm + 2 * kTBM * kTPitch);  // [2]
  uint32_t* lut = reinterpret_cast<uint32_t*>(tsm + 2 * (kTBM + kTBN) * kTPitch);                     // [9]
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int wm = warp & 1;   // 2 warps along M (32 rows each)
  const int wn = warp >> 1;  // 4 warps along N (16 cols each)
  const int rank = static_cast<int>(cluster.block_rank());
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kTBM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x / kTK) * kTBN;
  const int64_t w_begin = rank * slice_words;
  const int64_t w_end = w_begin + slice_words < kt ? w_begin + slice_words : kt;
  const int64_t nchunks = w_end > w_begin ? (w_end - w_begin + kTCW - 1) / kTCW : 0;

  if (tid < 9) {
    // bf16 bit patterns of (t_lo, t_hi) for base-9 digit v = (t_lo + 1) + 3 (t_hi + 1)
    const int lo = tid % 3, hi = tid / 3;  // digit = trit + 1
    const uint32_t blo = lo == 0 ? 0xBF80u : (lo == 2 ? 0x3F80u : 0u);
    const uint32_t bhi = hi == 0 ? 0xBF80u : (hi == 2 ? 0x3F80u : 0u);
    lut[tid] = blo | (bhi << 16);
  }

  auto load_x = [&](int64_t ch, int buf) {
    const int64_t kb = 10 * (w_begin + ch * kTCW);  // first trit of the chunk
    if constexpr (VECX) {
      // 64 rows x 10 pieces of 16 bytes; pieces past k are zero-filled
      for (int c = tid; c < kTBM * (kTCK / 8); c += kTThreads) {
        const int row = c / (kTCK / 8), piece = c % (kTCK / 8);
        const int64_t gm = m0 + row, gk = kb + 8 * piece;
        int bytes = 0;
        if (gm < m && gk < k) bytes = static_cast<int>((k - gk < 8 ? k - gk : 8) * 2);
        const uint16_t* src = bytes ? x + gm * k + gk : x;
        const unsigned saddr = static_cast<unsigned>(__cvta_generic_to_shared(&Xs[buf][row * kTPitch + 8 * piece]));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(saddr), "l"(src), "r"(bytes) : "memory");
      }
    } else {
      for (int c = tid; c < kTBM * kTCK; c += kTThreads) {
        const int row = c / kTCK, col = c % kTCK;
        const int64_t gm = m0 + row, gk = kb + col;
        Xs[buf][row * kTPitch + col] = (gm < m && gk < k) ? __ldg(x + gm * k + gk) : static_cast<uint16_t>(0);
      }
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
  };

  auto decode_w = [&](int64_t ch, int buf) {
    const int64_t wb = w_begin + ch * kTCW;
    for (int c = tid; c < kTBN * kTCW; c += kTThreads) {
      const int row = c / kTCW, wj = c % kTCW;
      const int64_t gn = n0 + row, gw = wb + wj;
      uint32_t* dst = reinterpret_cast<uint32_t*>(&Ws[buf][row * kTPitch + 10 * wj]);
      if (gn < n && gw < w_end) {
        uint32_t F = static_cast<uint32_t>(__ldg(packed + gn * kt + gw)) * kFixMul;
#pragma unroll
        for (int q = 4; q >= 0; --q) {
          const uint32_t v = __umulhi(F, 9u);
          F *= 9u;
          dst[q] = lut[v];
        }
      } else {
#pragma unroll
        for (int q = 0; q < 5; ++q) dst[q] = 0u;
      }
    }
  };

  float acc[2][2][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][b][c] = 0.0f;

  __syncthreads();  // lut ready
  if (nchunks > 0) {
    load_x(0, 0);
    decode_w(0, 0);
  }
  for (int64_t ch = 0; ch < nchunks; ++ch) {
    const int buf = static_cast<int>(ch & 1);
    if (ch + 1 < nchunks) {
      load_x(ch + 1, buf ^ 1);
      asm volatile("cp.async.wait_group 1;\n" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    }
    __syncthreads();  // chunk ch's activations landed and its weights are decoded
#pragma unroll
    for (int ks = 0; ks < kTCK; ks += 16) {
      uint32_t af[2][4], bfr[4];
#pragma unroll
      for (int mi = 0; mi < 2; ++mi) {
        const int row = wm * 32 + mi * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int col = ks + 8 * (lane >> 4);
        ldmatrix_x4(af[mi][0], af[mi][1], af[mi][2], af[mi][3], &Xs[buf][row * kTPitch + col]);
      }
      {
        // matrices: (n 0-7, k 0-7), (n 0-7, k 8-15), (n 8-15, k 0-7), (n 8-15, k 8-15)
        const int row = wn * 16 + (lane & 7) + 8 * (lane >> 4);
        const int col = ks + 8 * ((lane >> 3) & 1);
        ldmatrix_x4(bfr[0], bfr[1], bfr[2], bfr[3], &Ws[buf][row * kTPitch + col]);
      }
#pragma unroll
      for (int mi = 0; mi < 2; ++mi) {
        mma_bf16_16816(acc[mi][0], af[mi], &bfr[0]);
        mma_bf16_16816(acc[mi][1], af[mi], &bfr[2]);
      }
    }
    if (ch + 1 < nchunks) decode_w(ch + 1, buf ^ 1);
    __syncthreads();  // everyone is done with buffer `buf` before it is refilled
  }

  // Partial tile -> own shared memory; rank 0 adds the cluster's partials in rank order.
  float* part = reinterpret_cast<float*>(&Xs[0][0]);  // kTBM x kTBN floats (16 KiB) fit in Xs
  const int g = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int ni = 0; ni < 2; ++ni)
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int r = wm * 32 + mi * 16 + g + 8 * h;
          const int col = wn * 16 + ni * 8 + 2 * tq + c;
          part[r * kTBN + col] = acc[mi][ni][2 * h + c];
        }
  cluster.sync();
  if (rank == 0) {
    for (int idx = tid; idx < kTBM * kTBN; idx += kTThreads) {
      const int r = idx / kTBN, col = idx % kTBN;
      const int64_t gm = m0 + r, gn = n0 + col;
      float s = part[idx];
#pragma unroll
      for (int q = 1; q < kTK; ++q) s += cluster.map_shared_rank(part, q)[idx];
      if (gm < m && gn < n) out[gm * n + gn] = bias ? __ldg(scale + gn) * s + __ldg(bias + gn) : __ldg(scale + gn) * s;
    }
  }
  cluster.sync();  // keep every CTA's partial tile alive until rank 0 has read it
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
    BNN_TRY(bnn::scratch_alloc(reinterpret_cast<void**>(&partial), static_cast<size_t>(nparts) * sizeof(double), s));
    twn_abs_partial_kernel<<<static_cast<unsigned>(nparts), kRedThreads, 0, s>>>(w, total, partial);
    const bnn_status st = bnn::check_launch();
    if (st != BNN_OK) {
      cudaFreeAsync(partial, s);
      return st;
    }
  }
  const int64_t cap = static_cast<int64_t>(bnn::sm_count()) * 8;
  const int grid = static_cast<int>(n < 1 ? 1 : (n < cap ? n : cap));
  twn_pack_rows_kernel<kModeTWN><<<grid, kRedThreads, 0, s>>>(w, n, k, partial, nparts, total, packed, scale, delta);
  bnn_status st = bnn::check_launch();
  if (partial) {
    const cudaError_t e = cudaFreeAsync(partial, s);
    if (st == BNN_OK && e != cudaSuccess) st = bnn::cuda_fail(e);
  }
  return st;
}

namespace {
// Clusters of the c5 GEMV kernel that fit the GPU at once (cached per CUDA
// context; 0 when the occupancy query fails: the other m = 1 kernels are used).
int c5_clusters() {
  static std::mutex mu;
  static uint64_t ctx_cached = 0;
  static int cached = 0;
  std::lock_guard<std::mutex> lock(mu);
  const uint64_t ctx = bnn::context_id();
  if (ctx != 0 && ctx == ctx_cached) return cached;
  int num = 0;
  if (bnn::ensure_smem(ternary_gemv_c5_kernel<true>, c5_smem_bytes()) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kC5 * 64);
    cfg.blockDim = dim3(kC5Threads);
    cfg.dynamicSmemBytes = c5_smem_bytes();
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kC5;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&num, ternary_gemv_c5_kernel<true>, &cfg) != cudaSuccess) num = 0;
  }
  cudaGetLastError();  // a failed query leaves no error behind
  cached = num;
  ctx_cached = bnn::context_id();
  return num;
}

bnn_status ternary_gemm_impl(const uint16_t* x_bf16, const uint16_t* packed, const float* scale, const float* bias,
                             int64_t m, int64_t n, int64_t k, float* out, int algo, cudaStream_t s) {
  if (algo != BNN_TALGO_AUTO && algo != BNN_TALGO_CUDA_CORES && algo != BNN_TALGO_MMA && algo != BNN_TALGO_TC)
    return BNN_ERR_INVALID_ARG;
  if (algo == BNN_TALGO_CUDA_CORES && m > 8) return BNN_ERR_UNSUPPORTED;
  if (m < 0 || n < 0 || k < 0) return BNN_ERR_INVALID_ARG;
  if (m == 0 || n == 0) return BNN_OK;
  if (!scale || !out || (k > 0 && (!x_bf16 || !packed))) return BNN_ERR_INVALID_ARG;
  if ((x_bf16 && !bnn::aligned(x_bf16, 2)) || (packed && !bnn::aligned(packed, 2)) || !bnn::aligned(scale, 4) ||
      !bnn::aligned(out, 4) || (bias && !bnn::aligned(bias, 4)))
    return BNN_ERR_MISALIGNED;
  const int64_t kt = bnn::words10(k);
  if (algo == BNN_TALGO_TC) return bnn::ternary_gemm_tc(x_bf16, packed, scale, bias, m, n, k, out, s);
  // activations TMA can copy: the tcgen05 kernels (decoding into tensor memory
  // for one activation tile, into shared memory above that)
  if (algo == BNN_TALGO_AUTO && m > 8 && k % 8 == 0 && bnn::aligned(x_bf16, 16))
    return bnn::ternary_gemm_tc(x_bf16, packed, scale, bias, m, n, k, out, s);
  // (the table kernel addresses the words with 32-bit offsets)
  if (algo != BNN_TALGO_MMA && m == 1 && kt > 0 && kt <= kC5 * kC5Pitch && (n + 512) * kt < (int64_t{1} << 31)) {
    const int clusters = c5_clusters();
    if (clusters > 0) {
      // 32-bit word pairs where every row's slices start 4-byte aligned: kt even, the slice even
      const bool vec = kt % 2 == 0 && bnn::aligned(packed, 4);
      int slice = static_cast<int>((kt + kC5 - 1) / kC5);
      if (vec) slice += slice & 1;  // at most 96: kt <= 480
      const int64_t g = (n + 63) / 64 < clusters ? (n + 63) / 64 : clusters;  // at least 64 rows per cluster
      const size_t smem = c5_smem_bytes();
      if (vec) {
        BNN_TRY(bnn::ensure_smem(ternary_gemv_c5_kernel<true>, smem));
        BNN_TRY(bnn::launch_pdl(ternary_gemv_c5_kernel<true>, dim3(static_cast<unsigned>(kC5 * g)),
                                dim3(kC5Threads), smem, s, kC5, x_bf16, packed, scale, n, static_cast<int>(k),
                                static_cast<int>(kt), slice, out, bias));
      } else {
        BNN_TRY(bnn::ensure_smem(ternary_gemv_c5_kernel<false>, smem));
        BNN_TRY(bnn::launch_pdl(ternary_gemv_c5_kernel<false>, dim3(static_cast<unsigned>(kC5 * g)),
                                dim3(kC5Threads), smem, s, kC5, x_bf16, packed, scale, n, static_cast<int>(k),
                                static_cast<int>(kt), slice, out, bias));
      }
      return bnn::check_launch();
    }
  }
  if (algo != BNN_TALGO_MMA && m == 1 && kt > 0 && rows_smem_bytes(kt) <= 200 * 1024) {
    const size_t smem = rows_smem_bytes(kt);
    BNN_TRY(bnn::ensure_smem(ternary_gemv_rows_kernel, smem));
    const int64_t sms = bnn::sm_count();
    const int grid = static_cast<int>(n < sms ? n : sms);
    BNN_TRY(bnn::launch_pdl(ternary_gemv_rows_kernel, dim3(grid), dim3(kRowThreads), smem, s, 1, x_bf16, packed,
                            scale, n, static_cast<int>(k), static_cast<int>(kt), out, bias));
    return bnn::check_launch();
  }
  if (algo != BNN_TALGO_MMA && m <= 8) {
    const int64_t warps_per_block = 8;
    const int64_t blocks_needed = (n + warps_per_block - 1) / warps_per_block;
    const int64_t cap = static_cast<int64_t>(bnn::sm_count()) * 8;
    const int grid = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
    if (m == 1) ternary_gemv_kernel<1><<<grid, 256, 0, s>>>(x_bf16, packed, scale, 1, n, k, kt, out, bias);
    else if (m <= 4)
      ternary_gemv_kernel<4><<<grid, 256, 0, s>>>(x_bf16, packed, scale, static_cast<int>(m), n, k, kt, out, bias);
    else ternary_gemv_kernel<8><<<grid, 256, 0, s>>>(x_bf16, packed, scale, static_cast<int>(m), n, k, kt, out, bias);
    return bnn::check_launch();
  }
  const int64_t ntiles = (n + kTBN - 1) / kTBN, gy = (m + kTBM - 1) / kTBM;
  if (ntiles * kTK > 2147483647LL || gy > 65535) return BNN_ERR_INVALID_ARG;
  // each cluster rank takes a whole number of chunks
  const int64_t per = (kt + kTK - 1) / kTK;
  const int64_t slice_words = (per + kTCW - 1) / kTCW * kTCW;
  const dim3 grid(static_cast<unsigned>(ntiles * kTK), static_cast<unsigned>(gy));
  const size_t smem = 2 * static_cast<size_t>(kTBM + kTBN) * kTPitch * sizeof(uint16_t) + 9 * sizeof(uint32_t);
  if (k % 8 == 0 && bnn::aligned(x_bf16, 16)) {
    BNN_TRY(bnn::ensure_smem(ternary_gemm_mma_kernel<true>, smem));
    ternary_gemm_mma_kernel<true><<<grid, kTThreads, smem, s>>>(x_bf16, packed, scale, m, n, k, kt, slice_words, out,
                                                                bias);
  } else {
    BNN_TRY(bnn::ensure_smem(ternary_gemm_mma_kernel<false>, smem));
    ternary_gemm_mma_kernel<false><<<grid, kTThreads, smem, s>>>(x_bf16, packed, scale, m, n, k, kt, slice_words, out,
                                                                 bias);
  }
  return bnn::check_launch();
}
}  // namespace

extern "C" bnn_status bnn_ternary_gemm_algo(const uint16_t* x_bf16, const uint16_t* packed, const float* scale,
                                            int64_t m, int64_t n, int64_t k, float* out, int algo, cudaStream_t s) {
  return ternary_gemm_impl(x_bf16, packed, scale, nullptr, m, n, k, out, algo, s);
}

extern "C" bnn_status bnn_ternary_linear(const uint16_t* x_bf16, const uint16_t* packed, const float* scale,
                                         const float* bias, int64_t m, int64_t n, int64_t k, float* out,
                                         cudaStream_t s) {
  return ternary_gemm_impl(x_bf16, packed, scale, bias, m, n, k, out, BNN_TALGO_AUTO, s);
}

extern "C" bnn_status bnn_ternary_gemm(const uint16_t* x_bf16, const uint16_t* packed, const float* scale,
                                       int64_t m, int64_t n, int64_t k, float* out, cudaStream_t s) {
  return bnn_ternary_gemm_algo(x_bf16, packed, scale, m, n, k, out, BNN_TALGO_AUTO, s);
}

// ---------------------------------------------------------------------------
// bnn_ternary_pack_noalloc: the same TWN pack with its scratch in a fixed
// device array instead of memory taken from an allocator.
//
// The float64 partial sums of |W| (one per 65536 weights) live in the
// file-scope array below, which every GPU that loads this library holds
// until the process exits.  Its host-side name is only a stand-in for the
// symbol; the device address comes from cudaGetSymbolAddress, looked up on
// the first call in each CUDA context (with that device current) and cached.
// ---------------------------------------------------------------------------
constexpr int64_t kNoAllocMaxParts = 8192;  // 64 KiB of float64: up to 8192 * 65536 = 2^29 weights

static __device__ __align__(256) double g_twn_noalloc_partials[kNoAllocMaxParts];

namespace {

constexpr int kNoAllocMaxDevices = 64;
struct NoAllocSlot {
  uint64_t ctx;  // bnn::context_id() the address was looked up in
  double* ptr;
};
NoAllocSlot g_noalloc[kNoAllocMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of g_twn_noalloc_partials on the current device.  Looked up
// with cudaGetSymbolAddress on the first call in each CUDA context (with the
// device current) and cached for that context: after a device reset the
// context, and so the id, is new, and the address is looked up again.
bnn_status noalloc_scratch(double** out) {
  int dev = -1;
  BNN_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNoAllocMaxDevices) return BNN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  const uint64_t ctx = bnn::context_id();
  if (ctx == 0 || g_noalloc[dev].ctx != ctx || !g_noalloc[dev].ptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_twn_noalloc_partials);
    if (e != cudaSuccess) return bnn::cuda_fail(e);
    g_noalloc[dev] = NoAllocSlot{bnn::context_id(), static_cast<double*>(p)};
  }
  *out = g_noalloc[dev].ptr;
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
  twn_pack_rows_kernel<kModeTWN><<<grid, kRedThreads, 0, s>>>(w, n, k, partial, nparts, total, packed, scale, delta);
  return bnn::check_launch();
}

// ---------------------------------------------------------------------------
// bnn_ternary_pack_mode: the other ternarisation rules of the pages.
// ---------------------------------------------------------------------------
extern "C" bnn_status bnn_ternary_pack_mode(const float* w, int64_t n, int64_t k, int mode, float threshold,
                                            uint16_t* packed, float* scale, float* thresh_out, cudaStream_t s) {
  if (mode != kModeTWN && mode != kModeAbsmean && mode != kModeDelta) return BNN_ERR_INVALID_ARG;
  if (mode == kModeTWN) return bnn_ternary_pack(w, n, k, packed, scale, thresh_out, s);
  if (mode == kModeDelta && !(threshold >= 0.0f)) return BNN_ERR_INVALID_ARG;  // NaN or negative
  if (n < 0 || k < 0) return BNN_ERR_INVALID_ARG;
  if (!thresh_out) return BNN_ERR_INVALID_ARG;
  if (n > 0 && !scale) return BNN_ERR_INVALID_ARG;
  if (n > 0 && k > 0 && (!w || !packed)) return BNN_ERR_INVALID_ARG;
  if (k > 0 && n > (int64_t(1) << 40) / k) return BNN_ERR_INVALID_ARG;
  if ((w && !bnn::aligned(w, 4)) || (packed && !bnn::aligned(packed, 2)) || (scale && !bnn::aligned(scale, 4)) ||
      !bnn::aligned(thresh_out, 4))
    return BNN_ERR_MISALIGNED;
  const int64_t total = n * k;
  const int64_t cap = static_cast<int64_t>(bnn::sm_count()) * 8;
  const int grid = static_cast<int>(n < 1 ? 1 : (n < cap ? n : cap));
  if (mode == kModeDelta) {
    twn_pack_rows_kernel<kModeDelta><<<grid, kRedThreads, 0, s>>>(w, n, k, nullptr, 0, total, packed, scale,
                                                                  thresh_out, threshold);
    return bnn::check_launch();
  }
  const int64_t nparts = (total + kChunk - 1) / kChunk;
  double* partial = nullptr;
  if (nparts > 0) {
    BNN_TRY(bnn::scratch_alloc(reinterpret_cast<void**>(&partial), static_cast<size_t>(nparts) * sizeof(double), s));
    twn_abs_partial_kernel<<<static_cast<unsigned>(nparts), kRedThreads, 0, s>>>(w, total, partial);
    const bnn_status st = bnn::check_launch();
    if (st != BNN_OK) {
      cudaFreeAsync(partial, s);
      return st;
    }
  }
  twn_pack_rows_kernel<kModeAbsmean><<<grid, kRedThreads, 0, s>>>(w, n, k, partial, nparts, total, packed, scale,
                                                                  thresh_out);
  bnn_status st = bnn::check_launch();
  if (partial) {
    const cudaError_t e = cudaFreeAsync(partial, s);
    if (st == BNN_OK && e != cudaSuccess) st = bnn::cuda_fail(e);
  }
  return st;
}
