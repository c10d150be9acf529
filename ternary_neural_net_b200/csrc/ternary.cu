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
// Ternary GEMV, m = 1, k <= 4160: activation tables over 4 + 3 + 3 trits.
//
// A word's ten trits split into a 4-trit group (digits 0..3, the word mod 81),
// a 3-trit group (digits 4..6) and a 3-trit group (digits 7..9).  For word
// position j of the rows, table A_j holds, for each of the 81 digit patterns
// e of the first group, the partial dot sum_{i<4} x[10j+i] (d_i(e) - 1); B_j
// and C_j (27 patterns each) the same for the other two groups.  A word then
// costs three shared-memory loads and three adds: y = scale * sum_j
// (A_j[e_A] + B_j[e_B] + C_j[e_C]).  The group codes come from two exact
// multiply-shift divisions (by 81, then by 27; the constants are checked
// against every word at compile time below).
//
// One CTA per SM holds all 135 tables of the row length (135 x ktp floats,
// ktp = kt rounded up to 32: 218 KiB at k = 4096) and takes a contiguous
// block of rows.  Work unit = (row, pass): a warp's 32 lanes load 32
// consecutive 32-bit pairs of words of one row (128 coalesced bytes), so
// lane l of pass p holds words j = 64p + 2l + t, t = 0, 1.  Tables are stored
// entry-major with word column sigma(j) = 64p + t L + l (L = the pass's lane
// count), so for each of the six loads of a unit the 32 lanes read 32
// consecutive columns: 32 different banks, whatever patterns they decode.
// Lanes past the row's end decode the all-zero-trit pair, whose entries are 0
// in every column.  Each unit's lane sums are added by a shuffle tree and
// stored per (row, pass); the rows' pass sums are added in pass order, so the
// result does not depend on the launch shape.  Eight units per warp are in
// flight (their words loaded a group ahead); the first group is loaded
// before the programmatic-launch wait (weights do not depend on the kernel
// ahead), the tables are built after it (they depend on x).
// ---------------------------------------------------------------------------
constexpr int kLutThreads = 1024;
constexpr int kLutMaxKt = 416;         // 32-bit pairs of words need kt even; 135 x 416 floats = 219.4 KiB
constexpr int kLutRowsChunk = 256;     // rows whose unit sums are held at once
constexpr int kLutMaxPasses = (kLutMaxKt / 2 + 31) / 32;
constexpr int kLutMaxUnits = (kLutMaxPasses + 1) / 2;  // units (two passes each) per row
constexpr int kLutGroup = 4;           // units per warp in flight (two 32-bit loads each)
constexpr uint32_t kDiv81Mul = 25891u, kDiv81Shift = 21;  // floor(w / 81) for w < 3^10
constexpr uint32_t kDiv27Mul = 607u, kDiv27Shift = 14;    // floor(q / 27) for q < 3^6
constexpr uint32_t kZeroPair = 29524u | (29524u << 16);   // two all-zero-trit words

constexpr bool lut_divisions_exact() {
  for (uint32_t w = 0; w < 59049u; ++w)
    if ((w * kDiv81Mul) >> kDiv81Shift != w / 81u) return false;
  for (uint32_t q = 0; q < 729u; ++q)
    if ((q * kDiv27Mul) >> kDiv27Shift != q / 27u) return false;
  return true;
}
static_assert(lut_divisions_exact(), "multiply-shift division constants");

__host__ __device__ constexpr int lut_pitch(int kt) { return (kt + 31) & ~31; }

size_t lut_smem_bytes(int64_t kt) {
  return static_cast<size_t>(135 * lut_pitch(static_cast<int>(kt)) + kLutRowsChunk * kLutMaxUnits) * sizeof(float);
}

__device__ __forceinline__ float bf16f(const uint16_t* x, int e, int k) {
  return e < k ? __uint_as_float(static_cast<uint32_t>(__ldg(x + e)) << 16) : 0.0f;
}

// One word's three table entries, summed: colA/colB/colC are the byte
// addresses of the word's column in tables A, B and C, stride one entry row.
__device__ __forceinline__ float lut_word(uint32_t w, uint32_t colA, uint32_t colB, uint32_t colC, uint32_t stride) {
  const uint32_t q = (w * kDiv81Mul) >> kDiv81Shift;   // digits 4..9
  const uint32_t eA = w - 81u * q;                     // digits 0..3
  const uint32_t eC = (q * kDiv27Mul) >> kDiv27Shift;  // digits 7..9
  const uint32_t eB = q - 27u * eC;                    // digits 4..6
  float a, b, c;
  asm volatile("ld.shared.f32 %0, [%1];\n" : "=f"(a) : "r"(colA + eA * stride));
  asm volatile("ld.shared.f32 %0, [%1];\n" : "=f"(b) : "r"(colB + eB * stride));
  asm volatile("ld.shared.f32 %0, [%1];\n" : "=f"(c) : "r"(colC + eC * stride));
  return (a + b) + c;
}

__global__ void __launch_bounds__(kLutThreads, 1)
ternary_gemv_lut_kernel(const uint16_t* __restrict__ x, const uint32_t* __restrict__ packed2,
                        const float* __restrict__ scale, int64_t n, int k, int kt, float* __restrict__ out,
                        const float* __restrict__ bias) {
  extern __shared__ float T[];  // [135][ktp] tables, then [kLutRowsChunk][units per row] unit sums
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = kLutThreads / 32;
  const int ktp = lut_pitch(kt);
  const int kt2 = kt >> 1;                       // 32-bit pairs per row
  const int passes = (kt2 + 31) >> 5;            // 32 pairs (64 words) per pass
  const int upr = (passes + 1) >> 1;             // units per row: passes 2u and 2u + 1
  const int l_last = kt2 - 32 * (passes - 1);    // lanes of the last pass
  float* usum = T + 135 * ktp;
  const int64_t r_begin = n * blockIdx.x / gridDim.x, r_end = n * (blockIdx.x + 1) / gridDim.x;
  // warp-uniform walk over the units u = warp + kWarps i as (row, unit-of-row) pairs
  const int d_row = kWarps / upr, d_unit = kWarps - d_row * upr;
  auto advance = [&](int& rl, int& ur) {
    ur += d_unit;
    rl += d_row;
    if (ur >= upr) {
      ur -= upr;
      ++rl;
    }
  };
  bnn::pdl_trigger();

  // this lane's pairs of unit (rl, ur): passes 2 ur and 2 ur + 1 (zero pairs past the row);
  // offsets in 32 bits (the host keeps n * kt / 2 below 2^31)
  auto fetch = [&](int64_t r_chunk, int rows, int rl, int ur, uint32_t& v0, uint32_t& v1) {
    v0 = v1 = kZeroPair;
    if (rl < rows) {
      const int c = 64 * ur + lane;
      const uint32_t* src = packed2 + static_cast<uint32_t>(static_cast<int>(r_chunk) + rl) * static_cast<uint32_t>(kt2) + c;
      if (c < kt2) v0 = __ldcs(src);
      if (c + 32 < kt2) v1 = __ldcs(src + 32);
    }
  };

  int64_t r_chunk = r_begin;
  int rows = static_cast<int>(r_end - r_begin < kLutRowsChunk ? r_end - r_begin : kLutRowsChunk);
  int rl0 = warp / upr, ur0 = warp - rl0 * upr;  // the warp's first unit
  uint32_t cur[kLutGroup][2];
  int frl = rl0, fur = ur0;  // fetch cursor (runs kLutGroup units ahead of the compute cursor)
#pragma unroll
  for (int g = 0; g < kLutGroup; ++g) {
    fetch(r_chunk, rows, frl, fur, cur[g][0], cur[g][1]);
    advance(frl, fur);
  }

  bnn::pdl_wait();  // x may come from the kernel ahead
  // Tables.  Task f = part * kt + column: parts 0..8 fill A's entries
  // 9 part .. 9 part + 8, parts 9..11 B's, 12..14 C's.  Consecutive threads
  // write consecutive columns of one entry row (distinct banks).
  for (int f = tid; f < 15 * kt; f += kLutThreads) {
    const int part = f / kt, c = f - part * kt;
    const int p = c >> 6, o = c & 63;
    const int L = kt2 - 32 * p < 32 ? kt2 - 32 * p : 32;
    const int t = o >= L ? 1 : 0, l = o - t * L;
    const int j = 64 * p + 2 * l + t;          // the word position stored in column c
    const int e0 = 10 * j;
    float lo[9];
    float hi;
    int row0;
    if (part < 9) {                             // A: digits 0, 1 run over e_lo; digits 2, 3 fixed by part
      const float x0 = bf16f(x, e0, k), x1 = bf16f(x, e0 + 1, k);
      const float x2 = bf16f(x, e0 + 2, k), x3 = bf16f(x, e0 + 3, k);
#pragma unroll
      for (int v = 0; v < 9; ++v) lo[v] = x0 * static_cast<float>(v % 3 - 1) + x1 * static_cast<float>(v / 3 - 1);
      hi = x2 * static_cast<float>(part % 3 - 1) + x3 * static_cast<float>(part / 3 - 1);
      row0 = 9 * part;
    } else {                                    // B (digits 4..6) or C (digits 7..9): last digit fixed by part
      const int g = part < 12 ? 0 : 1, d = part - 9 - 3 * g;
      const int b = e0 + 4 + 3 * g;
      const float x0 = bf16f(x, b, k), x1 = bf16f(x, b + 1, k), x2 = bf16f(x, b + 2, k);
#pragma unroll
      for (int v = 0; v < 9; ++v) lo[v] = x0 * static_cast<float>(v % 3 - 1) + x1 * static_cast<float>(v / 3 - 1);
      hi = x2 * static_cast<float>(d - 1);
      row0 = 81 + 27 * g + 9 * d;
    }
    float* dst = T + row0 * ktp + c;
#pragma unroll
    for (int v = 0; v < 9; ++v) dst[v * ktp] = lo[v] + hi;
  }
  __syncthreads();

  const uint32_t stride = 4u * static_cast<uint32_t>(ktp);
  const uint32_t tA = static_cast<uint32_t>(__cvta_generic_to_shared(T));
  const uint32_t offB = 81u * stride, offC = 108u * stride;
  const uint32_t lane_full = 4u * static_cast<uint32_t>(lane);
  const uint32_t lane_last = 4u * static_cast<uint32_t>(lane < l_last ? lane : l_last - 1);  // valid column
  // the two words of pair v in pass p (warp-uniform p), added to acc
  auto pass_sum = [&](uint32_t v, int p) -> float {
    const bool last = p == passes - 1;
    const uint32_t c0 = tA + 256u * static_cast<uint32_t>(p) + (last ? lane_last : lane_full);
    const uint32_t c1 = c0 + 4u * static_cast<uint32_t>(last ? l_last : 32);
    return lut_word(v & 0xFFFFu, c0, c0 + offB, c0 + offC, stride) +
           lut_word(v >> 16, c1, c1 + offB, c1 + offC, stride);
  };

  while (true) {
    int rl = rl0, ur = ur0;
    while (rl < rows) {
      uint32_t nxt[kLutGroup][2];
#pragma unroll
      for (int g = 0; g < kLutGroup; ++g) {
        fetch(r_chunk, rows, frl, fur, nxt[g][0], nxt[g][1]);
        advance(frl, fur);
      }
      float sum[kLutGroup];
      int idx[kLutGroup];
#pragma unroll
      for (int g = 0; g < kLutGroup; ++g) {
        idx[g] = -1;
        sum[g] = 0.0f;
        if (rl < rows) {  // warp-uniform: units past the chunk's rows cost nothing
          idx[g] = rl * upr + ur;
          const int p = 2 * ur;
          sum[g] = pass_sum(cur[g][0], p);
          if (p + 1 < passes) sum[g] += pass_sum(cur[g][1], p + 1);
        }
        advance(rl, ur);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int g = 0; g < kLutGroup; ++g) sum[g] += __shfl_xor_sync(0xffffffffu, sum[g], off);
      if (lane == 0) {
#pragma unroll
        for (int g = 0; g < kLutGroup; ++g)
          if (idx[g] >= 0) usum[idx[g]] = sum[g];
      }
#pragma unroll
      for (int g = 0; g < kLutGroup; ++g) {
        cur[g][0] = nxt[g][0];
        cur[g][1] = nxt[g][1];
      }
    }
    __syncthreads();  // every unit sum of this chunk is stored
    for (int r = tid; r < rows; r += kLutThreads) {
      float acc = 0.0f;
      for (int u = 0; u < upr; ++u) acc += usum[r * upr + u];
      const int64_t gr = r_chunk + r;
      out[gr] = bias ? __ldg(scale + gr) * acc + __ldg(bias + gr) : __ldg(scale + gr) * acc;
    }
    r_chunk += rows;
    if (r_chunk >= r_end) break;
    __syncthreads();  // unit sums read before the next chunk overwrites them
    rows = static_cast<int>(r_end - r_chunk < kLutRowsChunk ? r_end - r_chunk : kLutRowsChunk);
    frl = rl0;
    fur = ur0;
#pragma unroll
    for (int g = 0; g < kLutGroup; ++g) {
      fetch(r_chunk, rows, frl, fur, cur[g][0], cur[g][1]);
      advance(frl, fur);
    }
  }
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
// tables (two [243][96] float arrays, 182 KiB), and every CTA of the cluster
// runs over the same block of rows: a warp takes whole rows, its 32 lanes
// consecutive word positions (so a lookup's 32 lanes read 32 consecutive
// columns: 32 banks), one 16-bit load per word, the next row's words in
// registers while this row is added.  Each row's slice sum (a shuffle tree) is
// stored in the CTA's shared memory; after a cluster barrier CTA q adds, for
// its share of the block's rows, the kC5 slice sums in rank order through
// distributed shared memory, scales once and writes.  Deterministic for a
// given launch shape.  The first row's words are loaded before the
// programmatic-launch wait, the tables (which depend on x) after it.
// ---------------------------------------------------------------------------
constexpr int kC5 = 5;                 // CTAs per cluster (slices of the row)
constexpr int kC5Threads = 1024;
constexpr int kC5Pitch = 96;           // table columns (word positions) per slice; a multiple of 32
constexpr int kC5Rows = 1024;          // rows of a block (slice sums held at once)
constexpr uint32_t kDiv243Mul = 69043u, kDiv243Shift = 24;  // floor(w / 243) for w < 3^10

constexpr bool div243_exact() {
  for (uint32_t w = 0; w < 59049u; ++w)
    if ((w * kDiv243Mul) >> kDiv243Shift != w / 243u) return false;
  return true;
}
static_assert(div243_exact(), "multiply-shift division by 243");

size_t c5_smem_bytes() { return (2u * 243u * kC5Pitch + kC5Rows) * sizeof(float); }

__global__ void __launch_bounds__(kC5Threads, 1)
ternary_gemv_c5_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ packed,
                       const float* __restrict__ scale, int64_t n, int k, int kt, int slice, int64_t block_rows,
                       float* __restrict__ out, const float* __restrict__ bias) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ float c5sm[];  // lo [243][kC5Pitch], hi [243][kC5Pitch], slice sums [kC5Rows]
  float* const lo = c5sm;
  float* const hi = c5sm + 243 * kC5Pitch;
  float* const psum = c5sm + 2 * 243 * kC5Pitch;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = kC5Threads / 32;
  const int rank = static_cast<int>(cluster.block_rank());
  const int64_t cl = blockIdx.x / kC5, nclusters = gridDim.x / kC5;
  const int w0 = rank * slice;                                  // this CTA's first word position
  const int sw = kt - w0 < slice ? (kt - w0 > 0 ? kt - w0 : 0) : slice;  // its word count (<= kC5Pitch)
  const int64_t nblocks = (n + block_rows - 1) / block_rows;
  bnn::pdl_trigger();

  // the words of row r at positions w0 + lane + 32 p (29524 = all-zero trits past the slice)
  auto fetch = [&](int64_t r, bool live, uint32_t (&v)[3]) {
#pragma unroll
    for (int p = 0; p < 3; ++p) {
      const int o = lane + 32 * p;
      v[p] = (live && o < sw) ? static_cast<uint32_t>(__ldcs(packed + r * kt + w0 + o)) : 29524u;
    }
  };
  int64_t blk = cl;
  int64_t b0 = blk * block_rows;
  int64_t b1 = b0 + block_rows < n ? b0 + block_rows : n;
  uint32_t cur[3];
  fetch(b0 + warp, blk < nblocks && b0 + warp < b1, cur);

  bnn::pdl_wait();  // x may come from the kernel ahead
  // Tables: task = (table t, high digits e_hi of the 5, word position o), nine
  // entries each (the two low digits run over 0..8); consecutive threads take
  // consecutive positions of one entry row (distinct banks).  Every column is
  // built, those past the slice with x = 0 (all their entries 0), since the
  // lanes past the slice look up the all-zero-trit word there.
  for (int f = tid; f < 2 * 27 * kC5Pitch; f += kC5Threads) {
    const int o = f % kC5Pitch, g = f / kC5Pitch, t = g / 27, eh = g - 27 * t;
    const int e0 = 10 * (w0 + o) + 5 * t;
    float xv[5];
#pragma unroll
    for (int i = 0; i < 5; ++i)
      xv[i] = (o < sw && e0 + i < k) ? __uint_as_float(static_cast<uint32_t>(__ldg(x + e0 + i)) << 16) : 0.0f;
    const float base = xv[2] * static_cast<float>(eh % 3 - 1) + xv[3] * static_cast<float>((eh / 3) % 3 - 1) +
                       xv[4] * static_cast<float>(eh / 9 - 1);
    float* dst = (t == 0 ? lo : hi) + (9 * eh) * kC5Pitch + o;
#pragma unroll
    for (int v = 0; v < 9; ++v)
      dst[v * kC5Pitch] = (xv[0] * static_cast<float>(v % 3 - 1) + xv[1] * static_cast<float>(v / 3 - 1)) + base;
  }
  __syncthreads();

  const uint32_t stride = 4u * kC5Pitch;
  const uint32_t lo_lane = static_cast<uint32_t>(__cvta_generic_to_shared(lo)) + 4u * static_cast<uint32_t>(lane);
  const uint32_t hi_lane = static_cast<uint32_t>(__cvta_generic_to_shared(hi)) + 4u * static_cast<uint32_t>(lane);
  for (; blk < nblocks; blk += nclusters) {
    const int rows = static_cast<int>(b1 - b0);
    for (int rl = warp; rl < rows; rl += kWarps) {
      // the next row of this warp (in this block, else the first of the next block)
      int64_t nr = b0 + rl + kWarps;
      bool nlive = rl + kWarps < rows;
      if (!nlive) {
        const int64_t nb = blk + nclusters;
        nr = nb * block_rows + warp;
        nlive = nb < nblocks && nr < (nb * block_rows + block_rows < n ? nb * block_rows + block_rows : n);
      }
      uint32_t nxt[3];
      fetch(nr, nlive, nxt);
      float acc = 0.0f;
#pragma unroll
      for (int p = 0; p < 3; ++p) {
        const uint32_t w = cur[p];
        const uint32_t qh = (w * kDiv243Mul) >> kDiv243Shift;  // digits 5..9
        const uint32_t ql = w - 243u * qh;                     // digits 0..4
        float a, b;
        asm volatile("ld.shared.f32 %0, [%1];\n" : "=f"(a) : "r"(lo_lane + 128u * p + ql * stride));
        asm volatile("ld.shared.f32 %0, [%1];\n" : "=f"(b) : "r"(hi_lane + 128u * p + qh * stride));
        acc += a + b;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) psum[rl] = acc;
#pragma unroll
      for (int p = 0; p < 3; ++p) cur[p] = nxt[p];
    }
    cluster.sync();  // every CTA's slice sums of this block are stored
    // this CTA finalises rows [q0, q1) of the block: slice sums added in rank order
    const int q0 = rows * rank / kC5, q1 = rows * (rank + 1) / kC5;
    for (int rl = q0 + tid; rl < q1; rl += kC5Threads) {
      float sum = 0.0f;
#pragma unroll
      for (int q = 0; q < kC5; ++q) sum += cluster.map_shared_rank(psum, q)[rl];
      const int64_t r = b0 + rl;
      out[r] = bias ? __ldg(scale + r) * sum + __ldg(bias + r) : __ldg(scale + r) * sum;
    }
    cluster.sync();  // slice sums read before the next block overwrites them (and before any CTA exits)
    b0 = (blk + nclusters) * block_rows;
    b1 = b0 + block_rows < n ? b0 + block_rows : n;
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
  if (bnn::ensure_smem(ternary_gemv_c5_kernel, c5_smem_bytes()) == cudaSuccess) {
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
    if (cudaOccupancyMaxActiveClusters(&num, ternary_gemv_c5_kernel, &cfg) != cudaSuccess) num = 0;
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
  if (algo != BNN_TALGO_MMA && m == 1 && kt > 0 && kt <= kC5 * kC5Pitch) {
    const int clusters = c5_clusters();
    if (clusters > 0) {
      const int slice = static_cast<int>((kt + kC5 - 1) / kC5);
      const int64_t g = (n + 63) / 64 < clusters ? (n + 63) / 64 : clusters;  // at least 64 rows per cluster
      int64_t block_rows = (n + g - 1) / g;
      if (block_rows > kC5Rows) block_rows = kC5Rows;
      const size_t smem = c5_smem_bytes();
      BNN_TRY(bnn::ensure_smem(ternary_gemv_c5_kernel, smem));
      BNN_TRY(bnn::launch_pdl(ternary_gemv_c5_kernel, dim3(static_cast<unsigned>(kC5 * g)), dim3(kC5Threads), smem, s,
                              kC5, x_bf16, packed, scale, n, static_cast<int>(k), static_cast<int>(kt), slice,
                              block_rows, out, bias));
      return bnn::check_launch();
    }
  }
  if (algo != BNN_TALGO_MMA && m == 1 && kt > 0 && kt <= kLutMaxKt && kt % 2 == 0 && bnn::aligned(packed, 4) &&
      n * (kt / 2) < (int64_t{1} << 31)) {
    const size_t smem = lut_smem_bytes(kt);
    BNN_TRY(bnn::ensure_smem(ternary_gemv_lut_kernel, smem));
    const int64_t sms = bnn::sm_count();
    const int grid = static_cast<int>(n < sms ? n : sms);
    BNN_TRY(bnn::launch_pdl(ternary_gemv_lut_kernel, dim3(grid), dim3(kLutThreads), smem, s, 1, x_bf16,
                            reinterpret_cast<const uint32_t*>(packed), scale, n, static_cast<int>(k),
                            static_cast<int>(kt), out, bias));
    return bnn::check_launch();
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
    BNN_TRY(cudaMallocAsync(reinterpret_cast<void**>(&partial), static_cast<size_t>(nparts) * sizeof(double), s));
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
