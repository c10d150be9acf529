// bnn_binary_gemm: packed XOR + popcount matmul with a per-output-channel scale.
//
// "Binary Math Effectiveness -- why / how / when", section 1: for +-1 vectors
// packed with bit 1 = -1, <x,w> = n - 2 * popcount(x XOR w) over the logical n
// (pad bits are 0 in both operands, so they never count); "Edge cases": n = 0
// gives 0, alpha = 0 gives 0.  "Architecture Decision Record", "Decision":
// binary_gemm_u64 over uint64 words.
//
// Two kernels:
//  * skinny (m <= 8): batch-1 GEMV shapes are HBM-bound on the weight stream.
//    A group of LPR lanes owns one weight row, reads it with 16-byte loads
//    (8-byte when the rows are not 16-byte aligned), XORs it with the
//    activation words (read through the read-only path, L1-resident) and
//    popcounts; R rows per group are in flight at once.  Shuffle reduction
//    within the group, fused alpha epilogue.
//  * tiled (m > 8): compute-bound on the integer pipe.  CTA tile BM x BN of
//    outputs, 16 x 16 threads each owning TM x TN outputs strided by 16 (so the
//    operand reads from shared memory are broadcast or conflict-free), operand
//    tiles of BK words per row staged through shared memory with cp.async in a
//    STAGES-deep ring (rows padded to an odd multiple of 16 bytes), int32
//    accumulators, fused k - 2d and alpha epilogue.
#include "bnn_internal.cuh"

namespace {

// ---------------------------------------------------------------------------
// skinny kernel
// ---------------------------------------------------------------------------
template <int VEC, int LPR, int R, int MT>
__global__ void __launch_bounds__(256)
binary_gemv_kernel(const uint64_t* __restrict__ xp, const uint64_t* __restrict__ wp,
                   const float* __restrict__ alpha, int m, int64_t n, int k, int kw,
                   int32_t* __restrict__ dots, float* __restrict__ out) {
  static_assert(VEC == 1 || VEC == 2, "VEC");
  constexpr int GROUPS_PER_WARP = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPR;                 // lane within its row group
  const int grp = lane / LPR;                 // row group within the warp
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t rows_per_warp_iter = static_cast<int64_t>(GROUPS_PER_WARP) * R;

  for (int64_t row0 = warp * rows_per_warp_iter; row0 < n; row0 += nwarps * rows_per_warp_iter) {
    uint32_t acc[R][MT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int t = 0; t < MT; ++t) acc[r][t] = 0;

    for (int w = sub * VEC; w < kw; w += LPR * VEC) {
      uint64_t wv[R][VEC];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int64_t row = row0 + static_cast<int64_t>(r) * GROUPS_PER_WARP + grp;
        if (row < n) {
          const uint64_t* p = wp + row * kw + w;
          if constexpr (VEC == 2) {
            const ulonglong2 v = __ldcs(reinterpret_cast<const ulonglong2*>(p));
            wv[r][0] = v.x;
            wv[r][VEC - 1] = v.y;
          } else {
            wv[r][0] = __ldcs(p);
          }
        } else {
#pragma unroll
          for (int v = 0; v < VEC; ++v) wv[r][v] = 0;
        }
      }
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        if (t < m) {
          uint64_t xv[VEC];
          if constexpr (VEC == 2) {
            const ulonglong2 v = __ldg(reinterpret_cast<const ulonglong2*>(xp + static_cast<int64_t>(t) * kw + w));
            xv[0] = v.x;
            xv[VEC - 1] = v.y;
          } else {
            xv[0] = __ldg(xp + static_cast<int64_t>(t) * kw + w);
          }
#pragma unroll
          for (int r = 0; r < R; ++r)
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[r][t] += __popcll(wv[r][v] ^ xv[v]);
        }
      }
    }
    // Reduce within each LPR-lane group.
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int t = 0; t < MT; ++t)
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) acc[r][t] += __shfl_xor_sync(0xffffffffu, acc[r][t], off);
    if (sub == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int64_t row = row0 + static_cast<int64_t>(r) * GROUPS_PER_WARP + grp;
        if (row >= n) continue;
        const float a = out ? alpha[row] : 0.0f;
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          if (t < m) {
            const int32_t d = k - 2 * static_cast<int32_t>(acc[r][t]);
            if (dots) dots[static_cast<int64_t>(t) * n + row] = d;
            if (out) out[static_cast<int64_t>(t) * n + row] = a * static_cast<float>(d);
          }
        }
      }
    }
  }
}

template <int VEC, int LPR, int R, int MT>
void launch_gemv(const uint64_t* xp, const uint64_t* wp, const float* alpha, int m, int64_t n, int k,
                 int kw, int32_t* dots, float* out, cudaStream_t s) {
  constexpr int threads = 256;
  constexpr int64_t rows_per_block = (threads / 32) * (32 / LPR) * R;
  const int64_t blocks_needed = (n + rows_per_block - 1) / rows_per_block;
  const int64_t cap = static_cast<int64_t>(bnn::sm_count()) * 8;
  const int grid = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
  binary_gemv_kernel<VEC, LPR, R, MT><<<grid, threads, 0, s>>>(xp, wp, alpha, m, n, k, kw, dots, out);
}

template <int VEC>
void dispatch_gemv(const uint64_t* xp, const uint64_t* wp, const float* alpha, int m, int64_t n, int k,
                   int kw, int32_t* dots, float* out, cudaStream_t s) {
  // Lanes per row: enough to cover a row in one pass where possible, at least 8.
  const int chunks = (kw + VEC - 1) / VEC;
  if (m <= 1) {
    if (chunks <= 8) launch_gemv<VEC, 8, 2, 1>(xp, wp, alpha, m, n, k, kw, dots, out, s);
    else if (chunks <= 16) launch_gemv<VEC, 16, 2, 1>(xp, wp, alpha, m, n, k, kw, dots, out, s);
    else launch_gemv<VEC, 32, 2, 1>(xp, wp, alpha, m, n, k, kw, dots, out, s);
  } else if (m <= 2) {
    if (chunks <= 8) launch_gemv<VEC, 8, 2, 2>(xp, wp, alpha, m, n, k, kw, dots, out, s);
    else launch_gemv<VEC, 32, 2, 2>(xp, wp, alpha, m, n, k, kw, dots, out, s);
  } else if (m <= 4) {
    if (chunks <= 8) launch_gemv<VEC, 8, 2, 4>(xp, wp, alpha, m, n, k, kw, dots, out, s);
    else launch_gemv<VEC, 32, 2, 4>(xp, wp, alpha, m, n, k, kw, dots, out, s);
  } else {
    if (chunks <= 8) launch_gemv<VEC, 8, 1, 8>(xp, wp, alpha, m, n, k, kw, dots, out, s);
    else launch_gemv<VEC, 32, 1, 8>(xp, wp, alpha, m, n, k, kw, dots, out, s);
  }
}

// ---------------------------------------------------------------------------
// tiled kernel
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async_16(void* smem, const void* gmem, bool valid) {
  const unsigned saddr = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  const int bytes = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(saddr), "l"(gmem), "r"(bytes));
}
__device__ __forceinline__ void cp_async_8(void* smem, const void* gmem, bool valid) {
  const unsigned saddr = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  const int bytes = valid ? 8 : 0;
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;\n" ::"r"(saddr), "l"(gmem), "r"(bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

constexpr int kBK = 8;            // words per stage per row
constexpr int kPitch = kBK + 2;   // 80-byte rows: an odd multiple of 16 bytes
constexpr int kStages = 4;

template <int TM, int TN, int VEC>
__global__ void __launch_bounds__(256)
binary_gemm_tiled_kernel(const uint64_t* __restrict__ xp, const uint64_t* __restrict__ wp,
                         const float* __restrict__ alpha, int64_t m, int64_t n, int k, int kw,
                         int32_t* __restrict__ dots, float* __restrict__ out) {
  constexpr int BM = 16 * TM;
  constexpr int BN = 16 * TN;
  constexpr int CH = kBK / VEC;                     // copy chunks per row per stage
  extern __shared__ __align__(16) uint64_t smem[];
  uint64_t* As = smem;                              // [kStages][BM][kPitch]
  uint64_t* Bs = smem + kStages * BM * kPitch;      // [kStages][BN][kPitch]

  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * BM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * BN;
  const int ktiles = (kw + kBK - 1) / kBK;

  auto load_stage = [&](int stage, int kt) {
    const int kbase = kt * kBK;
    for (int c = tid; c < BM * CH; c += 256) {
      const int row = c / CH, col = (c % CH) * VEC;
      const int64_t gm = m0 + row;
      const bool valid = gm < m && kbase + col < kw;
      const uint64_t* src = valid ? xp + gm * kw + kbase + col : xp;
      uint64_t* dst = As + (stage * BM + row) * kPitch + col;
      if constexpr (VEC == 2) cp_async_16(dst, src, valid); else cp_async_8(dst, src, valid);
    }
    for (int c = tid; c < BN * CH; c += 256) {
      const int row = c / CH, col = (c % CH) * VEC;
      const int64_t gn = n0 + row;
      const bool valid = gn < n && kbase + col < kw;
      const uint64_t* src = valid ? wp + gn * kw + kbase + col : wp;
      uint64_t* dst = Bs + (stage * BN + row) * kPitch + col;
      if constexpr (VEC == 2) cp_async_16(dst, src, valid); else cp_async_8(dst, src, valid);
    }
  };

  uint32_t acc[TM][TN];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0;

#pragma unroll
  for (int st = 0; st < kStages - 1; ++st) {
    if (st < ktiles) load_stage(st, st);
    cp_async_commit();
  }

  for (int kt = 0; kt < ktiles; ++kt) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    const int stage = kt % kStages;
    const uint64_t* A = As + stage * BM * kPitch;
    const uint64_t* B = Bs + stage * BN * kPitch;
#pragma unroll
    for (int kk = 0; kk < kBK; kk += 2) {
      ulonglong2 a[TM];
#pragma unroll
      for (int i = 0; i < TM; ++i) a[i] = *reinterpret_cast<const ulonglong2*>(A + (ty + 16 * i) * kPitch + kk);
#pragma unroll
      for (int j = 0; j < TN; ++j) {
        const ulonglong2 b = *reinterpret_cast<const ulonglong2*>(B + (tx + 16 * j) * kPitch + kk);
#pragma unroll
        for (int i = 0; i < TM; ++i) acc[i][j] += __popcll(a[i].x ^ b.x) + __popcll(a[i].y ^ b.y);
      }
    }
    // Refill the stage consumed one iteration ago (all threads passed the barrier above).
    const int next = kt + kStages - 1;
    if (next < ktiles) load_stage(next % kStages, next);
    cp_async_commit();
  }
  cp_async_wait<0>();

#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int64_t gm = m0 + ty + 16 * i;
    if (gm >= m) continue;
#pragma unroll
    for (int j = 0; j < TN; ++j) {
      const int64_t gn = n0 + tx + 16 * j;
      if (gn >= n) continue;
      const int32_t d = k - 2 * static_cast<int32_t>(acc[i][j]);
      if (dots) dots[gm * n + gn] = d;
      if (out) out[gm * n + gn] = __ldg(alpha + gn) * static_cast<float>(d);
    }
  }
}

template <int TM, int TN, int VEC>
bnn_status launch_tiled(const uint64_t* xp, const uint64_t* wp, const float* alpha, int64_t m, int64_t n,
                        int k, int kw, int32_t* dots, float* out, cudaStream_t s) {
  constexpr int BM = 16 * TM, BN = 16 * TN;
  const int64_t gx = (n + BN - 1) / BN, gy = (m + BM - 1) / BM;
  if (gx > 2147483647LL || gy > 65535) return BNN_ERR_INVALID_ARG;
  const size_t smem = static_cast<size_t>(kStages) * (BM + BN) * kPitch * sizeof(uint64_t);
  auto kern = binary_gemm_tiled_kernel<TM, TN, VEC>;
  BNN_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
  kern<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), 256, smem, s>>>(xp, wp, alpha, m, n, k, kw, dots, out);
  return bnn::check_launch();
}

}  // namespace

extern "C" bnn_status bnn_binary_gemm(const uint64_t* xp, const uint64_t* wp, const float* alpha,
                                      int64_t m, int64_t n, int64_t k, int32_t* dots, float* out,
                                      cudaStream_t s) {
  if (m < 0 || n < 0 || k < 0 || k > BNN_MAX_K_BINARY) return BNN_ERR_INVALID_ARG;
  if (!dots && !out) return BNN_ERR_INVALID_ARG;
  if (out && !alpha) return BNN_ERR_INVALID_ARG;
  if (m == 0 || n == 0) return BNN_OK;
  if (k > 0 && (!xp || !wp)) return BNN_ERR_INVALID_ARG;
  if ((xp && !bnn::aligned(xp, 8)) || (wp && !bnn::aligned(wp, 8)) || (alpha && !bnn::aligned(alpha, 4)) ||
      (dots && !bnn::aligned(dots, 4)) || (out && !bnn::aligned(out, 4)))
    return BNN_ERR_MISALIGNED;
  const int kw = static_cast<int>(bnn::words64(k));
  // 16-byte operand loads need every row 16-byte aligned: even kw and aligned bases.
  const bool vec2 = (kw % 2 == 0) && bnn::aligned(xp, 16) && bnn::aligned(wp, 16);
  const int ki = static_cast<int>(k);

  if (m <= 8) {
    if (vec2) dispatch_gemv<2>(xp, wp, alpha, static_cast<int>(m), n, ki, kw, dots, out, s);
    else dispatch_gemv<1>(xp, wp, alpha, static_cast<int>(m), n, ki, kw, dots, out, s);
    return bnn::check_launch();
  }
  // Large tiles when they still give at least two waves of CTAs, otherwise 64 x 64.
  const int64_t big_tiles = ((m + 127) / 128) * ((n + 127) / 128);
  const bool big = big_tiles >= 2LL * bnn::sm_count();
  if (big) {
    return vec2 ? launch_tiled<8, 8, 2>(xp, wp, alpha, m, n, ki, kw, dots, out, s)
                : launch_tiled<8, 8, 1>(xp, wp, alpha, m, n, ki, kw, dots, out, s);
  }
  return vec2 ? launch_tiled<4, 4, 2>(xp, wp, alpha, m, n, ki, kw, dots, out, s)
              : launch_tiled<4, 4, 1>(xp, wp, alpha, m, n, ki, kw, dots, out, s);
}
