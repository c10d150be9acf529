// bnn_binary_gemm: packed XOR + popcount matmul with a per-output-channel scale.
//
// "Binary Math Effectiveness -- why / how / when", section 1: for +-1 vectors
// packed with bit 1 = -1, <x,w> = n - 2 * popcount(x XOR w) over the logical n
// (pad bits are 0 in both operands, so they never count); "Edge cases": n = 0
// gives 0, alpha = 0 gives 0.  "Architecture Decision Record", "Decision":
// binary_gemm_u64 over uint64 words.
//
// Three kernels:
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
//  * int8 tensor-core (m > 8, the default there): the same packed words are
//    staged through shared memory, and each thread expands the bits it needs
//    straight into the registers of an m16n8k32 s8 MMA fragment as 0/-1 bytes
//    (one shift and one sign-replicating byte permute per 4 values); the MMA
//    sums popc(a AND b) exactly in int32 on the tensor cores and the epilogue
//    forms <x,w> = k - 2 popc(a) - 2 popc(b) + 4 popc(a AND b).
//    On B200 the s8 mma.sync path issues 3.7x the popcount rate of the
//    integer pipe, while the b1 XOR-popcount MMA issues below it.  Because the
//    dot product is a sum over k, any fixed bijection between the 32 bits of a
//    word and the 32 k-slots of the MMA gives the same result as long as both
//    operands use it; the one used here lets each thread build its fragment
//    bytes from byte-aligned sign bits.  Pad bits and zero-filled tail words
//    are 0 in both operands and add nothing to any count.
#include "bnn_internal.cuh"

namespace {

// ---------------------------------------------------------------------------
// skinny kernel
// ---------------------------------------------------------------------------
template <int VEC, int LPR, int R, int MT, int P>
__global__ void __launch_bounds__(256, MT == 1 ? 8 : 4)
binary_gemv_kernel(const uint64_t* __restrict__ xp, const uint64_t* __restrict__ wp,
                   const float* __restrict__ alpha, int m, int64_t n, int k, int kw,
                   int32_t* __restrict__ dots, float* __restrict__ out) {
  static_assert(VEC == 1 || VEC == 2, "VEC");
  constexpr int GROUPS_PER_WARP = 32 / LPR;
  constexpr int SPAN = LPR * VEC;             // words a row group covers in one pass
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPR;                 // lane within its row group
  const int grp = lane / LPR;                 // row group within the warp
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t rows_per_warp_iter = static_cast<int64_t>(GROUPS_PER_WARP) * R;
  bnn::pdl_trigger();
  bool waited = false;  // launched with launch_pdl: the first weight loads overlap the preceding kernel

  for (int64_t row0 = warp * rows_per_warp_iter; row0 < n; row0 += nwarps * rows_per_warp_iter) {
    uint32_t acc[R][MT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int t = 0; t < MT; ++t) acc[r][t] = 0;

    for (int wb = sub * VEC; wb < kw; wb += SPAN * P) {
      // all R x P loads of this step are issued before any is used
      uint64_t wv[R][P][VEC];
#pragma unroll
      for (int p = 0; p < P; ++p) {
        const int w = wb + p * SPAN;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int64_t row = row0 + static_cast<int64_t>(r) * GROUPS_PER_WARP + grp;
          if (row < n && w < kw) {
            const uint64_t* ptr = wp + row * kw + w;
            if constexpr (VEC == 2) {
              const ulonglong2 v = __ldcs(reinterpret_cast<const ulonglong2*>(ptr));
              wv[r][p][0] = v.x;
              wv[r][p][VEC - 1] = v.y;
            } else {
              wv[r][p][0] = __ldcs(ptr);
            }
          } else {
#pragma unroll
            for (int v = 0; v < VEC; ++v) wv[r][p][v] = 0;
          }
        }
      }
      if (!waited) {
        bnn::pdl_wait();  // x may come from the preceding kernel
        waited = true;
      }
#pragma unroll
      for (int p = 0; p < P; ++p) {
        const int w = wb + p * SPAN;
        if (w >= kw) continue;
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
              for (int v = 0; v < VEC; ++v) acc[r][t] += __popcll(wv[r][p][v] ^ xv[v]);
          }
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
    if (!waited) {
      bnn::pdl_wait();  // the outputs are written after the preceding kernel
      waited = true;
    }
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

template <int VEC, int LPR, int R, int MT, int P = 1>
void launch_gemv(const uint64_t* xp, const uint64_t* wp, const float* alpha, int m, int64_t n, int k,
                 int kw, int32_t* dots, float* out, cudaStream_t s) {
  constexpr int threads = 256;
  constexpr int64_t rows_per_block = (threads / 32) * (32 / LPR) * R;
  const int64_t blocks_needed = (n + rows_per_block - 1) / rows_per_block;
  // One block per row block (waves of 8 per SM): blocks that finish early
  // take the next ones, so the stream ends evenly.  A grid capped at one wave
  // (grid-stride) left half the warps a second pass at 1 x 28672 x 8192: 6.45
  // against 5.91 us.  The cap only bounds the grid for very large n.
  const int64_t cap = static_cast<int64_t>(bnn::sm_count()) * 64;
  const int grid = static_cast<int>(blocks_needed < cap ? blocks_needed : cap);
  bnn::launch_pdl(binary_gemv_kernel<VEC, LPR, R, MT, P>, dim3(grid), dim3(threads), 0, s, 1, xp, wp, alpha, m, n,
                  k, kw, dots, out);
}

template <int VEC>
void dispatch_gemv(const uint64_t* xp, const uint64_t* wp, const float* alpha, int m, int64_t n, int k,
                   int kw, int32_t* dots, float* out, cudaStream_t s) {
  // Lanes per row: enough to cover a row in one pass where possible, at least 8.
  const int chunks = (kw + VEC - 1) / VEC;
  if (m <= 1) {
    if (chunks <= 8) launch_gemv<VEC, 8, 2, 1>(xp, wp, alpha, m, n, k, kw, dots, out, s);
    else if (chunks <= 16) launch_gemv<VEC, 16, 2, 1>(xp, wp, alpha, m, n, k, kw, dots, out, s);
    else launch_gemv<VEC, 32, 2, 1, 2>(xp, wp, alpha, m, n, k, kw, dots, out, s);  // 4 loads in flight per lane
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
  BNN_TRY(bnn::ensure_smem(kern, smem));
  kern<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), 256, smem, s>>>(xp, wp, alpha, m, n, k, kw, dots, out);
  return bnn::check_launch();
}


// ---------------------------------------------------------------------------
// int8 tensor-core kernel
// ---------------------------------------------------------------------------
constexpr int kMBKW = 8;               // uint64 words per stage per row (512 bits = 16 k32 steps)
constexpr int kMPitch = 10;            // 80-byte rows: 8 consecutive rows hit distinct 16-byte slots
constexpr int kMStages = 4;

// Bytes j of the result are -1 (0xFF) where bit 8j+7-s of w is set, else 0;
// mul = 2^s.  The shift is a multiply so that it issues on the FMA pipe and
// leaves the integer pipe to the byte permute; the multipliers come from a
// constant table so that the compiler does not turn them back into shifts.
__constant__ uint32_t kShiftMul[8] = {1u, 2u, 4u, 8u, 16u, 32u, 64u, 128u};
__device__ __forceinline__ uint32_t expand_neg(uint32_t w, uint32_t mul) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %1, 0xBA98;\n" : "=r"(r) : "r"(w * mul));
  return r;
}

__device__ __forceinline__ void mma_s8_16832(int* c, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// CTA = WARPS_M x WARPS_N warps; each warp owns WM m16 tiles x WN n8 tiles.
//
// With sign bits a (activation) and b (weight), x = 1 - 2a and w = 1 - 2b, so
//   <x, w> = k - 2 popc(a) - 2 popc(b) + 4 popc(a AND b).
// The MMA operands are the bytes -a and -b (0 or -1: one shift and one
// sign-replicating byte permute per 4 values), whose products sum to
// popc(a AND b) exactly; the row popcounts are taken from the same staged
// tiles, every thread of the CTA owning one row (or a fixed share of one) so
// the side work is spread evenly.  Zero bits (pad bits, zero-filled tail
// words and rows) add nothing to any count.
// KSPLIT groups of WARPS_M x WARPS_N warps split the words of every stage
// between them (more warps per SM for the same tile); their partial counts
// are added through shared memory before the epilogue.
template <int WM, int WN, int WARPS_M, int WARPS_N, int KSPLIT, int VEC, int MINB>
__global__ void __launch_bounds__(WARPS_M * WARPS_N * KSPLIT * 32, MINB)
binary_gemm_mma_kernel(const uint64_t* __restrict__ xp, const uint64_t* __restrict__ wp,
                       const float* __restrict__ alpha, int64_t m, int64_t n, int k, int kw,
                       int32_t* __restrict__ dots, float* __restrict__ out) {
  constexpr int THREADS = WARPS_M * WARPS_N * KSPLIT * 32;
  constexpr int GROUP = WARPS_M * WARPS_N * 32;         // threads per K group
  constexpr int BM = 16 * WM * WARPS_M;
  constexpr int BN = 8 * WN * WARPS_N;
  constexpr int CH = kMBKW / VEC;                       // copy chunks per row per stage
  static_assert(kMBKW % KSPLIT == 0, "KSPLIT must divide the words per stage");
  extern __shared__ __align__(16) uint64_t smem[];
  uint64_t* As = smem;                                  // [kMStages][BM][kMPitch]
  uint64_t* Bs = smem + kMStages * BM * kMPitch;        // [kMStages][BN][kMPitch]

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = (tid % GROUP) >> 5;
  const int kg = tid / GROUP;                           // K group of this thread
  const int gid = lane >> 2, tq = lane & 3;
  const int wm = warp % WARPS_M, wn = warp / WARPS_M;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * BM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * BN;
  const int ktiles = (kw + kMBKW - 1) / kMBKW;
  const uint32_t s0 = kShiftMul[2 * tq], s1 = kShiftMul[2 * tq + 1];
  // side popcounts: thread -> (row of the A/B tile stack, share of its words)
  constexpr int PROWS = BM + BN;
  static_assert(THREADS % PROWS == 0, "threads must cover the tile rows evenly");
  constexpr int TPR = THREADS / PROWS;          // threads per row
  static_assert(kMBKW % TPR == 0, "row words must split evenly");
  constexpr int WPT = kMBKW / TPR;              // words per thread per stage
  const int prow = tid % PROWS;
  const int pw0 = (tid / PROWS) * WPT;
  int pcount = 0;

  auto load_stage = [&](int stage, int kt) {
    const int kbase = kt * kMBKW;
    for (int c = tid; c < BM * CH; c += THREADS) {
      const int row = c / CH, col = (c % CH) * VEC;
      const int64_t gm = m0 + row;
      const bool valid = gm < m && kbase + col < kw;
      const uint64_t* src = valid ? xp + gm * kw + kbase + col : xp;
      uint64_t* dst = As + (stage * BM + row) * kMPitch + col;
      if constexpr (VEC == 2) cp_async_16(dst, src, valid); else cp_async_8(dst, src, valid);
    }
    for (int c = tid; c < BN * CH; c += THREADS) {
      const int row = c / CH, col = (c % CH) * VEC;
      const int64_t gn = n0 + row;
      const bool valid = gn < n && kbase + col < kw;
      const uint64_t* src = valid ? wp + gn * kw + kbase + col : wp;
      uint64_t* dst = Bs + (stage * BN + row) * kMPitch + col;
      if constexpr (VEC == 2) cp_async_16(dst, src, valid); else cp_async_8(dst, src, valid);
    }
  };

  int acc[WM][WN][4];
#pragma unroll
  for (int i = 0; i < WM; ++i)
#pragma unroll
    for (int j = 0; j < WN; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[i][j][c] = 0;

#pragma unroll
  for (int st = 0; st < kMStages - 1; ++st) {
    if (st < ktiles) load_stage(st, st);
    cp_async_commit();
  }

  for (int kt = 0; kt < ktiles; ++kt) {
    cp_async_wait<kMStages - 2>();
    __syncthreads();
    const int stage = kt % kMStages;
    {
      const uint64_t* prow_ptr = prow < BM ? As + (stage * BM + prow) * kMPitch
                                           : Bs + (stage * BN + (prow - BM)) * kMPitch;
#pragma unroll
      for (int q = 0; q < WPT; ++q) pcount += __popcll(prow_ptr[pw0 + q]);
    }
    const uint64_t* A = As + (stage * BM + wm * 16 * WM + gid) * kMPitch;
    const uint64_t* B = Bs + (stage * BN + wn * 8 * WN + gid) * kMPitch;
#pragma unroll
    for (int kq = 0; kq < kMBKW / KSPLIT; ++kq) {
      const int kk = kq * KSPLIT + kg;
      // one uint64 word = two k32 MMA steps
      uint2 aw[WM][2], bw[WN];
#pragma unroll
      for (int i = 0; i < WM; ++i) {
        aw[i][0] = *reinterpret_cast<const uint2*>(A + (16 * i) * kMPitch + kk);
        aw[i][1] = *reinterpret_cast<const uint2*>(A + (16 * i + 8) * kMPitch + kk);
      }
#pragma unroll
      for (int j = 0; j < WN; ++j) bw[j] = *reinterpret_cast<const uint2*>(B + (8 * j) * kMPitch + kk);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t bf[WN][2];
#pragma unroll
        for (int j = 0; j < WN; ++j) {
          const uint32_t w = h ? bw[j].y : bw[j].x;
          bf[j][0] = expand_neg(w, s0);
          bf[j][1] = expand_neg(w, s1);
        }
#pragma unroll
        for (int i = 0; i < WM; ++i) {
          const uint32_t w0 = h ? aw[i][0].y : aw[i][0].x;
          const uint32_t w1 = h ? aw[i][1].y : aw[i][1].x;
          const uint32_t af[4] = {expand_neg(w0, s0), expand_neg(w1, s0), expand_neg(w0, s1),
                                  expand_neg(w1, s1)};
#pragma unroll
          for (int j = 0; j < WN; ++j) mma_s8_16832(acc[i][j], af, bf[j]);
        }
      }
    }
    const int next = kt + kMStages - 1;
    if (next < ktiles) load_stage(next % kMStages, next);
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();  // every warp is done with the operand tiles: reuse the space

  if constexpr (KSPLIT > 1) {
    // groups 1.. hand their partial AND-counts to group 0 (fixed order: exact integers anyway)
    int* xs = reinterpret_cast<int*>(smem);  // [KSPLIT-1][WM*WN*4][GROUP]: lanes hit consecutive banks
    constexpr int PER = WM * WN * 4;
    if (kg > 0) {
      int* dst = xs + (kg - 1) * PER * GROUP + (tid % GROUP);
#pragma unroll
      for (int i = 0; i < WM; ++i)
#pragma unroll
        for (int j = 0; j < WN; ++j)
#pragma unroll
          for (int c = 0; c < 4; ++c) dst[((i * WN + j) * 4 + c) * GROUP] = acc[i][j][c];
    }
    __syncthreads();
    if (kg == 0) {
      for (int g = 1; g < KSPLIT; ++g) {
        const int* src = xs + (g - 1) * PER * GROUP + tid;
#pragma unroll
        for (int i = 0; i < WM; ++i)
#pragma unroll
          for (int j = 0; j < WN; ++j)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[i][j][c] += src[((i * WN + j) * 4 + c) * GROUP];
      }
    }
    __syncthreads();
  }

  int* pa_s = reinterpret_cast<int*>(smem);  // [BM]
  int* pb_s = pa_s + BM;                      // [BN]
  for (int i = tid; i < PROWS; i += THREADS) pa_s[i] = 0;
  __syncthreads();
  atomicAdd(&pa_s[prow], pcount);  // integer adds: the order does not matter
  __syncthreads();
  if (kg != 0) return;

#pragma unroll
  for (int i = 0; i < WM; ++i) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int lr = wm * 16 * WM + 16 * i + gid + 8 * hr;
      const int64_t gm = m0 + lr;
      if (gm >= m) continue;
      const int base = k - 2 * pa_s[lr];
#pragma unroll
      for (int j = 0; j < WN; ++j) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int lc = wn * 8 * WN + 8 * j + 2 * tq + c;
          const int64_t gn = n0 + lc;
          if (gn >= n) continue;
          const int32_t d = base - 2 * pb_s[lc] + 4 * acc[i][j][2 * hr + c];
          if (dots) dots[gm * n + gn] = d;
          if (out) out[gm * n + gn] = __ldg(alpha + gn) * static_cast<float>(d);
        }
      }
    }
  }
}

template <int WM, int WN, int WARPS_M, int WARPS_N, int KSPLIT, int VEC, int MINB>
bnn_status launch_mma(const uint64_t* xp, const uint64_t* wp, const float* alpha, int64_t m, int64_t n,
                      int k, int kw, int32_t* dots, float* out, cudaStream_t s) {
  constexpr int BM = 16 * WM * WARPS_M, BN = 8 * WN * WARPS_N;
  const int64_t gx = (n + BN - 1) / BN, gy = (m + BM - 1) / BM;
  if (gx > 2147483647LL || gy > 65535) return BNN_ERR_INVALID_ARG;
  constexpr int THREADS = WARPS_M * WARPS_N * KSPLIT * 32;
  const size_t tiles = static_cast<size_t>(kMStages) * (BM + BN) * kMPitch * sizeof(uint64_t);
  const size_t xchg = static_cast<size_t>(KSPLIT - 1) * WARPS_M * WARPS_N * 32 * WM * WN * 4 * sizeof(int);
  const size_t smem = tiles > xchg ? tiles : xchg;
  auto kern = binary_gemm_mma_kernel<WM, WN, WARPS_M, WARPS_N, KSPLIT, VEC, MINB>;
  BNN_TRY(bnn::ensure_smem(kern, smem));
  kern<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), THREADS, smem, s>>>(
      xp, wp, alpha, m, n, k, kw, dots, out);
  return bnn::check_launch();
}

template <int VEC>
bnn_status dispatch_mma(const uint64_t* xp, const uint64_t* wp, const float* alpha, int64_t m, int64_t n,
                        int k, int kw, int32_t* dots, float* out, cudaStream_t s) {
  const int64_t big_tiles = ((m + 127) / 128) * ((n + 127) / 128);
  if (big_tiles >= 2LL * bnn::sm_count())
    return launch_mma<4, 4, 2, 4, 1, VEC, 1>(xp, wp, alpha, m, n, k, kw, dots, out, s);  // 128 x 128, 8 warps
  return launch_mma<2, 4, 2, 2, 2, VEC, 2>(xp, wp, alpha, m, n, k, kw, dots, out, s);    // 64 x 64, 2 x 4 warps
}

}  // namespace

extern "C" bnn_status bnn_binary_gemm_algo(const uint64_t* xp, const uint64_t* wp, const float* alpha,
                                           int64_t m, int64_t n, int64_t k, int32_t* dots, float* out,
                                           bnn_binary_algo algo, cudaStream_t s) {
  if (m < 0 || n < 0 || k < 0 || k > BNN_MAX_K_BINARY) return BNN_ERR_INVALID_ARG;
  if (algo != BNN_ALGO_AUTO && algo != BNN_ALGO_POPC && algo != BNN_ALGO_MMA_S8 && algo != BNN_ALGO_TC)
    return BNN_ERR_INVALID_ARG;
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

  // AUTO: tcgen05 from 64 activation rows up (measured faster than mma.sync from
  // the 64 x 4096 x 4096 layer to 8192^3), mma.sync for 9..63 rows, GEMV below.
  if (algo == BNN_ALGO_TC || (algo == BNN_ALGO_AUTO && m >= 64))
    return bnn::binary_gemm_tc(xp, wp, alpha, nullptr, m, n, ki, kw, dots, out, nullptr, s);
  if (algo == BNN_ALGO_MMA_S8 || (algo == BNN_ALGO_AUTO && m > 8)) {
    return vec2 ? dispatch_mma<2>(xp, wp, alpha, m, n, ki, kw, dots, out, s)
                : dispatch_mma<1>(xp, wp, alpha, m, n, ki, kw, dots, out, s);
  }
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

extern "C" bnn_status bnn_binary_linear(const uint64_t* xp, const uint64_t* wp, const float* alpha,
                                        const float* bias, int64_t m, int64_t n, int64_t k, int32_t* dots,
                                        float* out, uint64_t* next, cudaStream_t s) {
  if (m < 0 || n < 0 || k < 0 || k > BNN_MAX_K_BINARY) return BNN_ERR_INVALID_ARG;
  if (!dots && !out && !next) return BNN_ERR_INVALID_ARG;
  if ((out || next) && !alpha) return BNN_ERR_INVALID_ARG;
  if (m == 0 || n == 0) return BNN_OK;
  if (k > 0 && (!xp || !wp)) return BNN_ERR_INVALID_ARG;
  if ((xp && !bnn::aligned(xp, 8)) || (wp && !bnn::aligned(wp, 8)) || (alpha && !bnn::aligned(alpha, 4)) ||
      (bias && !bnn::aligned(bias, 4)) || (dots && !bnn::aligned(dots, 4)) || (out && !bnn::aligned(out, 4)) ||
      (next && !bnn::aligned(next, 8)))
    return BNN_ERR_MISALIGNED;
  return bnn::binary_gemm_tc(xp, wp, alpha, bias, m, n, static_cast<int>(k), static_cast<int>(bnn::words64(k)),
                             dots, out, next, s);
}

extern "C" bnn_status bnn_binary_gemm(const uint64_t* xp, const uint64_t* wp, const float* alpha,
                                      int64_t m, int64_t n, int64_t k, int32_t* dots, float* out,
                                      cudaStream_t s) {
  return bnn_binary_gemm_algo(xp, wp, alpha, m, n, k, dots, out, BNN_ALGO_AUTO, s);
}
