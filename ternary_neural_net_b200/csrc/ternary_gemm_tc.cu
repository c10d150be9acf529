// bnn_ternary_gemm on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// Three kernels: ternary_gemm_tmem_kernel (at most 64 activation rows, k a
// multiple of 8: the decoded trits are stored to tensor memory),
// ternary_gemm_tc2_kernel (more rows, k a multiple of 8: warp-specialised,
// decoded trits in shared memory) and ternary_gemm_tc_kernel (any shape,
// described first below).
//
// "BalancedTernaryEngine" README, "Module Overview" (Layer.forward) with the
// "Features" encoding: y[i,j] = scale_j * sum_e x[i,e] t[j,e], trits packed 10
// per 16-bit word in base 3.
//
// UMMA M = 128 weight rows, N = 64 activation rows, K in stages of 64 trits:
// D[128 x 64] (fp32) = T (bf16 trits) x X^T, accumulated in tensor memory.  A
// cluster of kTcK CTAs splits the packed words of one 128-row tile; their
// partial tiles are added in rank order through distributed shared memory.
// Per stage every thread decodes four (row, word) jobs: the words of a row that
// overlap the stage's 64 trits are split into base-9 digits (__umulhi on a
// fixed-point fraction, as in the other ternary kernels), each digit a
// 9-entry table lookup giving the bf16 pair (t_2q, t_2q+1), written as one
// 32-bit word into the 128-byte-swizzled K-major tile the tensor core reads;
// pairs never straddle a 64-trit boundary, and positions past the last word
// are written as zeros.  The activations are copied with 16-byte cp.async
// into the same layout two stages ahead.  One thread issues 4
// tcgen05.mma.kind::f16 (K = 16) per stage and commits to the stage's
// mbarrier; a buffer is refilled only after that commit has completed.  The
// output rows of a warp are consecutive weight rows, so the stores of the
// epilogue are coalesced along j.  Every mbarrier wait is bounded (see
// bnn_device_error_count).
#include <cooperative_groups.h>

#include <mutex>

#include "bnn_internal.cuh"
#include "tc_common.cuh"

// Bounded waits that ran out in this file's kernels (read by bnn_device_error_count).
__device__ unsigned int g_bnn_tc_ternary_errors = 0;

namespace {

constexpr int kTcStagesT = 4;
constexpr int kTcMW = 128;     // weight rows per CTA (UMMA M)
constexpr int kTcNX = 64;      // activation rows per CTA (UMMA N)
constexpr int kTcK = 2;        // CTAs per cluster (split of the trits)
constexpr int kTcThreads = 256;
constexpr int kPreT = 4;       // stages of weight words prefetched in registers
constexpr uint32_t kFix = 72736u;  // ceil(2^32 / 3^10)
constexpr int kAStage = kTcMW * 128;  // bytes per stage of the weight tile
constexpr int kBStage = kTcNX * 128;  // bytes per stage of the activation tile

__device__ __forceinline__ uint32_t s_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// bounded wait (polls for at most bnn::tc::kWaitNs of wall time)
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = bnn::tc::global_ns();
  for (uint32_t it = 1;; ++it) {
    if (bnn::tc::mbar_try(bar, parity)) return true;
    if ((it & 63u) == 0 && bnn::tc::global_ns() - t0 > bnn::tc::kWaitNs) return false;
  }
}

// byte offset of element (row, k) (k < 64, 2-byte elements) in a 128B-swizzled K-major tile
__device__ __forceinline__ uint32_t sw_off(int row, int k) {
  const uint32_t chunk = static_cast<uint32_t>(k >> 3);
  return static_cast<uint32_t>(row) * 128u + ((chunk ^ static_cast<uint32_t>(row & 7)) << 4) +
         static_cast<uint32_t>((k & 7) * 2);
}

template <bool VECX>
__global__ void __cluster_dims__(kTcK, 1, 1) __launch_bounds__(kTcThreads)
ternary_gemm_tc_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ packed,
                       const float* __restrict__ scale, int64_t m, int64_t n, int64_t k, int64_t kt,
                       int64_t slice_stages, float* __restrict__ out, const float* __restrict__ bias) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) uint8_t tsm_raw[];
  __shared__ __align__(8) uint64_t bars[kTcStagesT];
  __shared__ uint32_t tmem_holder;
  __shared__ uint32_t lut[9];
  uint8_t* const tsm = tsm_raw + ((1024u - (s_u32(tsm_raw) & 1023u)) & 1023u);
  uint8_t* const As = tsm;                                // [stages][128 rows x 128 B]
  uint8_t* const Bs = tsm + kTcStagesT * kAStage;         // [stages][64 rows x 128 B]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = static_cast<int>(cluster.block_rank());
  const int64_t n0 = static_cast<int64_t>(blockIdx.x / kTcK) * kTcMW;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kTcNX;
  const int64_t total_stages = (10 * kt + 63) / 64;       // 64-trit stages covering every packed trit
  const int64_t s_begin = rank * slice_stages;
  const int64_t s_end = s_begin + slice_stages < total_stages ? s_begin + slice_stages : total_stages;
  const int nst = s_end > s_begin ? static_cast<int>(s_end - s_begin) : 0;

  if (tid < 9) {
    const int lo = tid % 3, hi = tid / 3;  // digit = trit + 1
    const uint32_t blo = lo == 0 ? 0xBF80u : (lo == 2 ? 0x3F80u : 0u);
    const uint32_t bhi = hi == 0 ? 0xBF80u : (hi == 2 ? 0x3F80u : 0u);
    lut[tid] = blo | (bhi << 16);
  }
  if (tid == 0) {
    for (int i = 0; i < kTcStagesT; ++i) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(s_u32(&bars[i])));
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(s_u32(&tmem_holder)),
                 "r"(kTcNX));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const uint32_t tmem = tmem_holder;
  // D f32, A and B bf16, both K-major, N = 64, M = 128
  const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(kTcNX) >> 3) << 17) |
                         ((static_cast<uint32_t>(kTcMW) >> 4) << 24);

  // activations of stage s (global stage index) into buffer b: 64 rows x 8 chunks of 16 bytes
  auto load_x = [&](int64_t s, int b) {
    const int64_t kb = 64 * s;
    for (int c = tid; c < kTcNX * 8; c += kTcThreads) {
      const int row = c >> 3, ch = c & 7;
      const int64_t gm = m0 + row, gk = kb + 8 * ch;
      uint8_t* dst = Bs + b * kBStage + row * 128 + ((static_cast<uint32_t>(ch) ^ static_cast<uint32_t>(row & 7)) << 4);
      if constexpr (VECX) {
        int bytes = 0;
        if (gm < m && gk < k) bytes = static_cast<int>((k - gk < 8 ? k - gk : 8) * 2);
        const uint16_t* src = bytes ? x + gm * k + gk : x;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s_u32(dst)), "l"(src), "r"(bytes)
                     : "memory");
      } else {
        uint16_t v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = (gm < m && gk + e < k) ? __ldg(x + gm * k + gk + e) : uint16_t(0);
        uint4 q;
        q.x = v[0] | (static_cast<uint32_t>(v[1]) << 16);
        q.y = v[2] | (static_cast<uint32_t>(v[3]) << 16);
        q.z = v[4] | (static_cast<uint32_t>(v[5]) << 16);
        q.w = v[6] | (static_cast<uint32_t>(v[7]) << 16);
        *reinterpret_cast<uint4*>(dst) = q;
      }
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
  };

  // Every thread owns 4 (row, word-slot) jobs per stage: row = tid % 128,
  // slots tid / 128 + {0, 2, 4, 6} of the (up to) 8 words overlapping the stage.
  const int jrow = tid % kTcMW;
  const int jslot0 = tid / kTcMW;
  const int64_t jgn = n0 + jrow;
  const uint16_t* jsrc = packed + (jgn < n ? jgn : 0) * kt;
  // words of stage s for this thread's jobs (0xFFFF marks "no word": written as zeros)
  auto fetch_w = [&](int64_t s, uint32_t* wv) {
    const int64_t j_lo = (64 * s) / 10;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t j = j_lo + jslot0 + 2 * i;
      wv[i] = (jgn < n && j < kt) ? static_cast<uint32_t>(__ldg(jsrc + j)) : 0xFFFFu;
    }
  };
  // trits of stage s into buffer b from the fetched words
  auto decode_w = [&](int64_t s, int b, const uint32_t* wv) {
    const int64_t t0 = 64 * s;
    const int64_t j_lo = t0 / 10, j_hi = (t0 + 63) / 10;
    uint8_t* tile = As + b * kAStage;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t j = j_lo + jslot0 + 2 * i;
      if (j > j_hi) continue;
      const bool real = wv[i] != 0xFFFFu;
      uint32_t F = real ? wv[i] * kFix : 0u;
#pragma unroll
      for (int q = 4; q >= 0; --q) {
        uint32_t v = 4;  // digit pair (1, 1): trits (0, 0)
        if (real) {
          v = __umulhi(F, 9u);
          F *= 9u;
        }
        const int64_t tk = 10 * j + 2 * q - t0;  // position of the pair inside the stage
        if (tk >= 0 && tk < 64) *reinterpret_cast<uint32_t*>(tile + sw_off(jrow, static_cast<int>(tk))) = lut[v];
      }
    }
  };

  __syncthreads();  // lut ready
  // exactly two prologue groups (empty when the slice is shorter), so that in
  // iteration `it` "all but the newest two groups" is stage it's copy
  if (nst > 0) load_x(s_begin, 0); else asm volatile("cp.async.commit_group;\n" ::: "memory");
  if (nst > 1) load_x(s_begin + 1, 1); else asm volatile("cp.async.commit_group;\n" ::: "memory");
  bool ok = true;
  int committed = -1;
  // weight words kPreT stages ahead in a register ring (loop unrolled by kPreT: static ring indices)
  uint32_t ring[kPreT][4];
#pragma unroll
  for (int u = 0; u < kPreT; ++u)
    if (u < nst) fetch_w(s_begin + u, ring[u]);
  for (int it0 = 0; it0 < nst && ok; it0 += kPreT) {
#pragma unroll
    for (int u = 0; u < kPreT; ++u) {
      const int it = it0 + u;
      if (it >= nst || !ok) break;
      const int b = it % kTcStagesT;
      bool free_ok = true;
      if (it + 2 < nst) {
        const int bn = (it + 2) % kTcStagesT;
        if (it - 2 >= 0) free_ok = wait_bar(s_u32(&bars[bn]), static_cast<uint32_t>(((it - 2) / kTcStagesT) & 1));
        load_x(s_begin + it + 2, bn);
      } else {
        asm volatile("cp.async.commit_group;\n" ::: "memory");  // keep one group per iteration
      }
      uint32_t cur[4] = {ring[u][0], ring[u][1], ring[u][2], ring[u][3]};
      if (it + kPreT < nst) fetch_w(s_begin + it + kPreT, ring[u]);
      decode_w(s_begin + it, b, cur);
      asm volatile("cp.async.wait_group 2;\n" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      ok = __syncthreads_and(free_ok) != 0;
      if (!ok) break;
      if (tid == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
        const uint64_t ad = desc_sw128(s_u32(As + b * kAStage));
        const uint64_t bd = desc_sw128(s_u32(Bs + b * kBStage));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
          asm volatile(
              "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
              "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
              "l"(ad + static_cast<uint64_t>(2 * kk)), "l"(bd + static_cast<uint64_t>(2 * kk)), "r"(idesc), "r"(acc));
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                         s_u32(&bars[b]))
                     : "memory");
      }
      committed = it;
    }
  }
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
  bool drained = true;
  if (committed >= 0) {
    const uint32_t bar = s_u32(&bars[committed % kTcStagesT]);
    const uint32_t par = static_cast<uint32_t>((committed / kTcStagesT) & 1);
    drained = wait_bar(bar, par) || wait_bar(bar, par);
  }
  const bool good = __syncthreads_and(ok && drained) != 0;
  if (!good && tid == 0) atomicAdd(&g_bnn_tc_ternary_errors, 1u);
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");

  // partial tile [128 weight rows][64 activation rows] into this CTA's shared memory
  float* part = reinterpret_cast<float*>(tsm);  // the operand tiles are no longer read
  constexpr int PP = kTcNX + 1;                 // padded pitch
  if (warp < 4) {
    for (int c0 = 0; c0 < kTcNX; c0 += 32) {
      uint32_t r[32];
      if (committed >= 0 && good) {
        const uint32_t a = tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(c0);
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
            "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
              "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
              "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
              "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
            : "r"(a));
        asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) r[c] = 0u;
      }
      const int wr = warp * 32 + lane;
#pragma unroll
      for (int c = 0; c < 32; ++c) part[wr * PP + c0 + c] = __uint_as_float(r[c]);
    }
  }
  cluster.sync();
  if (rank == 0) {
    for (int idx = tid; idx < kTcMW * kTcNX; idx += kTcThreads) {
      const int wr = idx % kTcMW, xr = idx / kTcMW;  // consecutive threads: consecutive weight rows
      float sum = part[wr * PP + xr];
#pragma unroll
      for (int q = 1; q < kTcK; ++q) sum += cluster.map_shared_rank(part, q)[wr * PP + xr];
      const int64_t gn = n0 + wr, gm = m0 + xr;
      if (gn < n && gm < m) out[gm * n + gn] = bias ? __ldg(scale + gn) * sum + __ldg(bias + gn) : __ldg(scale + gn) * sum;
    }
  }
  cluster.sync();  // partial tiles stay alive until rank 0 has read them
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTcNX));
}


// ---------------------------------------------------------------------------
// Warp-specialised version (activation rows 16-byte aligned: TMA).
//
// Tile: 128 weight rows x BN activation rows (BN = 64 with two CTAs per SM,
// or 128 / 256 with one, so that each weight tile is decoded once per 128 or
// 256 activation rows instead of per 64), K stages of 64 trits.
// Roles: one thread copies the stage's 64-trit x BN-row bf16 activation box by
// TMA straight into the 128-byte-swizzled tile; 512 producer threads copy the
// stage's 8-word window of each weight row into shared memory (coalesced along
// the rows, one stage ahead) and then decode: warp w takes quarter w % 4 (16
// trits, 8 pairs) of 32 weight rows, reads the (up to) three words covering
// them and writes two 16-byte chunks; one thread issues 4
// tcgen05.mma.kind::f16 (K = 16) per stage; warps 0-7 read the float32
// accumulator.  A pair's word and base-9 digit depend only on the phase (first
// trit mod 10, one of 0, 2, 4, 6, 8), which is the same for every lane of a
// warp, so the decode is specialised per phase without divergence: per pair one
// multiply by a constant power of 9, one __umulhi and one 9-entry table load.
// The producers meet at one named barrier per stage (with an AND of their
// wait results, so that a wait that ran out stops all of them together); the
// rest is synchronised by mbarriers.  A cluster of KS CTAs
// splits the stages; each CTA pushes its partial sums (float4 stores into
// distributed shared memory) to the CTA owning those activation rows, which
// adds them in rank order (deterministic), scales and adds the bias.
// ---------------------------------------------------------------------------
constexpr int kT2M = 128;                            // weight rows (UMMA M)
constexpr int kT2N = 64;                             // activation rows (UMMA N)
constexpr int kT2S = 4;                              // stages of 64 trits
constexpr int kT2Prod = 4 * kT2M;                    // producer threads
constexpr int kT2Threads = kT2Prod + 64;             // + MMA warp + TMA warp
constexpr uint32_t kT2AStage = kT2M * 128u;          // one stage of decoded weights
constexpr int kT2Pre = 4;                            // stages of words prefetched in registers
constexpr uint32_t kZeroWord = 29524u;               // all ten trits 0 (every digit 1)

// floor(v / 10) for any 32-bit v (multiply-high by ceil(2^35 / 10))
__device__ __forceinline__ uint32_t div10(uint32_t v) { return __umulhi(v, 0xCCCCCCCDu) >> 3; }

// 9^p (0 <= p <= 4); not recursive, so that it folds to a constant in unrolled code
__host__ __device__ __forceinline__ constexpr uint32_t pow9(int p) {
  return p <= 0 ? 1u : (p == 1 ? 9u : (p == 2 ? 81u : (p == 3 ? 729u : 6561u)));
}

// the 8 bf16 pairs of 16 trits starting at phase R10 of word 0 (F[i] = word_i * kFix)
template <int R10>
__device__ __forceinline__ void decode16(const uint32_t (&F)[3], const uint32_t* lut, uint4& lo, uint4& hi) {
  uint32_t v[8];
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int kp = R10 / 2 + p;       // pair index counted from word 0
    const int j = kp / 5, q = kp % 5;  // word, base-9 digit (q = 4: trits 8, 9)
    // the digit is the integer part of 9 x (fraction of word / 9^5 scaled by 9^(4-q))
    v[p] = lut[__umulhi(F[j] * pow9(4 - q), 9u)];
  }
  lo = make_uint4(v[0], v[1], v[2], v[3]);
  hi = make_uint4(v[4], v[5], v[6], v[7]);
}

template <int KS, int BN>
__global__ void __launch_bounds__(kT2Threads, BN == 64 ? 2 : 1)
ternary_gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint16_t* __restrict__ packed,
                        const float* __restrict__ scale, const float* __restrict__ bias, int64_t m, int64_t n,
                        int64_t k, int64_t kt, float* __restrict__ out) {
  using namespace bnn::tc;
  constexpr uint32_t kT2Stage = kT2AStage + BN * 128u;  // decoded weights + BN activation rows
  constexpr int kCols = BN / KS;
  constexpr int kPitch = kCols + 4;  // padded receive row (floats)
  static_assert(KS * kT2M * kPitch * 4 <= kT2S * kT2Stage, "split-K shares must fit the stage memory");

  extern __shared__ __align__(16) uint8_t t2_raw[];
  __shared__ __align__(8) uint64_t full_bar[kT2S];
  __shared__ __align__(8) uint64_t empty_bar[kT2S];
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ uint32_t tmem_holder;
  __shared__ volatile int abort_flag;
  __shared__ int any_bad;
  __shared__ uint32_t lut[9];
  __shared__ uint32_t wtile[2][kT2M][9];  // packed words of a stage's window, 9-word pitch (odd: no bank conflicts)
  uint8_t* const smem = t2_raw + ((1024u - (smem_u32(t2_raw) & 1023u)) & 1023u);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int rank = KS > 1 ? static_cast<int>(blockIdx.x % KS) : 0;
  const int64_t j0 = static_cast<int64_t>(blockIdx.x / KS) * kT2M;  // first weight row
  const int64_t i0 = static_cast<int64_t>(blockIdx.y) * BN;        // first activation row
  const int64_t total = (k + 63) / 64;  // 64-trit stages up to trit k (past it, only pad trits of the last word)
  const int64_t share = (total + KS - 1) / KS;
  const int64_t sb = rank * share < total ? rank * share : total;
  const int64_t se = sb + share < total ? sb + share : total;
  const int nst = static_cast<int>(se - sb);
  constexpr int kMmaWarp = kT2Prod / 32, kTmaWarp = kMmaWarp + 1;

  if (tid < 9) {
    const int lo = tid % 3, hi = tid / 3;  // digit = trit + 1
    const uint32_t blo = lo == 0 ? 0xBF80u : (lo == 2 ? 0x3F80u : 0u);
    const uint32_t bhi = hi == 0 ? 0xBF80u : (hi == 2 ? 0x3F80u : 0u);
    lut[tid] = blo | (bhi << 16);
  }
  if (tid == 0) {
    for (int i = 0; i < kT2S; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 2);  // one producer after their barrier + the TMA thread's expect_tx
      mbar_init(smem_u32(&empty_bar[i]), 1);
    }
    mbar_init(smem_u32(&done_bar), 1);
    abort_flag = 0;
    any_bad = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (tid == kTmaWarp * 32)
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(&tmem_holder)),
                 "r"(BN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const uint32_t tmem = tmem_holder;
  bnn::pdl_trigger();

  if (tid < kT2Prod) {
    // ------------------------------------------------------------ producers
    // Copy: producer p stages words 2(p%4), 2(p%4)+1 of the stage's 8-word
    // window of weight row p/4 (coalesced along the row) into wtile, one stage
    // ahead, from registers loaded kT2Pre stages ahead.
    const int crow = tid >> 2, cw = 2 * (tid & 3);
    const int64_t cgn = j0 + crow;
    const bool clive = cgn < n;
    const uint16_t* csrc = packed + (clive ? cgn : 0) * kt;
    const uint32_t kt32 = static_cast<uint32_t>(kt), se32 = static_cast<uint32_t>(se);
    auto fetch = [&](uint32_t s, uint32_t& w0, uint32_t& w1) {
      const uint32_t j = div10(64u * s) + static_cast<uint32_t>(cw);
      w0 = (clive && s < se32 && j < kt32) ? static_cast<uint32_t>(__ldg(csrc + j)) : kZeroWord;
      w1 = (clive && s < se32 && j + 1 < kt32) ? static_cast<uint32_t>(__ldg(csrc + j + 1)) : kZeroWord;
    };
    auto stage_words = [&](int buf, uint32_t w0, uint32_t w1) {
      wtile[buf][crow][cw] = w0;
      wtile[buf][crow][cw + 1] = w1;
    };
    // Decode: warp w takes quarter w % 4 (trits 16q..16q+15 of the stage) of
    // 32 weight rows, so the word phase of a stage is the same for the whole warp.
    const int quarter = warp & 3, row = 32 * (warp >> 2) + (tid & 31);
    const uint32_t row_off = static_cast<uint32_t>(row) * 128u, swz = static_cast<uint32_t>(row & 7);

    const uint32_t sb32 = static_cast<uint32_t>(sb);
    uint32_t ring[kT2Pre][2];
#pragma unroll
    for (int u = 0; u < kT2Pre; ++u) fetch(sb32 + 1 + u, ring[u][0], ring[u][1]);
    {
      uint32_t w0, w1;
      fetch(sb32, w0, w1);
      stage_words(0, w0, w1);
    }
    bool ok = bnn::tc::producer_barrier_and(true, kT2Prod);
    for (int js = 0; js < nst && ok; js += kT2Pre) {
#pragma unroll
      for (int u = 0; u < kT2Pre; ++u) {
        const int jj = js + u;
        if (jj >= nst) break;
        // the next stage's window (ring[u] holds stage sb + jj + 1)
        stage_words((jj + 1) & 1, ring[u][0], ring[u][1]);
        fetch(sb32 + jj + 1 + kT2Pre, ring[u][0], ring[u][1]);
        const int b = jj % kT2S;
        const bool fine = jj < kT2S || mbar_wait(smem_u32(&empty_bar[b]),
                                                 static_cast<uint32_t>((jj / kT2S + 1) & 1), &abort_flag,
                                                 &g_bnn_tc_ternary_errors);
        if (fine) {
          const uint32_t s64 = 64u * (sb32 + jj), t0 = s64 + 16u * quarter;  // trit positions (< 2^31)
          const uint32_t jt = div10(t0);
          const uint32_t jrel = jt - div10(s64);
          const uint32_t* wr = wtile[jj & 1][row];
          const uint32_t F[3] = {wr[jrel] * kFix, wr[jrel + 1] * kFix, wr[jrel + 2] * kFix};
          uint4 lo, hi;
          switch (t0 - 10u * jt) {  // the phase, warp-uniform
            case 0: decode16<0>(F, lut, lo, hi); break;
            case 2: decode16<2>(F, lut, lo, hi); break;
            case 4: decode16<4>(F, lut, lo, hi); break;
            case 6: decode16<6>(F, lut, lo, hi); break;
            default: decode16<8>(F, lut, lo, hi); break;
          }
          uint8_t* dst = smem + b * kT2Stage + row_off;
          *reinterpret_cast<uint4*>(dst + (((2u * quarter) ^ swz) << 4)) = lo;
          *reinterpret_cast<uint4*>(dst + (((2u * quarter + 1u) ^ swz) << 4)) = hi;
          asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        }
        // one decision for all producers: the staged window is complete and the
        // decoded one may be overwritten; a wait that ran out stops them all.
        // After it one thread tells the tensor core that the stage is written.
        ok = bnn::tc::producer_barrier_and(fine, kT2Prod);
        if (!ok) break;
        if (tid == 0) mbar_arrive(smem_u32(&full_bar[b]));
      }
    }
  } else if (tid == kMmaWarp * 32) {
    // ------------------------------------------------------------ MMA issue
    // D f32, A and B bf16, both K-major, N = 64, M = 128
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(BN) >> 3) << 17) |
                           ((static_cast<uint32_t>(kT2M) >> 4) << 24);
    const uint32_t base = smem_u32(smem);
    for (int jj = 0; jj < nst; ++jj) {
      const int b = jj % kT2S;
      if (!mbar_wait(smem_u32(&full_bar[b]), static_cast<uint32_t>((jj / kT2S) & 1), &abort_flag,
                     &g_bnn_tc_ternary_errors))
        break;
      asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
      const uint64_t ad = sw128_desc(base + b * kT2Stage), bd = sw128_desc(base + b * kT2Stage + kT2AStage);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t acc = (jj > 0 || kk > 0) ? 1u : 0u;
        asm volatile(
            "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
            "l"(ad + static_cast<uint64_t>(2 * kk)), "l"(bd + static_cast<uint64_t>(2 * kk)), "r"(idesc), "r"(acc));
      }
      mma_commit(smem_u32(&empty_bar[b]));
    }
    mma_commit(smem_u32(&done_bar));
  } else if (tid == kTmaWarp * 32) {
    // ------------------------------------------------------------ TMA copies of the activations
    bnn::pdl_wait();  // x may come from the preceding kernel
    for (int jj = 0; jj < nst; ++jj) {
      const int b = jj % kT2S;
      if (jj >= kT2S && !mbar_wait(smem_u32(&empty_bar[b]), static_cast<uint32_t>((jj / kT2S + 1) & 1),
                                   &abort_flag, &g_bnn_tc_ternary_errors))
        break;
      const uint32_t bar = smem_u32(&full_bar[b]);
      mbar_expect_tx(bar, BN * 128u);
      tma_load_2d(smem_u32(smem + b * kT2Stage + kT2AStage), &tmap_x, static_cast<int>(64 * (sb + jj)),
                  static_cast<int>(i0), bar);
    }
  }
  __syncwarp();

  // -------------------------------------------------------------- epilogue
  bool drained = true;
  if (warp < 8) {
    drained = mbar_drain(smem_u32(&done_bar), 0u, &g_bnn_tc_ternary_errors);
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  }
  const bool good = __syncthreads_and(drained && abort_flag == 0) != 0;
  const int erow = 32 * (warp & 3) + (tid & 31);       // weight row (tensor-memory lane)
  const int ecol0 = (warp >> 2) * (BN / 2);          // half of the activation columns
  const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
  const int64_t jrow = j0 + erow;
  if constexpr (KS == 1) {
    if (warp < 8 && good) {
      const bool jlive = jrow < n;
      const float sc = jlive ? __ldg(scale + jrow) : 0.0f, bv = (bias && jlive) ? __ldg(bias + jrow) : 0.0f;
      for (int c0 = ecol0; c0 < ecol0 + BN / 2; c0 += 16) {
        uint32_t r[16];
        if (nst > 0) {  // every lane of the warp takes part in the collective load
          tmem_ld16(taddr + static_cast<uint32_t>(c0), r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) r[c] = 0u;
        }
        if (jlive) {
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int64_t gi = i0 + c0 + c;
            const float acc = __uint_as_float(r[c]);
            if (gi < m) out[gi * n + jrow] = bias ? sc * acc + bv : sc * acc;
          }
        }
      }
    }
  } else {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    float* recv = reinterpret_cast<float*>(smem);  // [source rank][weight row][column, padded]
    cluster.sync();                               // every CTA's tensor core is done with its stages
    if (tid == 0 && !good)
      for (int q = 0; q < KS; ++q) atomicExch(cluster.map_shared_rank(&any_bad, q), 1);
    if (warp < 8 && good) {
      for (int c0 = ecol0; c0 < ecol0 + BN / 2; c0 += 16) {
        uint32_t r[16];
        if (nst > 0) {
          tmem_ld16(taddr + static_cast<uint32_t>(c0), r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) r[c] = 0u;
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int col = c0 + 4 * g;
          float* dst = cluster.map_shared_rank(recv, col / kCols);
          *reinterpret_cast<float4*>(dst + (rank * kT2M + erow) * kPitch + col % kCols) =
              make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]), __uint_as_float(r[4 * g + 2]),
                          __uint_as_float(r[4 * g + 3]));
        }
      }
    }
    cluster.sync();  // every share has landed
    if (any_bad == 0) {
      for (int e = tid; e < kT2M * (kCols / 4); e += blockDim.x) {
        const int wr = e % kT2M, cl = 4 * (e / kT2M);
        const int64_t gj = j0 + wr;
        if (gj >= n) continue;
        float4 a = *reinterpret_cast<const float4*>(recv + wr * kPitch + cl);
#pragma unroll
        for (int q = 1; q < KS; ++q) {  // rank order
          const float4 v = *reinterpret_cast<const float4*>(recv + (q * kT2M + wr) * kPitch + cl);
          a.x += v.x;
          a.y += v.y;
          a.z += v.z;
          a.w += v.w;
        }
        const float sc = __ldg(scale + gj), bv = bias ? __ldg(bias + gj) : 0.0f;
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int64_t gi = i0 + rank * kCols + cl + t;
          if (gi < m) out[gi * n + gj] = bias ? sc * av[t] + bv : sc * av[t];
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  if (warp == kMmaWarp)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(BN));
}

template <int KS, int BN>
bnn_status launch_tc2(const CUtensorMap& tx, const uint16_t* packed, const float* scale, const float* bias, int64_t m,
                      int64_t n, int64_t k, int64_t kt, float* out, cudaStream_t s) {
  const int64_t gx = KS * ((n + kT2M - 1) / kT2M), gy = (m + BN - 1) / BN;
  if (gx > 2147483647LL || gy > 65535) return BNN_ERR_INVALID_ARG;
  const size_t smem = static_cast<size_t>(kT2S) * (kT2AStage + BN * 128u) + 1024;
  auto kern = ternary_gemm_tc2_kernel<KS, BN>;
  BNN_TRY(bnn::ensure_smem(kern, smem));
  const cudaError_t e = bnn::launch_pdl(kern, dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)),
                                   dim3(kT2Threads), smem, s, KS, tx, packed, scale, bias, m, n, k, kt, out);
  if (e != cudaSuccess) return bnn::cuda_fail(e);
  return bnn::check_launch();
}

// ---------------------------------------------------------------------------
// Decode-bound shapes (at most 64 activation rows): the decoded trits go to
// tensor memory.
//
// With one activation tile every packed word is decoded exactly once, so the
// decode is the whole cost.  Here it writes no shared memory: each producer
// thread owns one weight row (its tensor-memory lane) and one 64-trit quarter
// of a 256-trit stage, decodes its 32 bf16 pairs into registers (each word's
// five pairs from two 81-entry quad-table loads and one pair-table load,
// specialised per warp-uniform phase) and stores them with one
// tcgen05.st.32x32b.x32 into the stage's A slot of tensor memory; the MMA reads
// A from there ([a-tmem] operand) and B, the activations, from shared memory
// (four TMA boxes of 64 x 64 bf16 per stage, 128-byte swizzle).  The packed
// words reach shared memory without passing through registers.  When the
// tile's rows fit the word region (a CTA that takes every stage of its rows,
// rows x k <= about 600 K trits), they are one contiguous byte range of the
// matrix, which one thread bulk-copies at the start (before the programmatic-
// launch wait: weights do not depend on the kernel ahead), so the decode never
// waits for words again.  Otherwise the loader warps copy, per group of five
// stages (1280 trits = 128 words, 129 when the
// group starts inside a word), every row's window as 4-byte cp.async units
// (the row's bytes from the 4-byte boundary at or below its first word; units
// past the end of the matrix are zero-filled) into a [row][65 units] buffer
// (odd stride: a warp's 32 rows read 32 different banks), double-buffered and
// completed on an mbarrier by cp.async.mbarrier.arrive (eight loader warps; the
// producers sleep between polls while a group's words arrive, leaving the
// issue slots to the loaders).  Per stage a producer
// waits for its slot to be free, decodes, stores, waits for the store and
// arrives once per warp; one thread waits for the A slot and the B tile and
// issues 16 tcgen05.mma (K = 16).  A cluster of KS CTAs splits the stages;
// the partial tiles are added in rank order through distributed shared
// memory, each CTA owning a block of activation columns (multiples of 4).
// ---------------------------------------------------------------------------
constexpr int kT3M = 128;                              // weight rows = tensor-memory lanes
constexpr int kT3N = 64;                               // activation rows (UMMA N)
constexpr int kT3K = 256;                              // trits per stage
constexpr int kT3S = 3;                                // stages in flight
constexpr int kT3G = 5;                                // stages per word group (1280 trits)
constexpr int kT3GU = 65;                              // 4-byte units staged per row and group (129 words + offset)
constexpr int kT3Prod = 512;                           // producer threads (16 warps)
constexpr int kT3Load = 256;                           // loader threads (8 warps)
constexpr int kT3Threads = kT3Prod + 64 + kT3Load;     // + MMA warp + TMA warp + loaders
constexpr uint32_t kT3BAtom = kT3N * 128u;             // one 64-trit box of activations
constexpr uint32_t kT3BStage = 4 * kT3BAtom;
constexpr uint32_t kT3WBuf = kT3M * kT3GU * 4u;        // one group's words
constexpr uint32_t kT3WRegion = 120000u;               // packed words: two groups, or a whole tile (+ slack)
static_assert(2 * kT3WBuf <= kT3WRegion, "two word groups fit the word region");
constexpr uint32_t kT3Cols = 512;                      // D (64 columns) + kT3S A slots of 128
constexpr int kT3Units = kT3N / 4;                     // activation columns in units of 4
static_assert(kT3N + 128 * kT3S <= static_cast<int>(kT3Cols), "tensor-memory columns");
static_assert(kT3GU * 4 >= 2 + 2 * (kT3G * kT3K / 10 + 1), "a group's words (from a 2-byte offset) fit its units");

// Word decode for this kernel: a word's five bf16 pairs from three table loads.
// With F = w * kFix (the fixed-point fraction w / 3^10, see the file header),
// the high word of 81 F is the base-81 number of digits 6..9, and of 81 times
// the low word of 81 F that of digits 2..5; 9 times what remains gives digits
// 0..1 (the errors stay below the digit boundaries for every w < 3^10; checked
// at compile time below).  A 4-digit code indexes an 81-entry table of two
// bf16 pairs (8 bytes: the pairs of its digits (0,1) and (2,3)), a 2-digit code
// the 9-entry pair table.  The 81-entry table is stored 16 times, copy c in the
// 8-byte bank pair c (entry v of copy c at byte 128 v + 8 c), and lane l reads
// copy l % 16: the 16 lanes of each half-warp then hit 16 different bank pairs
// whatever codes they decode.
constexpr bool quad_digits_exact() {
  for (uint32_t w = 0; w < 59049u; ++w) {
    const uint32_t F = w * kFix;
    const uint32_t va = static_cast<uint32_t>((static_cast<uint64_t>(F) * 81u) >> 32);
    const uint32_t F1 = F * 81u;
    const uint32_t vb = static_cast<uint32_t>((static_cast<uint64_t>(F1) * 81u) >> 32);
    const uint32_t F2 = F1 * 81u;
    const uint32_t vc = static_cast<uint32_t>((static_cast<uint64_t>(F2) * 9u) >> 32);
    if (va != w / 729u || vb != (w / 9u) % 81u || vc != w % 9u) return false;
  }
  return true;
}
static_assert(quad_digits_exact(), "base-81 / base-9 digit extraction from the fixed-point fraction");

constexpr uint32_t kQuadTableBytes = 81u * 128u;  // 16 interleaved copies of 81 x 8 bytes

// the 32 bf16 pairs of 64 trits starting at phase PH of word 0 (w[i] = word i)
template <int PH>
__device__ __forceinline__ void decode64(const uint32_t (&w)[8], const uint32_t* lut, uint32_t quad_lane,
                                         uint32_t (&a)[32]) {
  constexpr int P0 = PH / 2;            // first pair, counted from word 0
  constexpr int W1 = (P0 + 31) / 5;     // last word needed
  uint32_t pr[8][5];
#pragma unroll
  for (int j = 0; j <= W1; ++j) {
    const uint32_t F = w[j] * kFix;
    const uint32_t va = __umulhi(F, 81u);        // digits 6..9
    const uint32_t F1 = F * 81u;
    const uint32_t vb = __umulhi(F1, 81u);       // digits 2..5
    const uint32_t vc = __umulhi(F1 * 81u, 9u);  // digits 0..1
    uint32_t a0, a1, b0, b1;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];\n" : "=r"(a0), "=r"(a1) : "r"(quad_lane + va * 128u));
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];\n" : "=r"(b0), "=r"(b1) : "r"(quad_lane + vb * 128u));
    pr[j][0] = lut[vc];
    pr[j][1] = b0;
    pr[j][2] = b1;
    pr[j][3] = a0;
    pr[j][4] = a1;
  }
#pragma unroll
  for (int p = 0; p < 32; ++p) a[p] = pr[(P0 + p) / 5][(P0 + p) % 5];
}

__device__ __forceinline__ void tmem_st32(uint32_t addr, const uint32_t (&a)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(addr),
      "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]), "r"(a[8]), "r"(a[9]),
      "r"(a[10]), "r"(a[11]), "r"(a[12]), "r"(a[13]), "r"(a[14]), "r"(a[15]), "r"(a[16]), "r"(a[17]), "r"(a[18]),
      "r"(a[19]), "r"(a[20]), "r"(a[21]), "r"(a[22]), "r"(a[23]), "r"(a[24]), "r"(a[25]), "r"(a[26]), "r"(a[27]),
      "r"(a[28]), "r"(a[29]), "r"(a[30]), "r"(a[31])
      : "memory");
}

// 4 bytes from global to shared (src_bytes of them read, the rest zero)
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// first activation column owned by cluster rank q (blocks of whole units of 4)
template <int KS>
__device__ __forceinline__ int t3_col_begin(int q) { return 4 * ((kT3Units * q) / KS); }

template <int KS>
__global__ void __launch_bounds__(kT3Threads, 1)
ternary_gemm_tmem_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint16_t* __restrict__ packed,
                         const float* __restrict__ scale, const float* __restrict__ bias, int64_t m, int64_t n,
                         int64_t k, int64_t kt, int rows_cta, int preload, float* __restrict__ out) {
  using namespace bnn::tc;
  constexpr int kMaxCols = 4 * ((kT3Units + KS - 1) / KS);
  constexpr int kPitch = kMaxCols + 4;  // padded receive row (floats)
  static_assert(KS * kT3M * kPitch * 4 <= kT3S * kT3BStage, "split-K shares must fit the activation stages");

  extern __shared__ __align__(16) uint8_t t3_raw[];
  __shared__ __align__(8) uint64_t a_full[kT3S];   // one arrive per producer warp
  __shared__ __align__(8) uint64_t b_full[kT3S];   // the TMA thread's expect_tx + bytes
  __shared__ __align__(8) uint64_t empty_bar[kT3S];
  __shared__ __align__(8) uint64_t w_full[2];      // the loaders' copies of a group's words
  __shared__ __align__(8) uint64_t w_empty[2];     // one arrive per producer warp after the group
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ uint32_t tmem_holder;
  __shared__ volatile int abort_flag;
  __shared__ int any_bad;
  __shared__ uint32_t lut[9];
  uint8_t* const bsm = t3_raw + ((1024u - (smem_u32(t3_raw) & 1023u)) & 1023u);  // kT3S activation stages
  // the packed words: the whole tile's rows (preload) or [2][kT3M][kT3GU] units of a word group
  uint8_t* const wbuf = bsm + kT3S * kT3BStage;
  uint2* const quad = reinterpret_cast<uint2*>(wbuf + kT3WRegion + 16);           // 81-entry table, 16 copies

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = KS > 1 ? static_cast<int>(blockIdx.x % KS) : 0;
  const int64_t j0 = static_cast<int64_t>(blockIdx.x / KS) * rows_cta;  // first weight row (rows_cta: 32..128)
  const int64_t i0 = static_cast<int64_t>(blockIdx.y) * kT3N;        // first activation row
  const int64_t total = (k + kT3K - 1) / kT3K;  // stages up to trit k (past it, only pad trits of the last word)
  const int64_t share = (total + KS - 1) / KS;
  const int64_t sb = rank * share < total ? rank * share : total;
  const int64_t se = sb + share < total ? sb + share : total;
  const int nst = static_cast<int>(se - sb);
  const int ngroups = (nst + kT3G - 1) / kT3G;
  constexpr int kMmaWarp = kT3Prod / 32, kTmaWarp = kMmaWarp + 1, kLoadWarp0 = kMmaWarp + 2;
  const int prod_warps = 4 * (rows_cta / 32);  // producer warps with rows: 4 quarters of the stage per 32 rows
  const int64_t rows_live = n - j0 < rows_cta ? n - j0 : rows_cta;

  if (tid < 9) {
    const int lo = tid % 3, hi = tid / 3;  // digit = trit + 1
    const uint32_t blo = lo == 0 ? 0xBF80u : (lo == 2 ? 0x3F80u : 0u);
    const uint32_t bhi = hi == 0 ? 0xBF80u : (hi == 2 ? 0x3F80u : 0u);
    lut[tid] = blo | (bhi << 16);
  }
  for (int e = tid; e < 81 * 16; e += kT3Threads) {  // entry v (digits d0..d3 of v), copy c
    const int v = e >> 4;
    uint32_t h[4];
#pragma unroll
    for (int i = 0, t = v; i < 4; ++i, t /= 3) h[i] = t % 3 == 0 ? 0xBF80u : (t % 3 == 2 ? 0x3F80u : 0u);
    quad[e] = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
  }
  if (tid == 0) {
    for (int i = 0; i < kT3S; ++i) {
      mbar_init(smem_u32(&a_full[i]), prod_warps);
      mbar_init(smem_u32(&b_full[i]), 1);
      mbar_init(smem_u32(&empty_bar[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&w_full[i]), preload ? 1 : kT3Load);  // preload: the copying thread's expect_tx
      mbar_init(smem_u32(&w_empty[i]), prod_warps);
    }
    mbar_init(smem_u32(&done_bar), 1);
    abort_flag = 0;
    any_bad = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (tid == kTmaWarp * 32)
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(&tmem_holder)),
                 "r"(kT3Cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const uint32_t tmem = tmem_holder;  // D: columns [0, 64); A slot i: columns [64 + 128 i, 192 + 128 i)
  bnn::pdl_trigger();

  if (tid < kT3Prod) {
    // ------------------------------------------------------------ producers
    // (warps whose 32 rows lie past rows_cta have nothing to do: their lanes
    // of the accumulator are never stored)
    const int row = 32 * (warp & 3) + lane;  // weight row of the tile = tensor-memory lane
    const int qk = warp >> 2;                // 64-trit quarter of each stage
    const uint32_t lane_field = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t quad_lane = smem_u32(quad) + 8u * static_cast<uint32_t>(lane & 15);  // this lane's table copy
    bool ok = 32 * (warp & 3) < rows_cta;
    // stage jj of this quarter from the words at wr (the word holding its first trit)
    auto stage = [&](int jj, const uint16_t* wr, int64_t jw, int64_t t0) -> bool {
      const int slot = jj % kT3S;
      const bool fine = jj < kT3S || mbar_wait(smem_u32(&empty_bar[slot]), static_cast<uint32_t>((jj / kT3S + 1) & 1),
                                               &abort_flag, &g_bnn_tc_ternary_errors);
      if (!__all_sync(0xffffffffu, fine)) return false;  // the tensor-memory store below is warp-collective
      asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
      uint32_t W[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) W[i] = wr[i];
      uint32_t av[32];
      switch (static_cast<int>(t0 - 10 * jw)) {  // the phase, warp-uniform
        case 0: decode64<0>(W, lut, quad_lane, av); break;
        case 2: decode64<2>(W, lut, quad_lane, av); break;
        case 4: decode64<4>(W, lut, quad_lane, av); break;
        case 6: decode64<6>(W, lut, quad_lane, av); break;
        default: decode64<8>(W, lut, quad_lane, av); break;
      }
      tmem_st32(tmem + lane_field + static_cast<uint32_t>(kT3N + 128 * slot + 32 * qk), av);
      asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
      asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&a_full[slot]));
      return true;
    };
    if (preload) {
      // every word of the tile's rows is in shared memory once the copy lands
      // (row r at byte pre_off + 2 kt r, pre_off = the tile's offset from a
      // 16-byte boundary)
      const bool fine = ok && mbar_wait_idle(smem_u32(&w_full[0]), 0u, &abort_flag, &g_bnn_tc_ternary_errors);
      if (!__all_sync(0xffffffffu, fine)) ok = false;
      const uint32_t pre_off = static_cast<uint32_t>((2 * j0 * kt) & 15);
      const uint16_t* wrow = reinterpret_cast<const uint16_t*>(wbuf + pre_off) + static_cast<int64_t>(row) * kt;
      for (int jj = 0; jj < nst && ok; ++jj) {
        const int64_t t0 = kT3K * (sb + jj) + 64 * qk;  // first trit of this quarter
        const int64_t jw = t0 / 10;
        ok = stage(jj, wrow + jw, jw, t0);
      }
    } else {
      for (int g = 0; g < ngroups && ok; ++g) {
        const int buf = g & 1;
        // sleeping between polls: the loaders need the issue slots while the group's words arrive
        const bool fine = mbar_wait_idle(smem_u32(&w_full[buf]), static_cast<uint32_t>((g >> 1) & 1), &abort_flag,
                                         &g_bnn_tc_ternary_errors);
        if (!__all_sync(0xffffffffu, fine)) break;
        const int64_t s0 = sb + kT3G * static_cast<int64_t>(g);  // first stage of the group
        const int64_t w0 = (kT3K * s0) / 10;                     // first word staged
        // this row's words in the buffer: its first staged byte sits at the row's
        // byte offset mod 4 within its units
        const int64_t rbyte = ((j0 + row) * kt + w0) * 2;
        const uint16_t* wrow =
            reinterpret_cast<const uint16_t*>(wbuf + buf * kT3WBuf + row * (kT3GU * 4) + (rbyte & 3));
        for (int u = 0; u < kT3G && ok; ++u) {
          const int jj = kT3G * g + u;
          if (jj >= nst) break;
          const int64_t t0 = kT3K * (sb + jj) + 64 * qk;  // first trit of this quarter
          const int64_t jw = t0 / 10;
          ok = stage(jj, wrow + (jw - w0), jw, t0);
        }
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(smem_u32(&w_empty[buf]));  // this warp is done with the group's words
      }
    }
  } else if (warp >= kLoadWarp0) {
    // ------------------------------------------------------------ loaders of the packed words
    const int lt = tid - kLoadWarp0 * 32;
    const uint8_t* gbase = reinterpret_cast<const uint8_t*>(packed);
    const int64_t total_bytes = n * kt * 2;
    if (preload) {
      // one thread: the tile's rows are one contiguous byte range [a0, a1) of the
      // matrix; bulk-copy it from the 16-byte boundary at or below a0 (pieces of
      // at most 32 KiB, ending at the last 16-byte boundary inside the matrix),
      // the bytes after that boundary (fewer than 16) by plain loads
      if (lt == 0) {
        const uint64_t base = reinterpret_cast<uint64_t>(gbase);
        const uint64_t a0 = base + static_cast<uint64_t>(2 * j0 * kt);
        const uint64_t a1 = base + static_cast<uint64_t>(2 * (j0 + rows_live) * kt);
        const uint64_t f0 = a0 & ~uint64_t{15};
        const uint64_t t16 = (base + static_cast<uint64_t>(total_bytes)) & ~uint64_t{15};
        uint64_t f1 = (a1 + 15u) & ~uint64_t{15};
        if (f1 > t16) f1 = t16;
        if (f1 < f0) f1 = f0;
        for (uint64_t p = (f1 > a0 ? f1 : a0); p < a1; ++p) wbuf[p - f0] = gbase[p - base];
        const uint32_t bar = smem_u32(&w_full[0]);
        mbar_expect_tx(bar, static_cast<uint32_t>(f1 - f0));  // after the plain stores: they are released with it
        for (uint64_t p = f0; p < f1; p += 32768u) {
          const uint32_t bytes = static_cast<uint32_t>(f1 - p < 32768u ? f1 - p : 32768u);
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                  smem_u32(wbuf + (p - f0))),
              "l"(p), "r"(bytes), "r"(bar)
              : "memory");
        }
        mbar_drain(bar, 0u, &g_bnn_tc_ternary_errors);  // no copy in flight when the CTA retires
      }
    } else {
    // this thread's units idx = lt + kT3Load i, walked as (row, unit) without divisions
    const int r_first = lt / kT3GU, u_first = lt - r_first * kT3GU;
    constexpr int kDr = kT3Load / kT3GU, kDu = kT3Load % kT3GU;
    for (int g = 0; g < ngroups; ++g) {
      const int buf = g & 1;
      if (g >= 2 && !mbar_wait_idle(smem_u32(&w_empty[buf]), static_cast<uint32_t>(((g >> 1) + 1) & 1), &abort_flag,
                               &g_bnn_tc_ternary_errors))
        break;
      const int64_t w0 = (kT3K * (sb + kT3G * static_cast<int64_t>(g))) / 10;
      const uint32_t dbase = smem_u32(wbuf + buf * kT3WBuf);
      const int64_t first = 2 * (j0 * kt + w0);  // byte of the group's first word in row 0 of the tile
      int r = r_first, un = u_first;
      for (int idx = lt; idx < rows_cta * kT3GU; idx += kT3Load) {
        const int64_t a = ((first + 2 * static_cast<int64_t>(r) * kt) & ~int64_t{3}) + 4 * un;  // 4-byte unit
        const int64_t left = r < rows_live ? total_bytes - a : 0;
        const uint32_t bytes = left >= 4 ? 4u : (left > 0 ? static_cast<uint32_t>(left) : 0u);
        cp_async4(dbase + static_cast<uint32_t>(idx) * 4u, gbase + (bytes ? a : 0), bytes);
        un += kDu;
        r += kDr;
        if (un >= kT3GU) {
          un -= kT3GU;
          ++r;
        }
      }
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(smem_u32(&w_full[buf])) : "memory");
    }
    asm volatile("cp.async.wait_all;\n" ::: "memory");  // no copy in flight when the CTA retires
    }
  } else if (tid == kMmaWarp * 32) {
    // ------------------------------------------------------------ MMA issue
    // D f32, A (tensor memory) and B bf16, K-major, N = 64, M = 128
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(kT3N) >> 3) << 17) |
                           ((static_cast<uint32_t>(kT3M) >> 4) << 24);
    const uint32_t base = smem_u32(bsm);
    for (int jj = 0; jj < nst; ++jj) {
      const int slot = jj % kT3S;
      const uint32_t par = static_cast<uint32_t>((jj / kT3S) & 1);
      if (!mbar_wait_idle(smem_u32(&b_full[slot]), par, &abort_flag, &g_bnn_tc_ternary_errors) ||
          !mbar_wait_idle(smem_u32(&a_full[slot]), par, &abort_flag, &g_bnn_tc_ternary_errors))
        break;
      asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        const uint64_t bd = sw128_desc(base + slot * kT3BStage + (kk >> 2) * kT3BAtom) +
                            static_cast<uint64_t>(2 * (kk & 3));
        const uint32_t at = tmem + static_cast<uint32_t>(kT3N + 128 * slot + 8 * kk);
        const uint32_t acc = (jj > 0 || kk > 0) ? 1u : 0u;
        asm volatile(
            "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(tmem),
            "r"(at), "l"(bd), "r"(idesc), "r"(acc));
      }
      mma_commit(smem_u32(&empty_bar[slot]));
    }
    mma_commit(smem_u32(&done_bar));
  } else if (tid == kTmaWarp * 32) {
    // ------------------------------------------------------------ TMA copies of the activations
    bnn::pdl_wait();  // x may come from the preceding kernel
    int issued = 0;
    for (int jj = 0; jj < nst; ++jj) {
      const int slot = jj % kT3S;
      if (jj >= kT3S && !mbar_wait_idle(smem_u32(&empty_bar[slot]), static_cast<uint32_t>((jj / kT3S + 1) & 1),
                                        &abort_flag, &g_bnn_tc_ternary_errors))
        break;
      const uint32_t bar = smem_u32(&b_full[slot]);
      const uint32_t dst = smem_u32(bsm + slot * kT3BStage);
      mbar_expect_tx(bar, kT3BStage);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        tma_load_2d(dst + q * kT3BAtom, &tmap_x, static_cast<int>(kT3K * (sb + jj) + 64 * q), static_cast<int>(i0),
                    bar);
      issued = jj + 1;
    }
    // no copy may still be in flight when the CTA retires
    for (int jj = issued - kT3S; jj < issued; ++jj)
      if (jj >= 0)
        mbar_drain(smem_u32(&b_full[jj % kT3S]), static_cast<uint32_t>((jj / kT3S) & 1), &g_bnn_tc_ternary_errors);
  }
  __syncwarp();

  // -------------------------------------------------------------- epilogue
  bool drained = true;
  if (warp < 8) {
    drained = mbar_drain(smem_u32(&done_bar), 0u, &g_bnn_tc_ternary_errors);
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  }
  const bool good = __syncthreads_and(drained && abort_flag == 0) != 0;
  const int erow = 32 * (warp & 3) + lane;       // weight row (tensor-memory lane)
  const int ecol0 = (warp >> 2) * (kT3N / 2);    // half of the activation columns
  const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
  const int64_t jrow = j0 + erow;
  if constexpr (KS == 1) {
    if (warp < 8 && good) {
      const bool jlive = erow < rows_live;
      const float sc = jlive ? __ldg(scale + jrow) : 0.0f, bv = (bias && jlive) ? __ldg(bias + jrow) : 0.0f;
      for (int c0 = ecol0; c0 < ecol0 + kT3N / 2; c0 += 16) {
        uint32_t r[16];
        if (nst > 0) {  // every lane of the warp takes part in the collective load
          tmem_ld16(taddr + static_cast<uint32_t>(c0), r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) r[c] = 0u;
        }
        if (jlive) {
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int64_t gi = i0 + c0 + c;
            const float acc = __uint_as_float(r[c]);
            if (gi < m) out[gi * n + jrow] = bias ? sc * acc + bv : sc * acc;
          }
        }
      }
    }
  } else {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    float* recv = reinterpret_cast<float*>(bsm);  // [source rank][weight row][owned column, padded]
    cluster.sync();                              // every CTA's tensor core is done with its stages
    if (tid == 0 && !good)
      for (int q = 0; q < KS; ++q) atomicExch(cluster.map_shared_rank(&any_bad, q), 1);
    if (warp < 8 && good) {
      for (int c0 = ecol0; c0 < ecol0 + kT3N / 2; c0 += 16) {
        uint32_t r[16];
        if (nst > 0) {
          tmem_ld16(taddr + static_cast<uint32_t>(c0), r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) r[c] = 0u;
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int col = c0 + 4 * g;
          int q = 0;
#pragma unroll
          for (int t = 1; t < KS; ++t) q += col >= t3_col_begin<KS>(t) ? 1 : 0;
          float* dst = cluster.map_shared_rank(recv, q);
          *reinterpret_cast<float4*>(dst + (rank * kT3M + erow) * kPitch + (col - t3_col_begin<KS>(q))) =
              make_float4(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1]), __uint_as_float(r[4 * g + 2]),
                          __uint_as_float(r[4 * g + 3]));
        }
      }
    }
    cluster.sync();  // every share has landed
    if (any_bad == 0) {
      const int cb = t3_col_begin<KS>(rank), ncols = t3_col_begin<KS>(rank + 1) - cb;
      for (int e = tid; e < kT3M * (ncols / 4); e += blockDim.x) {
        const int wr = e % kT3M, cl = 4 * (e / kT3M);
        const int64_t gj = j0 + wr;
        if (wr >= rows_live) continue;
        float4 a = *reinterpret_cast<const float4*>(recv + wr * kPitch + cl);
#pragma unroll
        for (int q = 1; q < KS; ++q) {  // rank order
          const float4 v = *reinterpret_cast<const float4*>(recv + (q * kT3M + wr) * kPitch + cl);
          a.x += v.x;
          a.y += v.y;
          a.z += v.z;
          a.w += v.w;
        }
        const float sc = __ldg(scale + gj), bv = bias ? __ldg(bias + gj) : 0.0f;
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int64_t gi = i0 + cb + cl + t;
          if (gi < m) out[gi * n + gj] = bias ? sc * av[t] + bv : sc * av[t];
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  if (warp == kMmaWarp)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kT3Cols));
}

// dynamic shared memory: 1024-byte alignment slack, the activation stages, two
// word buffers, 16 bytes past them (a producer may read, and not use, the word
// after its row's window) and the interleaved copies of the 81-entry table
size_t tmem_smem_bytes() { return 1024 + static_cast<size_t>(kT3S) * kT3BStage + kT3WRegion + 16 + kQuadTableBytes; }

// whether a tile of rows_cta rows fits the word region whole (with 16 bytes of
// alignment and 32 bytes read past the last word)
bool tmem_preload_fits(int rows_cta, int64_t kt) {
  return static_cast<int64_t>(rows_cta) * kt * 2 + 16 + 32 <= static_cast<int64_t>(kT3WRegion);
}

// clusters of KS CTAs of the tensor-memory kernel that can run at once (0 when unknown)
template <int KS>
int tmem_active_clusters() {
  static std::mutex mu;
  static int cached[64] = {};
  const int dev = bnn::current_device();
  if (dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] != 0) return cached[dev] > 0 ? cached[dev] : 0;
  auto kern = ternary_gemm_tmem_kernel<KS>;
  int num = 0;
  if (bnn::ensure_smem(kern, tmem_smem_bytes()) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(KS * 128, 1, 1);
    cfg.blockDim = dim3(kT3Threads, 1, 1);
    cfg.dynamicSmemBytes = tmem_smem_bytes();
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = KS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&num, kern, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      num = 0;
    }
  }
  cached[dev] = num > 0 ? num : -1;
  return num > 0 ? num : 0;
}

template <int KS>
bnn_status launch_tmem(const CUtensorMap& tx, const uint16_t* packed, const float* scale, const float* bias, int64_t m,
                       int64_t n, int64_t k, int64_t kt, int rows_cta, float* out, cudaStream_t s) {
  const int64_t gx = KS * ((n + rows_cta - 1) / rows_cta), gy = (m + kT3N - 1) / kT3N;
  if (gx > 2147483647LL || gy > 65535) return BNN_ERR_INVALID_ARG;
  auto kern = ternary_gemm_tmem_kernel<KS>;
  const size_t smem = tmem_smem_bytes();
  BNN_TRY(bnn::ensure_smem(kern, smem));
  // (a rank of a split-K cluster needs only its share of each row's words: group loads)
  const int preload = (KS == 1 && tmem_preload_fits(rows_cta, kt)) ? 1 : 0;
  const cudaError_t e = bnn::launch_pdl(kern, dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)),
                                        dim3(kT3Threads), smem, s, KS, tx, packed, scale, bias, m, n, k, kt, rows_cta,
                                        preload, out);
  if (e != cudaSuccess) return bnn::cuda_fail(e);
  return bnn::check_launch();
}

}  // namespace

namespace bnn {

int ternary_tc_error_count(int reset) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_bnn_tc_ternary_errors, sizeof(v)) != cudaSuccess) return -1;
  if (reset) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_bnn_tc_ternary_errors, &zero, sizeof(zero)) != cudaSuccess) return -1;
  }
  return static_cast<int>(v);
}

// Choose the rows per CTA (32..128) and the cluster split of the stages for
// the fewest waves times the time of a CTA, in units of a 128-row stage / 128:
// the decode scales with the rows (not below 64: fewer warps hide less
// latency), and every CTA pays about two stages of start-up (its first words),
// plus two for the exchange of a split.  CTAs of a cluster take whole SMs, so
// few clusters of 3 or 4 run at once.
void ternary_tmem_plan(int64_t n, int64_t k, const int active[4], int* rows, int* ks) {
  const int64_t stages = (k + kT3K - 1) / kT3K;
  int best_ks = 1, best_rows = kT3M;
  int64_t best_cost = INT64_MAX;
  for (int r = kT3M; r >= 32; r -= 32) {
    const int64_t tiles = (n + r - 1) / r;
    for (int c = 1; c <= 4; ++c) {
      if (active[c - 1] <= 0 || (c > 1 && stages < 2 * c)) continue;
      const int64_t waves = (tiles + active[c - 1] - 1) / active[c - 1];
      const int64_t cost = waves * ((r < 64 ? 64 : r) * ((stages + c - 1) / c) + 256 + (c > 1 ? 256 : 32));
      if (cost < best_cost) {
        best_cost = cost;
        best_ks = c;
        best_rows = r;
      }
    }
  }
  *rows = best_rows;
  *ks = best_ks;
}

bnn_status ternary_gemm_tc(const uint16_t* x_bf16, const uint16_t* packed, const float* scale, const float* bias,
                           int64_t m, int64_t n, int64_t k, float* out, cudaStream_t s) {
  const int64_t kt = words10(k);
  // activation rows TMA can copy (16-byte aligned): the warp-specialised kernel
  CUtensorMap tx;
  if (k > 0 && k % 8 == 0 && k < (1LL << 31) && aligned(x_bf16, 16) && m < (1LL << 31) &&
      encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x_bf16, static_cast<uint64_t>(k), static_cast<uint64_t>(m),
                     static_cast<uint64_t>(k) * 2u, 64, kT2N, CU_TENSOR_MAP_SWIZZLE_128B)) {
    if (m <= kT3N && aligned(packed, 4)) {
      // one activation tile: decode-bound
      const int active[4] = {tmem_active_clusters<1>(), tmem_active_clusters<2>(), tmem_active_clusters<3>(),
                             tmem_active_clusters<4>()};
      int rows = kT3M, ks = 1;
      ternary_tmem_plan(n, k, active, &rows, &ks);
      switch (ks) {
        case 4: return launch_tmem<4>(tx, packed, scale, bias, m, n, k, kt, rows, out, s);
        case 3: return launch_tmem<3>(tx, packed, scale, bias, m, n, k, kt, rows, out, s);
        case 2: return launch_tmem<2>(tx, packed, scale, bias, m, n, k, kt, rows, out, s);
        default: return launch_tmem<1>(tx, packed, scale, bias, m, n, k, kt, rows, out, s);
      }
    }
    // activation tiles of 256 rows above m = 128, 128 above m = 64 (each weight
    // tile is decoded once per activation tile), else 64 (two CTAs per SM)
    const int bn = m > 128 ? 256 : (m > 64 ? 128 : 64);
    CUtensorMap txw;
    if (bn != 64 &&
        !encode_tmap_2d(&txw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x_bf16, static_cast<uint64_t>(k),
                        static_cast<uint64_t>(m), static_cast<uint64_t>(k) * 2u, 64, static_cast<uint32_t>(bn),
                        CU_TENSOR_MAP_SWIZZLE_128B))
      return BNN_ERR_CUDA;
    const int64_t tiles = ((n + kT2M - 1) / kT2M) * ((m + bn - 1) / bn);
    const int64_t stages = (10 * kt + 63) / 64;
    const int64_t slots = (bn == 64 ? 2LL : 1LL) * sm_count();
    const int ks = (tiles * 4 <= slots && stages >= 16) ? 4 : ((tiles * 2 <= slots && stages >= 8) ? 2 : 1);
    if (bn == 256) {
      if (ks == 4) return launch_tc2<4, 256>(txw, packed, scale, bias, m, n, k, kt, out, s);
      if (ks == 2) return launch_tc2<2, 256>(txw, packed, scale, bias, m, n, k, kt, out, s);
      return launch_tc2<1, 256>(txw, packed, scale, bias, m, n, k, kt, out, s);
    }
    if (bn == 128) {
      if (ks == 4) return launch_tc2<4, 128>(txw, packed, scale, bias, m, n, k, kt, out, s);
      if (ks == 2) return launch_tc2<2, 128>(txw, packed, scale, bias, m, n, k, kt, out, s);
      return launch_tc2<1, 128>(txw, packed, scale, bias, m, n, k, kt, out, s);
    }
    if (ks == 4) return launch_tc2<4, 64>(tx, packed, scale, bias, m, n, k, kt, out, s);
    if (ks == 2) return launch_tc2<2, 64>(tx, packed, scale, bias, m, n, k, kt, out, s);
    return launch_tc2<1, 64>(tx, packed, scale, bias, m, n, k, kt, out, s);
  }
  const int64_t ntiles = (n + kTcMW - 1) / kTcMW, gy = (m + kTcNX - 1) / kTcNX;
  if (ntiles * kTcK > 2147483647LL || gy > 65535) return BNN_ERR_INVALID_ARG;
  const int64_t total_stages = (10 * kt + 63) / 64;
  const int64_t slice_stages = (total_stages + kTcK - 1) / kTcK;
  const size_t smem = static_cast<size_t>(kTcStagesT) * (kAStage + kBStage) + 1024;
  const dim3 grid(static_cast<unsigned>(ntiles * kTcK), static_cast<unsigned>(gy));
  if (k % 8 == 0 && aligned(x_bf16, 16)) {
    BNN_TRY(ensure_smem(ternary_gemm_tc_kernel<true>, smem));
    ternary_gemm_tc_kernel<true><<<grid, kTcThreads, smem, s>>>(x_bf16, packed, scale, m, n, k, kt, slice_stages, out,
                                                                bias);
  } else {
    BNN_TRY(ensure_smem(ternary_gemm_tc_kernel<false>, smem));
    ternary_gemm_tc_kernel<false><<<grid, kTcThreads, smem, s>>>(x_bf16, packed, scale, m, n, k, kt, slice_stages,
                                                                 out, bias);
  }
  return check_launch();
}

}  // namespace bnn
