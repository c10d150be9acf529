// bnn_ternary_gemm on the 5th-generation tensor cores (tcgen05, sm_100a).
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

#include "bnn_internal.cuh"

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
constexpr uint32_t kSpin = 1u << 24;
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

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity) {
  for (uint32_t it = 0; it < kSpin; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
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

bnn_status ternary_gemm_tc(const uint16_t* x_bf16, const uint16_t* packed, const float* scale, const float* bias,
                           int64_t m, int64_t n, int64_t k, float* out, cudaStream_t s) {
  const int64_t kt = words10(k);
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
