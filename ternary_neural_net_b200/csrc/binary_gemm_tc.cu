// bnn_binary_gemm on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "Binary Math Effectiveness -- why / how / when", section 1: for +-1 vectors
// packed with bit 1 = -1, <x,w> = n - 2 popcount(x XOR w).  Writing a and b
// for the bits of x and w, popcount(x XOR w) = pa + pb - 2 popcount(a AND b),
// so <x,w> = k - 2 pa - 2 pb + 4 popcount(a AND b), where pa and pb are the
// row popcounts.  popcount(a AND b) is the dot product of the rows' bits as
// 0/1 bytes, which an int8 MMA sums exactly into int32.  Pad bits are 0 in
// both rows and so add nothing to any of the three counts.
//
// Tile: UMMA M = 128 weight rows (operand A) x N = BN activation rows (operand
// B), K in stages of 128 bits.  Roles inside a CTA:
//   - producer threads, two per row of the stacked (weight, activation) tile,
//     each owning one 64-bit word of the row per stage: load it (prefetched
//     kPre stages ahead in registers), count its bits, and write its 64 0/1
//     bytes (per 4 bytes a shift and an AND) in the 128-byte-swizzled K-major
//     layout the tensor core reads, then arrive on the stage's "full" mbarrier;
//   - one MMA thread: waits for "full", issues 4 tcgen05.mma.kind::i8 (K = 32)
//     into the int32 accumulator in tensor memory and commits to the stage's
//     "empty" mbarrier, which the producers wait on before refilling it;
//   - the epilogue (warps 0-7; warp w reads tensor-memory lanes 32(w%4).. and
//     half w/4 of the columns): tcgen05.ld, the popcount correction, alpha,
//     and stores in which the 32 lanes of a warp write 32 consecutive weight
//     columns of one output row.
// Any bijection between the 128 bits and the 128 k-slots of a stage gives the
// same sum when both operands use it; here byte j of word s of 16-byte chunk
// 2h+q holds bit 32h + 8j + 4q + s.
// Narrow tiles (BN = 64) keep 96 KB of stages so that two CTAs share an SM:
// the producers' shift/AND/store chains need many warps to hide their latency.
//
// Split K: a cluster of KS CTAs shares one output tile, each taking a
// contiguous share of the stages.  Each CTA turns its accumulator into its
// share of the dot (-2 pa - 2 pb + 4 S over its stages) and stores it straight
// into the shared memory of the CTA that owns that output row (distributed
// shared memory); CTA r adds the KS shares of its BN/KS output rows and writes
// them.  Integer addition makes the result independent of the order.
//
// Every wait on an mbarrier is bounded.  A wait that runs out bumps a
// device-side error count (bnn_device_error_count) and raises a CTA-wide abort
// flag that ends the other waits; the CTA then skips its stores, waits
// (bounded) for the MMAs it issued, frees its tensor memory and returns.
#include <cooperative_groups.h>

#include "bnn_internal.cuh"

// Bounded waits that ran out in this file's kernels (read by bnn_device_error_count).
__device__ unsigned int g_bnn_device_errors = 0;

namespace {

constexpr int kTm = 128;                   // weight rows per tile (UMMA M)
constexpr int kPre = 8;                    // stages of packed words prefetched in registers
constexpr uint32_t kSpinLimit = 1u << 24;  // bounded mbarrier waits

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, 8-row
// groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);  // start address (16-byte units)
  d |= static_cast<uint64_t>(1) << 16;                 // leading-dimension offset (unused for this layout)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;         // stride between 8-row groups
  d |= static_cast<uint64_t>(1) << 46;                 // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                 // 128-byte swizzle
  return d;
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait; false when it ran out (counted, abort raised) or when another
// thread of the CTA raised the abort flag.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  for (uint32_t it = 0; it < kSpinLimit; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 255u) == 255u && *abort_flag) return false;
  }
  *abort_flag = 1;
  atomicAdd(&g_bnn_device_errors, 1u);
  return false;
}

// Bounded wait that ignores the abort flag (used for the final drain).
__device__ __forceinline__ bool mbar_drain(uint32_t bar, uint32_t parity) {
  for (uint32_t it = 0; it < kSpinLimit; ++it)
    if (mbar_try(bar, parity)) return true;
  atomicAdd(&g_bnn_device_errors, 1u);
  return false;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}

// 32 columns of this warp's 32 tensor-memory lanes
__device__ __forceinline__ void tmem_ld32(uint32_t addr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(addr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}

// operand stages per CTA: 4 x 24 KB for BN = 64 (two CTAs per SM), 4 x 48 KB for BN = 256
template <int BN>
__host__ __device__ constexpr int stages_for() {
  return 4;
}
template <int BN>
__host__ __device__ constexpr int stage_smem() {
  return stages_for<BN>() * (kTm + BN) * 128;
}
template <int BN>
__host__ __device__ constexpr int threads_for() {
  return 2 * (kTm + BN) + 32;
}

// grid: x = KS * (weight tiles of 128 rows), y = activation tiles of BN rows;
// clusters of KS CTAs along x
template <int BN, int KS>
__global__ void __launch_bounds__(threads_for<BN>(), BN <= 64 ? 2 : 1)
binary_gemm_tc_kernel(const uint64_t* __restrict__ xp, const uint64_t* __restrict__ wp,
                      const float* __restrict__ alpha, int64_t m, int64_t n, int k, int kw,
                      int32_t* __restrict__ dots, float* __restrict__ out) {
  constexpr int S = stages_for<BN>();
  constexpr int kRows = kTm + BN;
  constexpr int kProducers = 2 * kRows;
  constexpr uint32_t kStageBytes = static_cast<uint32_t>(kRows) * 128u;
  static_assert(S >= 2, "at least two operand stages");
  static_assert(KS == 1 || BN * kTm * 4 <= stage_smem<BN>(), "split-K shares must fit the stage memory");
  static_assert(BN % KS == 0, "activation columns split evenly across the cluster");

  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[S];
  __shared__ __align__(8) uint64_t empty_bar[S];
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ uint32_t tmem_holder;
  __shared__ volatile int abort_flag;
  __shared__ int any_bad;    // split K: some CTA of the cluster aborted
  __shared__ int pop_w[kTm];  // popcount of each weight row over this CTA's stages
  __shared__ int pop_x[BN];   // popcount of each activation row over this CTA's stages
  // the 128-byte swizzle repeats every 1024 bytes of address: align the tiles to it
  uint8_t* const smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int rank = KS > 1 ? static_cast<int>(blockIdx.x % KS) : 0;
  const int64_t j0 = static_cast<int64_t>(blockIdx.x / KS) * kTm;  // first weight row
  const int64_t i0 = static_cast<int64_t>(blockIdx.y) * BN;        // first activation row
  const int ktiles = (kw + 1) / 2;                                 // 2 words (128 bits) per stage
  const int share = (ktiles + KS - 1) / KS;
  const int kb = rank * share < ktiles ? rank * share : ktiles;
  const int ke = kb + share < ktiles ? kb + share : ktiles;
  const int nst = ke - kb;
  const uint32_t smem_base = smem_u32(smem);

  for (int i = tid; i < kRows; i += blockDim.x) (i < kTm ? pop_w[i] : pop_x[i - kTm]) = 0;
  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(&full_bar[i])), "r"(kProducers));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_u32(&empty_bar[i])));
    }
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_u32(&done_bar)));
    abort_flag = 0;
    any_bad = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == kProducers / 32) {  // the MMA warp owns the tensor memory
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(&tmem_holder)),
                 "r"(BN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const uint32_t tmem = tmem_holder;

  if (tid < kProducers) {
    // ------------------------------------------------------------ producers
    const int r2 = tid >> 1, part = tid & 1;  // stacked row, word of the stage
    const bool is_w = r2 < kTm;
    const int row = is_w ? r2 : r2 - kTm;
    const int64_t grow = is_w ? j0 + row : i0 + row;
    const bool live = grow < (is_w ? n : m);
    const uint64_t* src = (is_w ? wp : xp) + (live ? grow : 0) * static_cast<int64_t>(kw) + part;
    const uint32_t row_off = static_cast<uint32_t>(r2) * 128u;  // weight rows first, then activation rows
    const uint32_t swz = static_cast<uint32_t>(row & 7);

    auto fetch = [&](int jj) -> uint64_t {
      const int w = 2 * (kb + jj) + part;
      return (live && jj < nst && w < kw) ? __ldg(src + 2 * (kb + jj)) : 0ull;
    };
    uint64_t ring[kPre];
#pragma unroll
    for (int u = 0; u < kPre; ++u) ring[u] = fetch(u);

    int my_pop = 0;
    bool ok = true;
    for (int js = 0; js < nst && ok; js += kPre) {
#pragma unroll
      for (int u = 0; u < kPre; ++u) {
        const int j = js + u;
        if (j >= nst) break;
        const int b = j % S;
        // refill only after the tensor core has read the previous fill of this buffer
        if (j >= S && !mbar_wait(smem_u32(&empty_bar[b]), static_cast<uint32_t>((j / S + 1) & 1), &abort_flag)) {
          ok = false;
          break;
        }
        const uint64_t cw = ring[u];
        ring[u] = fetch(j + kPre);
        my_pop += __popcll(cw);
        uint8_t* dst = smem + b * kStageBytes + row_off;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int h = 2 * part + hh;  // half-word of the stage's 128 bits
          const uint32_t hw = static_cast<uint32_t>(cw >> (32 * hh));
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint4 v;
            v.x = (hw >> (4 * q + 0)) & 0x01010101u;
            v.y = (hw >> (4 * q + 1)) & 0x01010101u;
            v.z = (hw >> (4 * q + 2)) & 0x01010101u;
            v.w = (hw >> (4 * q + 3)) & 0x01010101u;
            const uint32_t chunk = static_cast<uint32_t>(2 * h + q);
            *reinterpret_cast<uint4*>(dst + ((chunk ^ swz) << 4)) = v;
          }
        }
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        mbar_arrive(smem_u32(&full_bar[b]));
      }
    }
    atomicAdd(is_w ? &pop_w[row] : &pop_x[row], my_pop);
  } else if (tid == kProducers) {
    // ------------------------------------------------------------ MMA issue
    // instruction descriptor: D s32, A and B 8-bit integers (0/1 bytes read
    // the same signed or unsigned), both K-major, N = BN, M = 128
    const uint32_t idesc = (2u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(BN) >> 3) << 17) |
                           ((static_cast<uint32_t>(kTm) >> 4) << 24);
    for (int j = 0; j < nst; ++j) {
      const int b = j % S;
      if (!mbar_wait(smem_u32(&full_bar[b]), static_cast<uint32_t>((j / S) & 1), &abort_flag)) break;
      asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
      const uint64_t ad = sw128_desc(smem_base + b * kStageBytes);
      const uint64_t bd = sw128_desc(smem_base + b * kStageBytes + kTm * 128u);  // activation rows
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
        asm volatile(
            "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
            "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
            "l"(ad + static_cast<uint64_t>(2 * kk)), "l"(bd + static_cast<uint64_t>(2 * kk)), "r"(idesc), "r"(acc));
      }
      asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                       smem_u32(&empty_bar[b]))
                   : "memory");
    }
    // arrives once every MMA issued above has completed
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                     smem_u32(&done_bar))
                 : "memory");
  }
  __syncwarp();

  // -------------------------------------------------------------- epilogue
  // every producer is past its loop (row popcounts added); the accumulator is final
  // once done_bar completes
  if (tid < kProducers) asm volatile("bar.sync 1, %0;\n" ::"r"(kProducers) : "memory");
  bool drained = true;
  if (warp < 8) {
    drained = mbar_drain(smem_u32(&done_bar), 0u);
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  }
  const bool good = __syncthreads_and(drained && abort_flag == 0) != 0;

  // epilogue warps 0-7: warp w reads tensor-memory lanes 32(w%4).. (weight rows)
  // and half w/4 of the BN accumulator columns (activation rows)
  const int erow = 32 * (warp & 3) + (tid & 31);
  const int ecol0 = (warp >> 2) * (BN / 2);
  const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
  if constexpr (KS == 1) {
    if (warp < 8 && good) {
      const int64_t jrow = j0 + erow;
      const bool jlive = jrow < n;
      const float a_j = (out && jlive) ? __ldg(alpha + jrow) : 0.0f;
      const int base = k - 2 * pop_w[erow];
      for (int c0 = ecol0; c0 < ecol0 + BN / 2; c0 += 32) {
        uint32_t r[32];
        if (nst > 0) {
          tmem_ld32(taddr + static_cast<uint32_t>(c0), r);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) r[c] = 0u;
        }
        const int64_t rows_left = m - (i0 + c0);
        if (jlive && rows_left > 0) {
          const int nc = rows_left < 32 ? static_cast<int>(rows_left) : 32;
          const int64_t off = (i0 + c0) * n + jrow;
          int32_t* dp = dots ? dots + off : nullptr;
          float* op = out ? out + off : nullptr;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            if (c < nc) {
              const int32_t d = base - 2 * pop_x[c0 + c] + 4 * static_cast<int32_t>(r[c]);
              if (dp) *dp = d;
              if (op) *op = a_j * static_cast<float>(d);
            }
            dp += n;
            op += n;
          }
        }
      }
    }
  } else {
    // Split K: CTA q of the cluster owns accumulator columns [q kCols, (q+1) kCols).
    // Every CTA pushes its share of each column to the owner's receive buffer
    // [source rank][column][weight row] (remote stores, no round trip), then
    // each owner adds the KS shares of its columns.
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    constexpr int kCols = BN / KS;
    int* recv = reinterpret_cast<int*>(smem);
    cluster.sync();  // every CTA's tensor core is done with its stage memory
    if (tid == 0 && !good)  // this CTA's shares will be missing: no CTA of the cluster writes
      for (int q = 0; q < KS; ++q) atomicExch(cluster.map_shared_rank(&any_bad, q), 1);
    if (warp < 8 && good) {
      const int base = -2 * pop_w[erow];
      for (int c0 = ecol0; c0 < ecol0 + BN / 2; c0 += 32) {
        uint32_t r[32];
        if (nst > 0) {
          tmem_ld32(taddr + static_cast<uint32_t>(c0), r);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) r[c] = 0u;
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int col = c0 + c;
          int* dst = cluster.map_shared_rank(recv, col / kCols);
          dst[(rank * kCols + col % kCols) * kTm + erow] = base - 2 * pop_x[col] + 4 * static_cast<int32_t>(r[c]);
        }
      }
    }
    cluster.sync();  // every share has landed
    if (any_bad == 0) {
      for (int e = tid; e < kCols * kTm; e += blockDim.x) {
        const int cl = e / kTm, row = e % kTm;
        const int64_t gi = i0 + rank * kCols + cl, jrow = j0 + row;
        if (gi < m && jrow < n) {
          int32_t d = k;
#pragma unroll
          for (int q = 0; q < KS; ++q) d += recv[(q * kCols + cl) * kTm + row];
          if (dots) dots[gi * n + jrow] = d;
          if (out) out[gi * n + jrow] = __ldg(alpha + jrow) * static_cast<float>(d);
        }
      }
    }
  }

  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  if (warp == kProducers / 32)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(BN));
}

template <int BN, int KS>
bnn_status launch_tc(const uint64_t* xp, const uint64_t* wp, const float* alpha, int64_t m, int64_t n, int k, int kw,
                     int32_t* dots, float* out, cudaStream_t s) {
  const int64_t gx = KS * ((n + kTm - 1) / kTm), gy = (m + BN - 1) / BN;
  if (gx > 2147483647LL || gy > 65535) return BNN_ERR_INVALID_ARG;
  const size_t smem = static_cast<size_t>(stage_smem<BN>()) + 1024;  // + 1024-byte alignment slack
  auto kern = binary_gemm_tc_kernel<BN, KS>;
  BNN_TRY(bnn::ensure_smem(kern, smem));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  cfg.blockDim = dim3(threads_for<BN>());
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = KS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = KS > 1 ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, xp, wp, alpha, m, n, k, kw, dots, out);
  if (e != cudaSuccess) return bnn::cuda_fail(e);
  return bnn::check_launch();
}

}  // namespace

namespace bnn {

// Tensor-core (tcgen05) binary GEMM.  m > 128 takes 256-row activation tiles
// (one CTA per SM; the widest MMA, fewest re-expansions of the operands);
// smaller m takes 64-row tiles (two CTAs per SM).  When the tiles alone would
// leave SMs idle, a cluster of 2 or 4 CTAs splits each tile's stages (at least
// 4 stages per CTA).
bnn_status binary_gemm_tc(const uint64_t* xp, const uint64_t* wp, const float* alpha, int64_t m, int64_t n, int k,
                          int kw, int32_t* dots, float* out, cudaStream_t s) {
  const int64_t wt = (n + kTm - 1) / kTm;
  const int64_t sms = sm_count();
  const int ktiles = (kw + 1) / 2;
  auto pick_ks = [&](int64_t tiles, int64_t capacity) {
    if (tiles * 4 <= capacity && ktiles >= 16) return 4;
    if (tiles * 2 <= capacity && ktiles >= 8) return 2;
    return 1;
  };
  if (m > 128) {
    switch (pick_ks(wt * ((m + 255) / 256), sms)) {
      case 4: return launch_tc<256, 4>(xp, wp, alpha, m, n, k, kw, dots, out, s);
      case 2: return launch_tc<256, 2>(xp, wp, alpha, m, n, k, kw, dots, out, s);
      default: return launch_tc<256, 1>(xp, wp, alpha, m, n, k, kw, dots, out, s);
    }
  }
  switch (pick_ks(wt * ((m + 63) / 64), 2 * sms)) {
    case 4: return launch_tc<64, 4>(xp, wp, alpha, m, n, k, kw, dots, out, s);
    case 2: return launch_tc<64, 2>(xp, wp, alpha, m, n, k, kw, dots, out, s);
    default: return launch_tc<64, 1>(xp, wp, alpha, m, n, k, kw, dots, out, s);
  }
}

}  // namespace bnn

extern "C" int bnn_device_error_count(int reset) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_bnn_device_errors, sizeof(v)) != cudaSuccess) return -1;
  if (reset) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_bnn_device_errors, &zero, sizeof(zero)) != cudaSuccess) return -1;
  }
  const int t = bnn::ternary_tc_error_count(reset);
  if (t < 0) return -1;
  return static_cast<int>(v) + t;
}
