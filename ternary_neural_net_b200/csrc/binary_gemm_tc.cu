// bnn_binary_gemm on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "Binary Math Effectiveness -- why / how / when", section 1: for +-1 vectors
// packed with bit 1 = -1, <x,w> = n - 2 popcount(x XOR w).  Writing a and b
// for the bits of x and w, popcount(x XOR w) = pa + pb - 2 popcount(a AND b),
// so <x,w> = k - 2 pa - 2 pb + 4 popcount(a AND b), where pa and pb are the
// row popcounts.  popcount(a AND b) is the dot product of the rows' bits as
// 0/1 values.  Here each bit becomes an e2m1 float, 1.0 (code 0b0010) or 0.0,
// and the tensor cores run tcgen05.mma.kind::mxf4.block_scale.block32 with
// every ue8m0 scale factor 127 (2^0): the products are exactly 0 or 1 and the
// float32 accumulator holds the count exactly (every integer up to 2^24 is a
// float32, and the ABI bounds k by 2^24).  Pad bits are 0 in both rows and so
// add nothing to any of the three counts.
//
// One-SM kernel.  Tile: UMMA M = 128 weight rows (operand A) x N = BN
// activation rows (operand B), K in stages of 256 bits (4 words, 128 bytes of
// nibbles per row).  Tensor memory holds the accumulator (BN columns) and the
// scale factors (the next BN columns, 127 in every byte).  Roles inside a CTA:
//   - a TMA thread (when every row is 16-byte aligned): copies the packed words
//     of 2 stages of all the tile's rows (a 64-byte-swizzled box of each
//     operand) into a double-buffered chunk ring, signalling an mbarrier with
//     the byte count;
//   - producer threads, two per row of the stacked (weight, activation) tile,
//     each owning two 64-bit words of the row per stage: read them (from the
//     chunk ring, or without TMA straight from global memory, prefetched kPre
//     stages ahead in registers), count their bits, and write their 64 bytes
//     of nibbles (per 4 bytes a shift and an AND) in the 128-byte-swizzled
//     K-major layout the tensor core reads, then arrive on the stage's "full"
//     mbarrier;
//   - one MMA thread: waits for "full", issues 4 MMAs (K = 64) into the float32
//     accumulator in tensor memory and commits to the stage's "empty"
//     mbarrier, which the producers wait on before refilling it;
//   - the epilogue (warps 0-7; warp w reads tensor-memory lanes 32(w%4).. and
//     half w/4 of the columns): tcgen05.ld, the count as an integer, the
//     popcount correction, alpha, the optional bias, and stores in which the
//     32 lanes of a warp write 32 consecutive weight columns of one output
//     row.  Those 32 columns are also one 32-bit half of a word of the next
//     layer's packed input, so the optional sign pack of the layer output is
//     one __ballot_sync per row.
// Any bijection between the 256 bits and the 256 k-slots of a stage gives the
// same sum when both operands use it; here nibble j of word s of the 16-byte
// unit built from 32-bit half h holds bit 32h + 4j + s.
//
// Split K: a cluster of KS CTAs shares one output tile, each taking a
// contiguous share of the stages.  Each CTA turns its accumulator into its
// share of the dot (-2 pa - 2 pb + 4 S over its stages) and stores it, four
// columns per 16-byte store, straight into the shared memory of the CTA that
// owns those output rows (distributed shared memory); CTA r adds the KS shares
// of its BN/KS output rows and writes them.  Integer addition makes the
// result independent of the order.
//
// Every wait on an mbarrier is bounded.  A wait that runs out bumps a
// device-side error count (bnn_device_error_count) and raises a CTA-wide abort
// flag that ends the other waits; the CTA then skips its stores, waits
// (bounded) for the MMAs it issued, frees its tensor memory and returns.
#include <cooperative_groups.h>

#include <atomic>
#include <mutex>

#include "bnn_internal.cuh"
#include "bnn_probe.h"
#include "tc_common.cuh"

// Bounded waits that ran out in this file's kernels (read by bnn_device_error_count).
__device__ unsigned int g_bnn_device_errors = 0;

// Polls of the main mbarrier waits of the kernels below (the final drains keep
// the full bound): 0 = the normal time bound; a small value is set only by the
// diagnostic bnn_probe_wait_limit, so that a test can make the waits run out.
static std::atomic<uint32_t> g_wait_limit{0};

namespace {

using bnn::tc::mbar_arrive;
using bnn::tc::mbar_expect_tx;
using bnn::tc::mbar_try;
using bnn::tc::smem_u32;
using bnn::tc::sw128_desc;
using bnn::tc::tma_load_2d;
using bnn::tc::tmem_ld16;
using bnn::tc::tmem_ld32;
using bnn::tc::tmem_wait_ld;

constexpr int kTm = 128;                   // weight rows per tile (UMMA M)
constexpr int kPre = 4;                    // without TMA: stages of words prefetched in registers
constexpr int kChunkStages = 4;            // CTA pairs: stages per packed chunk (128 bytes of every row)
constexpr int kTcWords = 4;                // one-SM kernel: packed words per row and stage (256 bits of k)
constexpr int kTcChunkStages = 2;          // one-SM kernel with TMA: stages per packed chunk (64 bytes of every row)
static_assert(BNN_MAX_K_BINARY <= (1 << 24), "AND counts accumulated in float32 stay exact integers");

// WIDE (64- and 128-row tiles): one CTA per SM with a deeper ring of expanded
// stages; otherwise 64-row tiles keep 96 KB so that two CTAs share an SM.
template <int BN, bool TMA, bool WIDE>
struct TcCfg {
  static_assert(!WIDE || BN <= 128, "deep rings for the 64- and 128-row tiles");
  static constexpr int kRows = kTm + BN;                             // stacked weight + activation rows
  static constexpr uint32_t kStageBytes = kRows * 128u;              // one expanded stage
  static constexpr uint32_t kChunkBytes = kRows * 8u * kTcWords * kTcChunkStages;  // one packed chunk (64 B a row)
  static constexpr int S = !WIDE ? (TMA ? 3 : 4)                     // expanded stages
                                 : (BN == 64 ? (TMA ? 6 : 8) : (TMA ? 5 : 6));
  static constexpr int P = TMA ? 2 : 0;                              // packed chunks
  static constexpr uint32_t kSmem = S * kStageBytes + P * kChunkBytes;
  static constexpr int kProducers = 2 * kRows;
  static constexpr int kThreads = kProducers + 64;                   // + MMA warp + TMA warp
  static constexpr int kMinBlocks = (BN <= 64 && !WIDE) ? 2 : 1;
};

// 32 bits of a packed row as one 16-byte unit of e2m1 nibbles (0 or 2 = 1.0):
// word s of the unit holds bits s, s + 4, ..., s + 28 of hw (nibble j = bit
// 4j + s), the same permutation of k in both operands
__device__ __forceinline__ uint4 nibbles_of(uint32_t hw) {
  uint4 v;
  v.x = (hw << 1) & 0x22222222u;
  v.y = hw & 0x22222222u;
  v.z = (hw >> 1) & 0x22222222u;
  v.w = (hw >> 2) & 0x22222222u;
  return v;
}

// one-SM kernel: a thread's two words of a stage (v: four 32-bit halves) ->
// units 4 part .. 4 part + 3 of its row of the expanded stage (128-byte swizzle)
__device__ __forceinline__ void expand_pair(uint8_t* dst_row, uint32_t swz, int part, const uint4& v) {
  const uint32_t h[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(dst_row + ((static_cast<uint32_t>(4 * part + q) ^ swz) << 4)) = nibbles_of(h[q]);
}

// grid: x = KS * (weight tiles of 128 rows), y = activation tiles of BN rows;
// clusters of KS CTAs along x
template <int BN, int KS, bool TMA, bool WIDE>
__global__ void __launch_bounds__(TcCfg<BN, TMA, WIDE>::kThreads, TcCfg<BN, TMA, WIDE>::kMinBlocks)
binary_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                      const uint64_t* __restrict__ xp, const uint64_t* __restrict__ wp,
                      const float* __restrict__ alpha, const float* __restrict__ bias, int64_t m, int64_t n,
                      int k, int kw, int32_t* __restrict__ dots, float* __restrict__ out,
                      uint32_t* __restrict__ next, int64_t next_w32, uint32_t wait_limit) {
  using Cfg = TcCfg<BN, TMA, WIDE>;
  constexpr int S = Cfg::S;
  constexpr int P = TMA ? Cfg::P : 1;
  constexpr int kRows = Cfg::kRows;
  constexpr int kProducers = Cfg::kProducers;
  constexpr uint32_t kStageBytes = Cfg::kStageBytes;
  constexpr int kCols = BN / KS;          // split K: accumulator columns each CTA owns
  constexpr int kPitch = kCols + 4;       // split K: padded receive row (ints)
  static_assert(S >= 2, "at least two operand stages");
  static_assert(BN % KS == 0 && kCols % 4 == 0, "activation columns split evenly, four at a time");
  static_assert(KS == 1 || KS * kTm * kPitch * 4 <= Cfg::kSmem, "split-K shares must fit the stage memory");

  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[S];
  __shared__ __align__(8) uint64_t empty_bar[S];
  __shared__ __align__(8) uint64_t chunk_full[P];
  __shared__ __align__(8) uint64_t chunk_empty[P];
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ uint32_t tmem_holder;
  __shared__ volatile int abort_flag;
  __shared__ int any_bad;      // split K: some CTA of the cluster aborted
  __shared__ int pop_w[kTm];   // popcount of each weight row over this CTA's stages
  __shared__ int pop_x[BN];    // popcount of each activation row over this CTA's stages
  // the 128-byte swizzle repeats every 1024 bytes of address: align the tiles to it
  uint8_t* const smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* const chunks = smem + S * kStageBytes;  // TMA: packed chunk ring

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int rank = KS > 1 ? static_cast<int>(blockIdx.x % KS) : 0;
  const int64_t j0 = static_cast<int64_t>(blockIdx.x / KS) * kTm;  // first weight row
  const int64_t i0 = static_cast<int64_t>(blockIdx.y) * BN;        // first activation row
  const int ktiles = (kw + kTcWords - 1) / kTcWords;               // 4 words (256 bits) per stage
  const int share = (ktiles + KS - 1) / KS;
  const int kb = rank * share < ktiles ? rank * share : ktiles;
  const int ke = kb + share < ktiles ? kb + share : ktiles;
  const int nst = ke - kb;
  const uint32_t smem_base = smem_u32(smem);
  constexpr int kMmaWarp = kProducers / 32, kTmaWarp = kMmaWarp + 1;

  for (int i = tid; i < kRows; i += blockDim.x) (i < kTm ? pop_w[i] : pop_x[i - kTm]) = 0;
  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(&full_bar[i])), "r"(kProducers));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_u32(&empty_bar[i])));
    }
    for (int i = 0; i < P; ++i) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_u32(&chunk_full[i])));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(&chunk_empty[i])), "r"(kProducers));
    }
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_u32(&done_bar)));
    abort_flag = 0;
    any_bad = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (TMA && tid == kTmaWarp * 32) {  // bring both descriptors on chip while the CTA sets up
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
  }
  if (warp == kMmaWarp) {  // the MMA warp owns the tensor memory
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(&tmem_holder)),
                 "r"(2 * BN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  // accumulator: columns [0, BN); the MMA's scale factors: 127 (2^0) in every
  // byte of columns [BN, 2 BN), written by warps 0-3 before the first MMA
  const uint32_t tmem = tmem_holder;
  if (warp < 4) {
    const uint32_t lanes = static_cast<uint32_t>(32 * warp) << 16;
    for (uint32_t c = BN; c < 2u * BN; c += 8)
      asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1};\n" ::"r"(tmem + lanes + c),
                   "r"(0x7F7F7F7Fu)
                   : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  bnn::pdl_trigger();

  if (tid < kProducers) {
    // ------------------------------------------------------------ producers
    const int r2 = tid >> 1, part = tid & 1;  // stacked row, word of the stage
    const bool is_w = r2 < kTm;
    const int row = is_w ? r2 : r2 - kTm;
    const uint32_t row_off = static_cast<uint32_t>(r2) * 128u;  // weight rows first, then activation rows
    const uint32_t swz = static_cast<uint32_t>(row & 7);
    int my_pop = 0;
    bool ok = true;
    if constexpr (TMA) {
      // this thread's two words of stage s of a chunk: row r2 (64 bytes), 16-byte
      // unit 2 s + part under the 64-byte swizzle (unit ^ bits 7-8 of the address)
      const uint32_t rd_off = static_cast<uint32_t>(r2) * 64u;
      const uint32_t rd_swz = static_cast<uint32_t>((r2 >> 1) & 3);
      for (int j = 0; j < nst; ++j) {
        const int c = j / kTcChunkStages, s = j % kTcChunkStages, pb = c % P;
        if (s == 0 && !bnn::tc::mbar_wait(smem_u32(&chunk_full[pb]), static_cast<uint32_t>((c / P) & 1), &abort_flag,
                                          &g_bnn_device_errors, wait_limit)) {
          ok = false;
          break;
        }
        const uint4 cw = *reinterpret_cast<const uint4*>(
            chunks + pb * Cfg::kChunkBytes + rd_off + ((static_cast<uint32_t>(2 * s + part) ^ rd_swz) << 4));
        if (s == kTcChunkStages - 1 || j == nst - 1) mbar_arrive(smem_u32(&chunk_empty[pb]));
        const int b = j % S;
        // refill only after the tensor core has read the previous fill of this buffer
        if (j >= S && !bnn::tc::mbar_wait(smem_u32(&empty_bar[b]), static_cast<uint32_t>((j / S + 1) & 1), &abort_flag,
                                          &g_bnn_device_errors, wait_limit)) {
          ok = false;
          break;
        }
        my_pop += __popc(cw.x) + __popc(cw.y) + __popc(cw.z) + __popc(cw.w);
        expand_pair(smem + b * kStageBytes + row_off, swz, part, cw);
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        mbar_arrive(smem_u32(&full_bar[b]));
      }
    } else {
      const int64_t grow = is_w ? j0 + row : i0 + row;
      const bool live = grow < (is_w ? n : m);
      const uint64_t* src = (is_w ? wp : xp) + (live ? grow : 0) * static_cast<int64_t>(kw) + 2 * part;
      if (!is_w) bnn::pdl_wait();  // the activations may come from the preceding kernel
      // this thread's two words of stage jj (words 4 (kb + jj) + 2 part and the next; 0 past the row)
      auto fetch = [&](int jj) -> uint4 {
        const int w = kTcWords * (kb + jj) + 2 * part;
        const bool in = live && jj < nst;
        const uint64_t a = (in && w < kw) ? __ldg(src + kTcWords * (kb + jj)) : 0ull;
        const uint64_t b2 = (in && w + 1 < kw) ? __ldg(src + kTcWords * (kb + jj) + 1) : 0ull;
        return make_uint4(static_cast<uint32_t>(a), static_cast<uint32_t>(a >> 32), static_cast<uint32_t>(b2),
                          static_cast<uint32_t>(b2 >> 32));
      };
      uint4 ring[kPre];
#pragma unroll
      for (int u = 0; u < kPre; ++u) ring[u] = fetch(u);
      for (int js = 0; js < nst && ok; js += kPre) {
#pragma unroll
        for (int u = 0; u < kPre; ++u) {
          const int j = js + u;
          if (j >= nst) break;
          const int b = j % S;
          if (j >= S && !bnn::tc::mbar_wait(smem_u32(&empty_bar[b]), static_cast<uint32_t>((j / S + 1) & 1), &abort_flag,
                                          &g_bnn_device_errors, wait_limit)) {
            ok = false;
            break;
          }
          const uint4 cw = ring[u];
          ring[u] = fetch(j + kPre);
          my_pop += __popc(cw.x) + __popc(cw.y) + __popc(cw.z) + __popc(cw.w);
          expand_pair(smem + b * kStageBytes + row_off, swz, part, cw);
          asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
          mbar_arrive(smem_u32(&full_bar[b]));
        }
      }
    }
    atomicAdd(is_w ? &pop_w[row] : &pop_x[row], my_pop);
  } else if (tid == kMmaWarp * 32) {
    // ------------------------------------------------------------ MMA issue
    // instruction descriptor: D f32; A and B e2m1 (format 1), K-major; ue8m0
    // scale factors (bit 23, every one 127 = 2^0); N = BN, M = 128; dense K = 64
    const uint32_t idesc = (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(BN) >> 3) << 17) | (1u << 23) |
                           ((static_cast<uint32_t>(kTm) >> 4) << 24);
    const uint32_t sfa = tmem + static_cast<uint32_t>(BN), sfb = tmem + static_cast<uint32_t>(BN + BN / 2);
    for (int j = 0; j < nst; ++j) {
      const int b = j % S;
      if (!bnn::tc::mbar_wait(smem_u32(&full_bar[b]), static_cast<uint32_t>((j / S) & 1), &abort_flag,
                              &g_bnn_device_errors, wait_limit))
        break;
      asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
      const uint64_t ad = sw128_desc(smem_base + b * kStageBytes);
      const uint64_t bd = sw128_desc(smem_base + b * kStageBytes + kTm * 128u);  // activation rows
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
        asm volatile(
            "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
            "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(
                tmem),
            "l"(ad + static_cast<uint64_t>(2 * kk)), "l"(bd + static_cast<uint64_t>(2 * kk)), "r"(idesc), "r"(acc),
            "r"(sfa), "r"(sfb));
      }
      asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                       smem_u32(&empty_bar[b]))
                   : "memory");
    }
    // arrives once every MMA issued above has completed
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                     smem_u32(&done_bar))
                 : "memory");
  } else if (TMA && tid == kTmaWarp * 32) {
    // ------------------------------------------------------------ TMA copies
    const int nch = (nst + kTcChunkStages - 1) / kTcChunkStages;
    const int pre = nch < P ? nch : P;
    // first word of chunk c (even: 16-byte aligned)
    auto chunk_x = [&](int c) { return kTcWords * kb + kTcWords * kTcChunkStages * c; };
    // the weights do not depend on the preceding kernel: their first chunks
    // are copied before waiting for it, the activations after
    for (int c = 0; c < pre; ++c) {
      mbar_expect_tx(smem_u32(&chunk_full[c]), Cfg::kChunkBytes);
      tma_load_2d(smem_u32(chunks + c * Cfg::kChunkBytes), &tmap_w, chunk_x(c), static_cast<int>(j0),
                  smem_u32(&chunk_full[c]));
    }
    bnn::pdl_wait();
    for (int c = 0; c < pre; ++c)
      tma_load_2d(smem_u32(chunks + c * Cfg::kChunkBytes) + kTm * 64u, &tmap_x, chunk_x(c),
                  static_cast<int>(i0), smem_u32(&chunk_full[c]));
    int issued = pre;
    for (int c = pre; c < nch; ++c) {
      const int pb = c % P;
      if (!bnn::tc::mbar_wait(smem_u32(&chunk_empty[pb]), static_cast<uint32_t>((c / P + 1) & 1), &abort_flag,
                              &g_bnn_device_errors, wait_limit))
        break;
      const uint32_t dst = smem_u32(chunks + pb * Cfg::kChunkBytes);
      const uint32_t bar = smem_u32(&chunk_full[pb]);
      mbar_expect_tx(bar, Cfg::kChunkBytes);
      tma_load_2d(dst, &tmap_w, chunk_x(c), static_cast<int>(j0), bar);
      tma_load_2d(dst + kTm * 64u, &tmap_x, chunk_x(c), static_cast<int>(i0), bar);
      issued = c + 1;
    }
    // the CTA must not retire with copies in flight (producers that aborted no
    // longer wait for them): wait for the last chunk issued into each buffer
    for (int c = issued - P; c < issued; ++c)
      if (c >= 0) bnn::tc::mbar_drain(smem_u32(&chunk_full[c % P]), static_cast<uint32_t>((c / P) & 1), &g_bnn_device_errors);
  }
  __syncwarp();

  // -------------------------------------------------------------- epilogue
  // every producer is past its loop (row popcounts added); the accumulator is
  // final once done_bar completes
  if (tid < kProducers) asm volatile("bar.sync 1, %0;\n" ::"r"(kProducers) : "memory");
  bool drained = true;
  if (warp < 8) {
    drained = bnn::tc::mbar_drain(smem_u32(&done_bar), 0u, &g_bnn_device_errors);
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  }
  const bool good = __syncthreads_and(drained && abort_flag == 0) != 0;

  // epilogue warps 0-7: warp w reads tensor-memory lanes 32(w%4).. (weight rows)
  // and half w/4 of the BN accumulator columns (activation rows)
  const int erow = 32 * (warp & 3) + (tid & 31);
  const int ecol0 = (warp >> 2) * (BN / 2);
  const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
  // the tile's accumulated popc(a AND b) for 16 columns from c0 (the float32
  // counts, exact integers, converted)
  auto load16 = [&](int c0, uint32_t (&r)[16]) {
    if (nst > 0) {
      tmem_ld16(taddr + static_cast<uint32_t>(c0), r);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 16; ++c) r[c] = static_cast<uint32_t>(static_cast<int32_t>(__uint_as_float(r[c])));
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c) r[c] = 0u;
    }
  };
  // y = fl32(alpha * dot), then fl32(y + bias) when there is a bias (two
  // roundings: no fused multiply-add); the next layer's input bit is !(y > 0)
  auto layer_y = [&](float a, float b, int32_t d) {
    const float y = __fmul_rn(a, static_cast<float>(d));
    return bias ? __fadd_rn(y, b) : y;
  };
  const bool need_y = out || next;
  if constexpr (KS == 1) {
    if (warp < 8 && good) {
      const int64_t jrow = j0 + erow;
      const bool jlive = jrow < n;
      const float a_j = (need_y && jlive) ? __ldg(alpha + jrow) : 0.0f;
      const float b_j = (bias && jlive) ? __ldg(bias + jrow) : 0.0f;
      const int base = k - 2 * pop_w[erow];
      // this warp's 32 weight rows form one 32-bit half of a packed word of `next`
      const int64_t half = (j0 + 32 * (warp & 3)) / 32;
      const bool pack = next && half < next_w32;  // uniform across the warp
      for (int c0 = ecol0; c0 < ecol0 + BN / 2; c0 += 16) {
        uint32_t r[16];
        load16(c0, r);
        const int64_t rows_left = m - (i0 + c0);
        const int nc = rows_left <= 0 ? 0 : (rows_left < 16 ? static_cast<int>(rows_left) : 16);
        const int64_t off = (i0 + c0) * n + jrow;
        int32_t* dp = dots ? dots + off : nullptr;
        float* op = out ? out + off : nullptr;
        uint32_t* np = pack ? next + (i0 + c0) * next_w32 + half : nullptr;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int32_t d = base - 2 * pop_x[c0 + c] + 4 * static_cast<int32_t>(r[c]);
          const float y = layer_y(a_j, b_j, d);
          if (c < nc && jlive) {
            if (dp) *dp = d;
            if (op) *op = y;
          }
          if (np) {
            const unsigned bits = __ballot_sync(0xffffffffu, jlive && !(y > 0.0f));
            if ((tid & 31) == 0 && c < nc) *np = bits;
            np += next_w32;
          }
          dp += n;
          op += n;
        }
      }
    }
  } else {
    // Split K: CTA q of the cluster owns accumulator columns [q kCols, (q+1) kCols).
    // Every CTA pushes its share of each column to the owner's receive buffer
    // [source rank][weight row][column, padded] (16-byte remote stores, no
    // round trip), then each owner adds the KS shares of its columns.
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    int* recv = reinterpret_cast<int*>(smem);
    cluster.sync();  // every CTA's tensor core is done with its stage memory
    if (tid == 0 && !good)  // this CTA's shares will be missing: no CTA of the cluster writes
      for (int q = 0; q < KS; ++q) atomicExch(cluster.map_shared_rank(&any_bad, q), 1);
    if (warp < 8 && good) {
      const int base = -2 * pop_w[erow];
      for (int c0 = ecol0; c0 < ecol0 + BN / 2; c0 += 16) {
        uint32_t r[16];
        load16(c0, r);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int col = c0 + 4 * g;
          int4 v;
          v.x = base - 2 * pop_x[col + 0] + 4 * static_cast<int32_t>(r[4 * g + 0]);
          v.y = base - 2 * pop_x[col + 1] + 4 * static_cast<int32_t>(r[4 * g + 1]);
          v.z = base - 2 * pop_x[col + 2] + 4 * static_cast<int32_t>(r[4 * g + 2]);
          v.w = base - 2 * pop_x[col + 3] + 4 * static_cast<int32_t>(r[4 * g + 3]);
          int* dst = cluster.map_shared_rank(recv, col / kCols);
          *reinterpret_cast<int4*>(dst + (rank * kTm + erow) * kPitch + col % kCols) = v;
        }
      }
    }
    cluster.sync();  // every share has landed
    if (any_bad == 0) {
      // a warp's 32 lanes take 32 consecutive weight rows (one 32-bit half of a
      // packed word of `next`) and the same four activation rows
      for (int e = tid; e < kTm * (kCols / 4); e += blockDim.x) {
        const int row = e % kTm, cl = 4 * (e / kTm);
        const int64_t jrow = j0 + row;
        const bool jlive = jrow < n;
        int4 d = make_int4(k, k, k, k);
#pragma unroll
        for (int q = 0; q < KS; ++q) {
          const int4 v = *reinterpret_cast<const int4*>(recv + (q * kTm + row) * kPitch + cl);
          d.x += v.x;
          d.y += v.y;
          d.z += v.z;
          d.w += v.w;
        }
        const float a_j = (need_y && jlive) ? __ldg(alpha + jrow) : 0.0f;
        const float b_j = (bias && jlive) ? __ldg(bias + jrow) : 0.0f;
        const int64_t half = (j0 + row - (tid & 31)) / 32;
        const bool pack = next && half < next_w32;  // uniform across the warp
        const int dv[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int64_t gi = i0 + rank * kCols + cl + t;
          const float y = layer_y(a_j, b_j, dv[t]);
          if (gi < m && jlive) {
            if (dots) dots[gi * n + jrow] = dv[t];
            if (out) out[gi * n + jrow] = y;
          }
          if (pack) {
            const unsigned bits = __ballot_sync(0xffffffffu, jlive && !(y > 0.0f));
            if ((tid & 31) == 0 && gi < m) next[gi * next_w32 + half] = bits;
          }
        }
      }
    }
  }

  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  if (warp == kMmaWarp)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(2 * BN));
}

// ---------------------------------------------------------------------------
// Two-SM persistent variant for large GEMMs, on the 4-bit float tensor cores.
//
// The AND count popc(a AND b) is a dot product of 0/1 vectors.  Here each bit
// becomes an e2m1 float, 1.0 (code 0b0010) or 0.0, and the pair runs
// tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 with every ue8m0
// scale factor 127 (2^0): the products are exactly 0 or 1 and the float32
// accumulator holds the count exactly (every integer up to 2^24 is a float32,
// and the ABI bounds k by BNN_MAX_K_BINARY = 2^24).  Per instruction K = 64
// at twice the int8 rate, and an expanded bit takes half a byte.
//
// A cluster of two CTAs computes tiles of 256 weight rows x kPN = 224
// activation rows (UMMA M = 256, N = 224): CTA q of the pair holds weight
// rows 128q.. of the tile (its half of operand A, and the tensor-memory lanes
// of those rows) and activation rows 112q.. (its half of operand B); one MMA
// reads both CTAs' shared memory.  The pairs are persistent: pair p takes
// tiles p, p + P, ... (P pairs, at most as many as fit the GPU at once).  The
// accumulator is double-buffered in tensor memory (2 x 224 columns, so the
// epilogue of one tile overlaps the mainloop of the next); columns 448..511
// hold the scale factors, written once by the epilogue warps of both CTAs
// before the first MMA (every byte 127, so their layout within those columns
// does not matter).
//
// Roles per CTA:
//   - a TMA thread copies the packed chunks (4 stages of 4 words, 128 bytes of
//     each of its own 128 weight and 112 activation rows, 128-byte swizzle)
//     into a two-chunk ring;
//   - four producer groups of 128 threads; group g takes stage g of every
//     chunk, thread t weight row t and activation row t (t < 112): each 32
//     bits of a row's four words become one 16-byte unit of nibbles (word s
//     of the unit holds bits s, s + 4, ... as 0 or 2, the same permutation of
//     k in both operands), so four stages are expanded at once and the latency
//     of one (loads, stores, proxy fence, barrier) hides behind the others.
//     After a named barrier of its 128 threads a group arrives once on the
//     stage's "full" mbarrier of CTA 0 (at cluster scope), which thus
//     completes once both CTAs' groups have written the stage;
//   - CTA 0's MMA thread waits for "full", issues 4 MMAs (K = 64) into
//     accumulator buffer t % 2, and commits with a two-CTA mask to the stage's
//     "empty" barrier in both CTAs (and to "acc_full" after a tile's last
//     stage); before a tile it waits on "acc_empty" for the epilogue that read
//     the buffer two tiles back;
//   - eight epilogue warps (two per quarter of the tensor-memory lanes, each
//     half of the columns) read the accumulator (the count, exact in float32),
//     apply the popcount correction (row popcounts from a pass before the
//     kernel), alpha and the optional bias, store, and arrive on CTA 0's
//     "acc_empty".
// The stage, chunk and accumulator rings run on across tiles.  Every wait is
// bounded; a wait that runs out stops every role of the CTA (the other CTA's
// waits then run out too) and leaves the outputs unspecified.
// ---------------------------------------------------------------------------
constexpr int kPX = 112;                                        // activation rows per CTA (N / 2)
constexpr int kPN = 2 * kPX;                                    // activation rows per tile (UMMA N)
constexpr int kQRows = kTm + kPX;                               // stacked rows per CTA (128 weight + 112 activation)
constexpr int kQWords = 4;                                      // packed words per row and stage (K = 256 bits)
constexpr uint32_t kQRowBytes = 8u * kQWords * kChunkStages;    // a packed chunk row (128 bytes)
constexpr uint32_t kQStageBytes = kQRows * 128u;                // one expanded stage (30 KiB)
constexpr uint32_t kQChunkBytes = kQRows * kQRowBytes;          // one packed chunk (30 KiB)
constexpr int kQS = 5, kQP = 2;                                 // expanded stages, packed chunks
constexpr int kQG = kChunkStages;                               // producer groups (one stage of every chunk each)
constexpr int kQGroup = kTm;                                    // threads per group
constexpr int kQProducers = kQG * kQGroup;                      // 512
constexpr int kQMmaWarp = kQProducers / 32, kQTmaWarp = kQMmaWarp + 1, kQEpiWarp0 = kQMmaWarp + 2;
constexpr int kQEpi = 8;                                        // epilogue warps (two per lane quarter)
constexpr int kQThreads = kQProducers + 64 + 32 * kQEpi;        // + MMA warp + TMA warp + epilogue warps
constexpr uint32_t kQSmem = kQS * kQStageBytes + kQP * kQChunkBytes;
constexpr uint32_t kQTmemCols = 512;                            // two 224-column accumulators + scale factors
constexpr uint32_t kQSfCol = 2 * kPN;                           // scale factors: columns [448, 512)
constexpr int kQEpiBar = 2 + kQG;                               // named barrier of the epilogue warps
static_assert(kPX % 8 == 0 && kPN % 32 == 0 && kPN % 16 == 0 && kPN <= 256, "UMMA N and the epilogue's column blocks");
static_assert(kQStageBytes % 1024 == 0 && kQChunkBytes % 1024 == 0, "128-byte swizzle atoms stay 1024-byte aligned");
static_assert(kQSfCol + 64 <= kQTmemCols, "scale-factor columns");
static_assert(kQS > kQG, "the four groups expand four stages of a chunk at once: one buffer each, and one ahead");

__global__ void __launch_bounds__(kQThreads, 1)
binary_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                        const float* __restrict__ alpha, const float* __restrict__ bias,
                        const int* __restrict__ pop_x, const int* __restrict__ pop_w, int64_t m, int64_t n, int k,
                        int kw, int32_t* __restrict__ dots, float* __restrict__ out, uint32_t* __restrict__ next,
                        int64_t next_w32, uint32_t wait_limit) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kQS];   // CTA 0's: one arrival per CTA
  __shared__ __align__(8) uint64_t empty_bar[kQS];
  __shared__ __align__(8) uint64_t chunk_full[kQP];
  __shared__ __align__(8) uint64_t chunk_empty[kQP];
  __shared__ __align__(8) uint64_t acc_full[2];
  __shared__ __align__(8) uint64_t acc_empty[2];    // CTA 0's: one arrival per CTA
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ uint32_t tmem_holder;
  __shared__ volatile int abort_flag;
  __shared__ int pop_xs[kPN];                      // the epilogue's tile: activation-row popcounts
  uint8_t* const smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* const chunks = smem + kQS * kQStageBytes;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster.block_rank();
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int64_t ntn = (n + 255) / 256, ntiles = ntn * ((m + kPN - 1) / kPN);
  const int nst = (kw + kQWords - 1) / kQWords, nch = (nst + kChunkStages - 1) / kChunkStages;
  const uint32_t smem_base = smem_u32(smem);

  if (tid == 0) {
    for (int i = 0; i < kQS; ++i) {
      bnn::tc::mbar_init(smem_u32(&full_bar[i]), 2);
      bnn::tc::mbar_init(smem_u32(&empty_bar[i]), 1);
    }
    for (int i = 0; i < kQP; ++i) {
      bnn::tc::mbar_init(smem_u32(&chunk_full[i]), 1);
      bnn::tc::mbar_init(smem_u32(&chunk_empty[i]), kQG);
    }
    for (int i = 0; i < 2; ++i) {
      bnn::tc::mbar_init(smem_u32(&acc_full[i]), 1);
      bnn::tc::mbar_init(smem_u32(&acc_empty[i]), 2);
    }
    bnn::tc::mbar_init(smem_u32(&done_bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (tid == kQTmaWarp * 32) {
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
  }
  if (warp == kQMmaWarp) {  // the same warp of both CTAs allocates the pair's tensor memory
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(&tmem_holder)),
                 "r"(kQTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;\n" ::);
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const uint32_t tmem = tmem_holder;
  if (warp >= kQEpiWarp0 && warp < kQEpiWarp0 + 4) {  // scale factors: 127 in every byte of columns [448, 512)
    const uint32_t lanes = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    for (uint32_t c = kQSfCol; c < kQTmemCols; c += 8)
      asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1};\n" ::"r"(tmem + lanes + c),
                   "r"(0x7F7F7F7Fu)
                   : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  cluster.sync();  // both CTAs' barriers and scale factors exist before any arrival or MMA
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  bnn::pdl_trigger();

  if (tid < kQProducers) {
    // ------------------------------------------------------------ producers
    const int g = tid / kQGroup, t = tid % kQGroup;
    const uint32_t swz = static_cast<uint32_t>(t & 7);  // 128-byte swizzle phase of rows t and 128 + t
    // stage g's two 16-byte units of a chunk row under the 128-byte swizzle
    const uint32_t rd0 = ((2u * g) ^ swz) << 4, rd1 = ((2u * g + 1u) ^ swz) << 4;
    const bool has_x = t < kPX;
    bool ok = true;
    uint32_t gc = 0;  // chunks consumed so far (all tiles)
    uint32_t ts = 0;  // first stage of the tile, counted over all tiles (the launch keeps it below 2^31)
    for (int64_t tile = pair; tile < ntiles && ok; tile += npairs, ts += static_cast<uint32_t>(nst)) {
      for (int c = 0; c < nch; ++c, ++gc) {
        const int pb = static_cast<int>(gc % kQP);
        const int j = kChunkStages * c + g;           // this group's stage of the chunk
        const bool has = j < nst;
        const uint32_t gs = ts + static_cast<uint32_t>(j);
        const int b = static_cast<int>(gs % kQS);
        ok = bnn::tc::mbar_wait(smem_u32(&chunk_full[pb]), (gc / kQP) & 1u, &abort_flag, &g_bnn_device_errors,
                                wait_limit);
        // refill only after the tensor core has read the previous fill of this buffer
        if (ok && has && gs >= static_cast<uint32_t>(kQS))
          ok = bnn::tc::mbar_wait(smem_u32(&empty_bar[b]), (gs / kQS + 1) & 1u, &abort_flag, &g_bnn_device_errors,
                                  wait_limit);
        if (ok && has) {
          // row r's four words of the stage (eight 32-bit halves) -> units 0..7 of its stage row
          auto expand_row = [&](int r) {
            const uint8_t* ck = chunks + pb * kQChunkBytes + static_cast<uint32_t>(r) * kQRowBytes;
            const uint4 v0 = *reinterpret_cast<const uint4*>(ck + rd0);
            const uint4 v1 = *reinterpret_cast<const uint4*>(ck + rd1);
            uint8_t* dst = smem + b * kQStageBytes + static_cast<uint32_t>(r) * 128u;
            const uint32_t h[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
            for (int u = 0; u < 8; ++u)
              *reinterpret_cast<uint4*>(dst + ((static_cast<uint32_t>(u) ^ swz) << 4)) = nibbles_of(h[u]);
          };
          expand_row(t);
          if (has_x) expand_row(kTm + t);
          asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        }
        // the group's rows of the stage are written (or a wait ran out: the group stops together)
        ok = bnn::tc::named_barrier_and(ok, 2 + g, kQGroup);
        if (!ok) break;
        if (t == 0) {
          mbar_arrive(smem_u32(&chunk_empty[pb]));  // this group is done with the chunk
          if (has) bnn::tc::mbar_arrive_rank(smem_u32(&full_bar[b]), 0u);
        }
      }
    }
  } else if (warp == kQMmaWarp) {
    // ------------------------------------------------------------ MMA issue (CTA 0)
    if (rank == 0 && lane == 0) {
      // D f32; A and B e2m1 (format 1), K-major; ue8m0 scales (bit 23); N = 224, M = 256 (two CTAs);
      // dense K = 64; scale-factor ids 0
      const uint32_t idesc = (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(kPN) >> 3) << 17) | (1u << 23) |
                             ((256u >> 4) << 24);
      const uint32_t sfa = tmem + kQSfCol, sfb = tmem + kQSfCol + 32u;
      bool ok = true;
      for (int64_t tile = pair, ti = 0; tile < ntiles && ok; tile += npairs, ++ti) {
        const int tb = static_cast<int>(ti & 1);
        // the epilogues (both CTAs) have read this buffer's previous tile
        if (ti >= 2)
          ok = bnn::tc::mbar_wait_cluster(smem_u32(&acc_empty[tb]), static_cast<uint32_t>((ti / 2 + 1) & 1),
                                          &abort_flag, &g_bnn_device_errors, wait_limit);
        const uint32_t d = tmem + static_cast<uint32_t>(kPN) * static_cast<uint32_t>(tb);
        for (int j = 0; j < nst && ok; ++j) {
          const uint32_t gs = static_cast<uint32_t>(ti) * static_cast<uint32_t>(nst) + static_cast<uint32_t>(j);
          const int b = static_cast<int>(gs % kQS);
          ok = bnn::tc::mbar_wait_cluster(smem_u32(&full_bar[b]), (gs / kQS) & 1u, &abort_flag,
                                          &g_bnn_device_errors, wait_limit);
          if (!ok) break;
          asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
          const uint64_t ad = sw128_desc(smem_base + b * kQStageBytes);
          const uint64_t bd = sw128_desc(smem_base + b * kQStageBytes + kTm * 128u);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
            asm volatile(
                "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
                "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(
                    d),
                "l"(ad + static_cast<uint64_t>(2 * kk)), "l"(bd + static_cast<uint64_t>(2 * kk)), "r"(idesc),
                "r"(acc), "r"(sfa), "r"(sfb));
          }
          asm volatile(
              "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n" ::
                  "r"(smem_u32(&empty_bar[b])),
              "h"(static_cast<uint16_t>(3))
              : "memory");
        }
        if (!ok) break;
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n" ::"r"(
                smem_u32(&acc_full[tb])),
            "h"(static_cast<uint16_t>(3))
            : "memory");
      }
      // arrives (in both CTAs) once every MMA issued above has completed
      asm volatile(
          "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n" ::"r"(
              smem_u32(&done_bar)),
          "h"(static_cast<uint16_t>(3))
          : "memory");
    }
  } else if (warp == kQTmaWarp) {
    // ------------------------------------------------------------ TMA copies
    if (lane == 0) {
      bnn::pdl_wait();  // the activations may come from the preceding kernel
      uint32_t gc = 0;
      bool ok = true;
      for (int64_t tile = pair; tile < ntiles && ok; tile += npairs) {
        const int j0 = static_cast<int>((tile % ntn) * 256 + 128 * rank);
        const int iq = static_cast<int>((tile / ntn) * kPN + kPX * rank);
        for (int c = 0; c < nch; ++c, ++gc) {
          const int pb = static_cast<int>(gc % kQP);
          if (gc >= static_cast<uint32_t>(kQP) &&
              !bnn::tc::mbar_wait(smem_u32(&chunk_empty[pb]), (gc / kQP + 1) & 1u, &abort_flag,
                                  &g_bnn_device_errors, wait_limit)) {
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(chunks + pb * kQChunkBytes);
          const uint32_t bar = smem_u32(&chunk_full[pb]);
          mbar_expect_tx(bar, kQChunkBytes);
          tma_load_2d(dst, &tmap_w, kQWords * kChunkStages * c, j0, bar);
          tma_load_2d(dst + kTm * kQRowBytes, &tmap_x, kQWords * kChunkStages * c, iq, bar);
        }
      }
      // the CTA must not retire with copies in flight: wait for the last chunk issued into each buffer
      for (uint32_t c = gc >= static_cast<uint32_t>(kQP) ? gc - kQP : 0; c < gc; ++c)
        bnn::tc::mbar_drain(smem_u32(&chunk_full[c % kQP]), (c / kQP) & 1u, &g_bnn_device_errors);
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    // warp ew reads lanes 32 q.. (q = warp % 4) of activation columns
    // [112 h, 112 h + 112), h = ew / 4
    bnn::pdl_wait();  // the row popcounts come from the preceding kernel
    const int et = tid - kQEpiWarp0 * 32;           // 0..255
    const int q = warp & 3;                         // tensor-memory lanes 32q..32q+31
    const int cbeg = (et / 128) * (kPN / 2);        // this warp's first column
    const int erow = 32 * q + lane;
    const uint32_t lane_field = static_cast<uint32_t>(32 * q) << 16;
    const bool need_y = out || next;
    for (int64_t tile = pair, ti = 0; tile < ntiles; tile += npairs, ++ti) {
      const int tb = static_cast<int>(ti & 1);
      const int64_t j0 = (tile % ntn) * 256 + 128 * rank, i0 = (tile / ntn) * kPN;
      const bool ok = bnn::tc::mbar_wait_idle(smem_u32(&acc_full[tb]), static_cast<uint32_t>((ti / 2) & 1),
                                              &abort_flag, &g_bnn_device_errors);
      // the tile's kPN activation-row popcounts (0 past m) into shared memory
      for (int i = et; i < kPN; i += 32 * kQEpi) pop_xs[i] = i0 + i < m ? __ldg(pop_x + i0 + i) : 0;
      if (!bnn::tc::named_barrier_and(ok, kQEpiBar, 32 * kQEpi)) break;  // the epilogue warps stop together
      asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
      const int64_t jrow = j0 + erow;
      const bool jlive = jrow < n;
      const float a_j = (need_y && jlive) ? __ldg(alpha + jrow) : 0.0f;
      const float b_j = (bias && jlive) ? __ldg(bias + jrow) : 0.0f;
      const int base = k - 2 * (jlive ? __ldg(pop_w + jrow) : 0);
      const int64_t half = (j0 + 32 * q) / 32;
      const bool pack = next && half < next_w32;
      const uint32_t taddr = tmem + lane_field + static_cast<uint32_t>(kPN) * static_cast<uint32_t>(tb);
      for (int c0 = cbeg; c0 < cbeg + kPN / 2; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(taddr + static_cast<uint32_t>(c0), r);
        tmem_wait_ld();
        const int64_t rows_left = m - (i0 + c0);
        const int nc = rows_left <= 0 ? 0 : (rows_left < 16 ? static_cast<int>(rows_left) : 16);
        const int64_t off = (i0 + c0) * n + jrow;
        int32_t* dp = dots ? dots + off : nullptr;
        float* op = out ? out + off : nullptr;
        uint32_t* np = pack ? next + (i0 + c0) * next_w32 + half : nullptr;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          // the AND count: an integer of at most 2^24, exact in the float32 accumulator
          const int32_t dv = base - 2 * pop_xs[c0 + c] + 4 * static_cast<int32_t>(__uint_as_float(r[c]));
          const float y0 = __fmul_rn(a_j, static_cast<float>(dv));
          const float y = bias ? __fadd_rn(y0, b_j) : y0;
          if (c < nc && jlive) {
            if (dp) *dp = dv;
            if (op) *op = y;
          }
          if (np) {
            const unsigned bits = __ballot_sync(0xffffffffu, jlive && !(y > 0.0f));
            if (lane == 0 && c < nc) *np = bits;
            np += next_w32;
          }
          dp += n;
          op += n;
        }
      }
      // this CTA's epilogue warps have read the buffer: one arrival on CTA 0's acc_empty
      asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
      asm volatile("bar.sync %0, %1;\n" ::"r"(kQEpiBar), "r"(32 * kQEpi) : "memory");
      if (warp == kQEpiWarp0 && lane == 0) bnn::tc::mbar_arrive_rank(smem_u32(&acc_empty[tb]), 0u);
    }
  }
  __syncwarp();

  // every MMA issued has completed before the tensor memory is freed
  if (tid == 0) bnn::tc::mbar_drain(smem_u32(&done_bar), 0u, &g_bnn_device_errors);
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  cluster.sync();  // neither CTA leaves while the pair's tensor memory or shared memory is in use
  if (warp == kQMmaWarp)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kQTmemCols));
}

// Popcount of every packed row of x (rows 0..m-1) and w (rows m..m+n-1), one
// warp per row, for the CTA-pair kernel's epilogue.
__global__ void row_popcount_kernel(const uint64_t* __restrict__ xp, const uint64_t* __restrict__ wp, int64_t m,
                                    int64_t n, int kw, int* __restrict__ pop) {
  bnn::pdl_trigger();
  bnn::pdl_wait();  // the activations may come from the preceding kernel
  const int lane = threadIdx.x & 31;
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < m + n;
       r += (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) {
    const uint64_t* row = r < m ? xp + r * kw : wp + (r - m) * kw;
    int c = 0;
    for (int i = lane; i < kw; i += 32) c += __popcll(__ldg(row + i));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
    if (lane == 0) pop[r] = c;
  }
}

// Clusters of the pair kernel that fit the GPU at once (cached per context).
int pair_clusters() {
  static std::mutex mu;
  static uint64_t ctx_cached = 0;
  static int cached = 0;
  std::lock_guard<std::mutex> lock(mu);
  const uint64_t ctx = bnn::context_id();
  if (ctx != 0 && ctx == ctx_cached) return cached;
  int num = 0;
  const size_t smem = static_cast<size_t>(kQSmem) + 1024;
  if (bnn::ensure_smem(binary_gemm_pair_kernel, smem) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 128);
    cfg.blockDim = dim3(kQThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&num, binary_gemm_pair_kernel, &cfg) != cudaSuccess) num = 0;
  }
  cudaGetLastError();  // a failed query leaves no error behind
  cached = num;
  ctx_cached = bnn::context_id();
  return num;
}

bnn_status launch_pair(const uint64_t* xp, const uint64_t* wp, const float* alpha, const float* bias, int64_t m,
                       int64_t n, int k, int kw, int32_t* dots, float* out, uint64_t* next, cudaStream_t s,
                       bool* launched) {
  *launched = false;
  const int64_t ntiles = ((n + 255) / 256) * ((m + kPN - 1) / kPN);
  // TMA rows (16-byte aligned: even kw, aligned bases) and int32 coordinates
  // (the AND counts, at most k <= BNN_MAX_K_BINARY = 2^24, are exact in float32)
  if (kw <= 0 || kw % 2 != 0 || !bnn::aligned(xp, 16) || !bnn::aligned(wp, 16) || n >= (1LL << 31) ||
      m >= (1LL << 31))
    return BNN_OK;
  const int clusters = pair_clusters();
  if (clusters <= 0) return BNN_OK;
  // the kernel counts stages over a pair's tiles in 32 bits
  const int64_t nst = (kw + kQWords - 1) / kQWords, per_pair = (ntiles + clusters - 1) / clusters;
  if (per_pair * nst >= (int64_t{1} << 31)) return BNN_OK;
  CUtensorMap tw, tx;
  if (!bnn::encode_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT64, wp, static_cast<uint64_t>(kw),
                           static_cast<uint64_t>(n), static_cast<uint64_t>(kw) * 8u, kQWords * kChunkStages, kTm,
                           CU_TENSOR_MAP_SWIZZLE_128B) ||
      !bnn::encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT64, xp, static_cast<uint64_t>(kw),
                           static_cast<uint64_t>(m), static_cast<uint64_t>(kw) * 8u, kQWords * kChunkStages, kPX,
                           CU_TENSOR_MAP_SWIZZLE_128B))
    return BNN_OK;
  int* pop = nullptr;
  BNN_TRY(bnn::scratch_alloc(reinterpret_cast<void**>(&pop), static_cast<size_t>(m + n) * sizeof(int), s));
  const int64_t warps = m + n, blocks = (warps + 7) / 8;
  const int pgrid = static_cast<int>(blocks < 4 * bnn::sm_count() ? blocks : 4 * bnn::sm_count());
  cudaError_t e = bnn::launch_pdl(row_popcount_kernel, dim3(pgrid), dim3(256), 0, s, 1u, xp, wp, m, n, kw, pop);
  if (e == cudaSuccess) {
    const size_t smem = static_cast<size_t>(kQSmem) + 1024;
    const int64_t np = ntiles < clusters ? ntiles : clusters;
    e = bnn::ensure_smem(binary_gemm_pair_kernel, smem);
    if (e == cudaSuccess)
      e = bnn::launch_pdl(binary_gemm_pair_kernel, dim3(static_cast<unsigned>(2 * np)), dim3(kQThreads), smem, s, 2u,
                          tw, tx, alpha, bias, static_cast<const int*>(pop), static_cast<const int*>(pop + m), m, n,
                          k, kw, dots, out, reinterpret_cast<uint32_t*>(next), 2 * bnn::words64(n),
                          g_wait_limit.load());
  }
  const cudaError_t ef = cudaFreeAsync(pop, s);
  if (e != cudaSuccess) return bnn::cuda_fail(e);
  if (ef != cudaSuccess) return bnn::cuda_fail(ef);
  *launched = true;
  return bnn::check_launch();
}

template <int BN, int KS, bool WIDE = false>
bnn_status launch_tc(const uint64_t* xp, const uint64_t* wp, const float* alpha, const float* bias, int64_t m,
                     int64_t n, int k, int kw, int32_t* dots, float* out, uint64_t* next, cudaStream_t s) {
  const int64_t gx = KS * ((n + kTm - 1) / kTm), gy = (m + BN - 1) / BN;
  if (gx > 2147483647LL || gy > 65535) return BNN_ERR_INVALID_ARG;
  // TMA needs 16-byte aligned rows (even kw, aligned bases) and coordinates that fit int32
  CUtensorMap tw, tx;
  bool tma = kw > 0 && kw % 2 == 0 && bnn::aligned(xp, 16) && bnn::aligned(wp, 16) && n < (1LL << 31) &&
             m < (1LL << 31);
  if (tma)
    tma = bnn::encode_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT64, wp, static_cast<uint64_t>(kw),
                              static_cast<uint64_t>(n), static_cast<uint64_t>(kw) * 8u, kTcWords * kTcChunkStages,
                              kTm, CU_TENSOR_MAP_SWIZZLE_64B) &&
          bnn::encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT64, xp, static_cast<uint64_t>(kw),
                              static_cast<uint64_t>(m), static_cast<uint64_t>(kw) * 8u, kTcWords * kTcChunkStages,
                              BN, CU_TENSOR_MAP_SWIZZLE_64B);
  if (!tma) memset(&tw, 0, sizeof(tw)), memset(&tx, 0, sizeof(tx));
  const size_t smem =
      static_cast<size_t>(tma ? TcCfg<BN, true, WIDE>::kSmem : TcCfg<BN, false, WIDE>::kSmem) + 1024;
  auto kern = tma ? binary_gemm_tc_kernel<BN, KS, true, WIDE> : binary_gemm_tc_kernel<BN, KS, false, WIDE>;
  BNN_TRY(bnn::ensure_smem(kern, smem));
  const cudaError_t e = bnn::launch_pdl(kern, dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)),
                                        dim3(tma ? TcCfg<BN, true, WIDE>::kThreads : TcCfg<BN, false, WIDE>::kThreads),
                                        smem, s,
                                        KS, tw, tx, xp, wp, alpha, bias, m, n, k, kw, dots, out,
                                        reinterpret_cast<uint32_t*>(next), 2 * bnn::words64(n),
                                        g_wait_limit.load());
  if (e != cudaSuccess) return bnn::cuda_fail(e);
  return bnn::check_launch();
}

}  // namespace

namespace bnn {

// Tensor-core (tcgen05) binary GEMM.  m <= 128: 64-row activation tiles (from
// a sweep over M = 64 .. 8192 at N = K = 4096 and 8192); when the tiles leave
// SMs idle a cluster of 4 or 2 CTAs splits each tile's stages (at least 4
// 128-bit stages' worth per CTA).  Larger m: two-SM 256 x 224 tiles when they
// make two waves of CTA pairs or more (16-byte aligned rows); else the one-SM
// plan (activation tile 128 or 256 rows, cluster split 1 or 2) of least
// modelled time: waves x 256-bit stages per CTA x the rows a CTA expands per
// stage (128 + BN), at ~3.3 ns per row-stage, plus ~3 us per 128 activation
// rows of a split's exchange (fitted to 256..1024 x 4096 x 4096 and 256 x 11008
// x 4096, where it picks the measured best).  CTAs that fit one per SM take
// the deep ring (more stages in flight); otherwise 64-row-tile CTAs pair up on
// an SM.
bnn_status binary_gemm_tc(const uint64_t* xp, const uint64_t* wp, const float* alpha, const float* bias, int64_t m,
                          int64_t n, int k, int kw, int32_t* dots, float* out, uint64_t* next, cudaStream_t s) {
  const int64_t wt = (n + kTm - 1) / kTm;
  const int64_t sms = sm_count();
  const int ktiles = (kw + 1) / 2;
  if (m > 128) {
    if (((n + 255) / 256) * ((m + kPN - 1) / kPN) >= sms) {  // at least two waves of 256 x 224 pair tiles
      bool launched = false;
      const bnn_status st = launch_pair(xp, wp, alpha, bias, m, n, k, kw, dots, out, next, s, &launched);
      if (st != BNN_OK || launched) return st;
    }
    const int64_t st = (kw + kTcWords - 1) / kTcWords;  // 256-bit stages
    auto modelled_us = [&](int bn, int ks) -> double {
      const int64_t ctas = ks * wt * ((m + bn - 1) / bn);
      const int64_t waves = (ctas + sms - 1) / sms, per = (st + ks - 1) / ks;
      return static_cast<double>(waves * per * (kTm + bn)) * 3.3e-3 + (ks > 1 ? 3.0 * bn / 128.0 : 0.0);
    };
    int bn = 256, ks = 1;
    double best = modelled_us(256, 1);
    const int plans[3][2] = {{128, 1}, {128, 2}, {256, 2}};
    for (const auto& pl : plans) {
      if (pl[1] > 1 && st < 4 * pl[1]) continue;  // at least 4 stages per CTA of a split
      const double us = modelled_us(pl[0], pl[1]);
      if (us < best) {
        best = us;
        bn = pl[0];
        ks = pl[1];
      }
    }
    const int64_t ctas = ks * wt * ((m + bn - 1) / bn);
    if (bn == 256)
      return ks == 2 ? launch_tc<256, 2>(xp, wp, alpha, bias, m, n, k, kw, dots, out, next, s)
                     : launch_tc<256, 1>(xp, wp, alpha, bias, m, n, k, kw, dots, out, next, s);
    if (ks == 2)
      return ctas <= sms ? launch_tc<128, 2, true>(xp, wp, alpha, bias, m, n, k, kw, dots, out, next, s)
                         : launch_tc<128, 2, false>(xp, wp, alpha, bias, m, n, k, kw, dots, out, next, s);
    return ctas <= sms ? launch_tc<128, 1, true>(xp, wp, alpha, bias, m, n, k, kw, dots, out, next, s)
                       : launch_tc<128, 1, false>(xp, wp, alpha, bias, m, n, k, kw, dots, out, next, s);
  }
  const int64_t tiles = wt * ((m + 63) / 64);
  if (tiles * 4 <= sms && ktiles >= 16)
    return launch_tc<64, 4, true>(xp, wp, alpha, bias, m, n, k, kw, dots, out, next, s);
  if (tiles * 2 <= sms && ktiles >= 8)
    return launch_tc<64, 2, true>(xp, wp, alpha, bias, m, n, k, kw, dots, out, next, s);
  if (tiles * 2 <= 2 * sms && ktiles >= 8)
    return launch_tc<64, 2, false>(xp, wp, alpha, bias, m, n, k, kw, dots, out, next, s);
  if (tiles <= sms) return launch_tc<64, 1, true>(xp, wp, alpha, bias, m, n, k, kw, dots, out, next, s);
  return launch_tc<64, 1, false>(xp, wp, alpha, bias, m, n, k, kw, dots, out, next, s);
}

}  // namespace bnn

namespace bnn {

namespace {
constexpr int kCounterDevices = 64;
struct CounterSlot {
  uint64_t ctx;
  unsigned int* ptr;
};
CounterSlot g_counter[kCounterDevices] = {};
std::mutex g_counter_mu;
}  // namespace

unsigned int* device_error_counter() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kCounterDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_counter_mu);
  const uint64_t ctx = context_id();
  if (ctx == 0 || g_counter[dev].ctx != ctx || !g_counter[dev].ptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bnn_device_errors) != cudaSuccess) return nullptr;
    g_counter[dev] = CounterSlot{context_id(), static_cast<unsigned int*>(p)};
  }
  return g_counter[dev].ptr;
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

extern "C" bnn_status bnn_probe_wait_limit(uint32_t polls) {
  g_wait_limit.store(polls);
  return BNN_OK;
}
