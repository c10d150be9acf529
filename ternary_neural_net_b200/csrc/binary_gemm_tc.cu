// bnn_binary_gemm on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "Binary Math Effectiveness -- why / how / when", section 1: for +-1 vectors
// packed with bit 1 = -1, <x,w> = sum_e x_e w_e = n - 2 popcount(x XOR w).
// +-1 is exact in int8 and the sum is exact in int32, so an int8 MMA over the
// expanded signs computes the same dot as the XOR + popcount identity.
//
// Per CTA: a 128 x BN output tile (UMMA M = 128 activation rows, N = BN weight
// rows), K in stages of 128 bits.  Every thread owns one row of the stacked
// (activation, weight) tile: it loads the row's two 64-bit words of the stage
// (prefetched kTcPre stages ahead in registers), expands the 128 signs to 128
// +-1 bytes in the 128-byte-swizzled K-major shared-memory layout the tensor
// core reads (per 4 bytes: a shift, a sign-replicating byte permute and an
// OR), and one thread issues 4 tcgen05.mma.kind::i8 (K = 32 each) into an
// int32 accumulator in tensor memory, committing to the stage's mbarrier so
// the buffer is refilled only after the tensor core has read it.  Any fixed
// bijection between bits and k-slots gives the same dot when both operands
// use it; the one used makes every 4-byte group a byte permute of one
// shifted 32-bit half-word.  Bits past k (pad bits and zero-filled words)
// are 0 in both operands and each adds exactly +1; the epilogue subtracts
// their count, reads the accumulator back with tcgen05.ld and applies alpha.
//
// Every wait on an mbarrier is bounded; a wait that runs out sets a
// device-side error count (bnn_device_error_count) and the CTA drains its
// MMAs (again bounded), frees its tensor memory and returns.
#include "bnn_internal.cuh"

// Bounded waits that ran out in this file's kernels (read by bnn_device_error_count).
__device__ unsigned int g_bnn_device_errors = 0;

namespace {

constexpr int kTcStages = 4;
constexpr int kTcPre = 8;                  // stages of words prefetched in registers
constexpr int kTcBM = 128;
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

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  for (uint32_t it = 0; it < kSpinLimit; ++it) {
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

// 4 bytes, byte j = -1 where bit 8j+7-s of w is set, else +1.
__device__ __forceinline__ uint32_t pm1_bytes(uint32_t w, int s) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %1, 0xBA98;\n" : "=r"(r) : "r"(w << s));
  return r | 0x01010101u;
}

template <int BN>
__global__ void __launch_bounds__(kTcBM + BN, 1)
binary_gemm_tc_kernel(const uint64_t* __restrict__ xp, const uint64_t* __restrict__ wp,
                      const float* __restrict__ alpha, int64_t m, int64_t n, int k, int kw,
                      int32_t* __restrict__ dots, float* __restrict__ out) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kTcStages];
  __shared__ uint32_t tmem_holder;
  // the 128-byte swizzle repeats every 1024 bytes of address: align the tiles to it
  uint8_t* const smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kTcBM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * BN;
  const int ktiles = (kw + 1) / 2;                 // 2 words (128 bits) per stage

  // this thread's row of the stacked tile
  const bool is_a = tid < kTcBM;
  const int64_t grow = is_a ? m0 + tid : n0 + (tid - kTcBM);
  const bool live = grow < (is_a ? m : n);
  const uint64_t* src = (is_a ? xp : wp) + (live ? grow : 0) * static_cast<int64_t>(kw);
  const uint32_t row_off = is_a ? tid * 128u : kTcBM * 128u * kTcStages + (tid - kTcBM) * 128u;
  // A region: kTcStages x [128 rows x 128 B]; B region after it: kTcStages x [BN rows x 128 B]
  const uint32_t a_stage = kTcBM * 128u, b_stage = BN * 128u;
  const uint32_t swz = static_cast<uint32_t>(tid & 7);

  if (tid == 0) {
    for (int i = 0; i < kTcStages; ++i)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_u32(&bars[i])));
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(&tmem_holder)),
                 "r"(BN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const uint32_t tmem = tmem_holder;

  // instruction descriptor: D s32, A and B s8, both K-major, N = BN, M = 128
  const uint32_t idesc = (2u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(BN) >> 3) << 17) |
                         ((static_cast<uint32_t>(kTcBM) >> 4) << 24);
  const uint32_t smem_base = smem_u32(smem);

  // this row's words, prefetched kTcPre stages ahead into a register ring
  // (the k-loop is unrolled by kTcPre so that every ring index is static)
  auto fetch = [&](int kt, uint64_t& lo, uint64_t& hi) {
    const int w0 = 2 * kt;
    lo = (live && w0 < kw) ? __ldg(src + w0) : 0ull;
    hi = (live && w0 + 1 < kw) ? __ldg(src + w0 + 1) : 0ull;
  };
  uint64_t ring_lo[kTcPre], ring_hi[kTcPre];
#pragma unroll
  for (int u = 0; u < kTcPre; ++u) fetch(u, ring_lo[u], ring_hi[u]);

  bool ok = true;
  int committed = -1;  // last stage whose MMAs were committed (uniform across the CTA)
  for (int kt0 = 0; kt0 < ktiles && ok; kt0 += kTcPre) {
#pragma unroll
    for (int u = 0; u < kTcPre; ++u) {
      const int kt = kt0 + u;
      if (kt >= ktiles || !ok) break;
      const int b = kt % kTcStages;
      // the tensor core must be done with this buffer (stage kt - kTcStages)
      const bool free_ok =
          kt < kTcStages || mbar_wait(smem_u32(&bars[b]), static_cast<uint32_t>((kt / kTcStages - 1) & 1));
      const uint64_t cur[2] = {ring_lo[u], ring_hi[u]};
      if (kt + kTcPre < ktiles) fetch(kt + kTcPre, ring_lo[u], ring_hi[u]);
      if (free_ok) {
        // expand 128 bits -> 128 bytes: half-word h fills 16-byte chunks 2h and 2h+1
        uint8_t* row_ptr = smem + row_off + (is_a ? b * a_stage : b * b_stage);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const uint32_t hw = static_cast<uint32_t>(cur[h >> 1] >> (32 * (h & 1)));
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint4 v;
            v.x = pm1_bytes(hw, 4 * q + 0);
            v.y = pm1_bytes(hw, 4 * q + 1);
            v.z = pm1_bytes(hw, 4 * q + 2);
            v.w = pm1_bytes(hw, 4 * q + 3);
            const uint32_t chunk = static_cast<uint32_t>(2 * h + q);
            *reinterpret_cast<uint4*>(row_ptr + ((chunk ^ swz) << 4)) = v;
          }
        }
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      ok = __syncthreads_and(free_ok) != 0;  // one decision for the whole CTA
      if (!ok) break;
      if (tid == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
        const uint64_t ad = sw128_desc(smem_base + b * a_stage);
        const uint64_t bd = sw128_desc(smem_base + kTcBM * 128u * kTcStages + b * b_stage);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t acc = (kt > 0 || kk > 0) ? 1u : 0u;
          asm volatile(
              "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
              "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
              "l"(ad + static_cast<uint64_t>(2 * kk)), "l"(bd + static_cast<uint64_t>(2 * kk)), "r"(idesc), "r"(acc));
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                         smem_u32(&bars[b]))
                     : "memory");
      }
      committed = kt;
    }
  }
  // the last commit covers every MMA issued before it (second bounded wait after a timeout)
  bool drained = true;
  if (committed >= 0) {
    const uint32_t bar = smem_u32(&bars[committed % kTcStages]);
    const uint32_t par = static_cast<uint32_t>((committed / kTcStages) & 1);
    drained = mbar_wait(bar, par) || mbar_wait(bar, par);
  }
  const bool good = __syncthreads_and(ok && drained) != 0;
  if (!good && tid == 0) atomicAdd(&g_bnn_device_errors, 1u);
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");

  // epilogue: warps 0-3 own TMEM lanes 32w..32w+31 = tile rows; each 32x32
  // block is transposed through shared memory so the stores are row-coalesced
  if (warp < 4 && good) {
    const int pad = ktiles * 128 - k;
    int* tr = reinterpret_cast<int*>(smem) + warp * 32 * 33;  // operand tiles are no longer read
    for (int c0 = 0; c0 < BN; c0 += 32) {
      uint32_t r[32];
      if (ktiles > 0) {
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
#pragma unroll
      for (int c = 0; c < 32; ++c) tr[lane * 33 + c] = static_cast<int>(r[c]) - pad;  // [row][col]
      __syncwarp();
      const int64_t gn = n0 + c0 + lane;
      const float a_n = (out && gn < n) ? __ldg(alpha + gn) : 0.0f;
#pragma unroll 4
      for (int i = 0; i < 32; ++i) {
        const int64_t gm = m0 + warp * 32 + i;
        if (gm < m && gn < n) {
          const int32_t d = tr[i * 33 + lane];
          if (dots) dots[gm * n + gn] = d;
          if (out) out[gm * n + gn] = a_n * static_cast<float>(d);
        }
      }
      __syncwarp();
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(BN));
}

template <int BN>
bnn_status launch_tc(const uint64_t* xp, const uint64_t* wp, const float* alpha, int64_t m, int64_t n, int k, int kw,
                     int32_t* dots, float* out, cudaStream_t s) {
  const int64_t gx = (n + BN - 1) / BN, gy = (m + kTcBM - 1) / kTcBM;
  if (gx > 2147483647LL || gy > 65535) return BNN_ERR_INVALID_ARG;
  const size_t smem = static_cast<size_t>(kTcStages) * (kTcBM + BN) * 128 + 1024;  // + 1024-byte alignment slack
  auto kern = binary_gemm_tc_kernel<BN>;
  BNN_TRY(bnn::ensure_smem(kern, smem));
  kern<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), kTcBM + BN, smem, s>>>(xp, wp, alpha, m, n, k,
                                                                                          kw, dots, out);
  return bnn::check_launch();
}

}  // namespace

namespace bnn {

// Tensor-core (tcgen05) binary GEMM; picks the tile width by problem size.
bnn_status binary_gemm_tc(const uint64_t* xp, const uint64_t* wp, const float* alpha, int64_t m, int64_t n, int k,
                          int kw, int32_t* dots, float* out, cudaStream_t s) {
  const int64_t mt = (m + kTcBM - 1) / kTcBM;
  if (mt * ((n + 255) / 256) >= 2LL * sm_count()) return launch_tc<256>(xp, wp, alpha, m, n, k, kw, dots, out, s);
  if (mt * ((n + 127) / 128) >= sm_count()) return launch_tc<128>(xp, wp, alpha, m, n, k, kw, dots, out, s);
  return launch_tc<64>(xp, wp, alpha, m, n, k, kw, dots, out, s);
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
